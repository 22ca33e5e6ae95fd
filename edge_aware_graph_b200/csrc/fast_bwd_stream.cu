// Backward pair kernel for de = 64, H = 8, dh = 32, bf16 storage (sm_100a).
//
// Chain rule of the layer (formulas as in the forward, differentiated):
//   u_ij^h = We[h,:] . dE'_ij          dA^h_ij = dO_ih . v_jh + u_ij^h
//   D_ih   = sum_j a_ij dA_ij          dS'_ij  = a_ij (dA_ij - D_ih)
//   dgamma = dS' s,  dbeta = dS',  ds = dS' (1 + gamma)
//   dq_i = sum_j ds_ij k_j / sqrt(dh),  dk_j = sum_i ds_ij q_i / sqrt(dh),  dv_j = sum_i a_ij dO_i
//   dE = dE' + [dgamma|dbeta] Wfe^T,  dWfe = sum E^T [dgamma|dbeta],  dWe = sum a^T dE',  dg = sum [dgamma|dbeta]
// with a_ij = exp(s'_ij - LSE_i) from the forward's saved row statistics.
//
// One CTA owns the 8 query rows i of one row block of one graph and streams
// the columns j of those rows in chunks of 32 (256 pairs: two 16 KB E tiles,
// two 16 KB dE' tiles, the 16 KB K and V chunks), twice, because D needs a
// whole row before any dS' exists:
//   pass 1: FiLM f = E Wfe and u = dE' We^T on the tensor cores (tcgen05,
//           fp32 in TMEM), S = Q K^T and dP = dO V^T on warp MMAs, a, dA, and
//           a running D per thread; S and dP stay in TMEM for pass 2 (32
//           columns per chunk, n <= 224; larger n reloads K and V);
//   pass 2: (the chunks in reverse, so that E and dE' come back from L2) dS',
//           dgamma, dbeta, ds; dWfe += E^T df and dWe^T += dE'^T a on the
//           tensor cores (MN-major operands straight from the tiles,
//           accumulated in TMEM over the row block); dE = dE' + df Wfe^T on the
//           tensor cores, added in place to the dE' tile once those products
//           have read it, and stored with TMA;
//           dq += ds K (warp MMAs); and the row block's share of dk_j, dv_j for
//           the chunk's columns (warp MMAs over the 8 rows), added into fp32
//           accumulators [B,n,H*dh] with vector reductions in L2.
// E and dE' leave HBM once, dE is written once, and no per-pair quantity is
// written anywhere: no [B,H,n,n] array.  The dk, dv sums over row blocks
// arrive in whatever order the CTAs run (fp32 additions: the last bits of dk,
// dv may differ from run to run); everything else is summed in a fixed order.
// No CTA waits for another.
//
// Block sparsity, as in the forward: a chunk with no valid pair adds nothing
// to D, dq, dk, dv, dg or the weight gradients, and its dE is its dE'.  The
// TMA warp copies its dE' tiles to dE; no other warp sees it.
//
// Warp roles as in the forward pair kernel: 16 compute warps (warp W reads
// TMEM quadrant W%4 and handles heads 2(W/4), 2(W/4)+1), one MMA warp (FiLM
// and u one chunk ahead into double-buffered TMEM ranges, dE and the weight
// gradients when the compute warps have written df), one TMA warp (a ring of
// twelve 16 KB slots, dE stores).  They meet only on mbarriers.  The pair <->
// lane mapping is the forward's: row 4j + ic of E tile s is the pair (j, i =
// 2ic + s), which lane t of quadrant q = j/8 holds in accumulator register s
// of its m16n8 tile S^T[j, i].
#include <math.h>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using namespace dev;

constexpr int BS_SLOTS = 12;
constexpr uint32_t BS_SLOT = 16384;
constexpr int BS_NFULL = 4;
constexpr int BS_THR = NTHR + 64;
constexpr int BS_KEEP_MAX_CHUNKS = 7;     // S and dP of up to 7 chunks (n <= 224) stay in TMEM

struct BsSmem {
    // offsets from a 1024-aligned base
    static constexpr uint32_t IMG = BS_SLOTS * BS_SLOT;       // Wfe^T sw (FiLM), We sw (u), Wfe ns (dE): 2 KB each
    static constexpr uint32_t DA = IMG + 6144;                // 2 tiles [128][32] ns: [dgamma | dbeta | a | 0]
    static constexpr uint32_t WD = DA + 16384;                // per-quadrant D [4][8 i][8 h]
    static constexpr uint32_t WDG = WD + 1024;                // per-warp dg [16][4]
    static constexpr uint32_t G = WDG + 256;                  // g_b [16]
    static constexpr uint32_t MJ = G + 64;                    // node mask [n <= 1024]
    static constexpr uint32_t BAR = MJ + 1024;
    static constexpr uint32_t TM = BAR + 8 * 21;              // TMEM base address
    static constexpr uint32_t FAIL = TM + 4;                  // CTA failure flag (a wait ran out)
    static constexpr uint32_t STAB = TM + 16;                 // slot table [4 live iterations][8] u8
    static constexpr uint32_t CTAB = STAB + 32;               // slots of the copies [4][2] u8
    static constexpr uint32_t LIVE = CTAB + 8;                // live-chunk mask of the row block
    static constexpr uint32_t LC = LIVE + 8;                  // the live chunks, ascending [32] u8
    static constexpr uint32_t DC = LC + 32;                   // the dead chunks, ascending [32] u8
    static constexpr uint32_t BYTES = DC + 32 + 1024;
    // after pass 2, in the DA tiles: dq quadrant sums of four heads [4][8][128] f32 (16 KB)
};
// mbarriers: full[4] (loads of live iterations), film_full[2], film_empty[2], df_full, de_full,
// stage_done[4], mma_final, wg_done[2] (the weight-gradient products of pass-2 live chunk p2,
// by p2 & 1), copy[4] (loads of dead chunks)
constexpr int BB_FULL = 0, BB_FILM_FULL = 4, BB_FILM_EMPTY = 6, BB_DF_FULL = 8, BB_DE_FULL = 9,
              BB_STAGE_DONE = 10, BB_MMA_FINAL = 14, BB_WG_DONE = 15, BB_COPY = 17;
constexpr int BS_NCOPY = 4;               // dead-chunk copies in flight

// TMEM: FiLM 0..63 and u 64..127 (two buffers each), dE 128..255, kept S / dP
// 256..479 (32 per chunk), and at 480 the weight-gradient accumulator
// [E | dE']^T [df | a]: lanes 0..63 the E channels, 64..127 the dE' channels,
// columns 0..31 the df and a columns; its blocks E^T df = dWfe [c][k] and
// dE'^T a = dWe^T [c][h] are the ones used
constexpr uint32_t BS_TM_COLS = 512, BS_TM_FILM = 0, BS_TM_U = 64, BS_TM_DE = 128, BS_TM_KEEP = 256,
                   BS_TM_W = 480;

// Byte offset of element (row, col) of a [128][32] bf16 tile in 8 x 8 core
// matrices: 128 B apart along the columns, 512 B along the rows.
__device__ __forceinline__ uint32_t ns32(uint32_t row, uint32_t col) {
    return (row >> 3) * 512u + (col >> 3) * 128u + (row & 7u) * 16u + (col & 7u) * 2u;
}

struct BwdStreamParams {
    const int *order;        // [B * row blocks]: the row block each CTA takes (longest first)
    const __nv_bfloat16 *Q, *dO;
    const float *LSE, *g;
    const uint8_t *img, *M;
    __nv_bfloat16 *dQ;       // [B,n,256] out (scaled by 1/sqrt(dh))
    __nv_bfloat16 *dE;       // [B,n,n,64] out
    float *rparts;           // [graph * row block][RPART] out
    float *dK32, *dV32;      // [B,n,256] fp32 accumulators of dk (unscaled), dv (zero at launch)
    int *status;
    int n;
    int row0, rows;          // the slab of rows this call owns (E, dE', dE hold rows row0 .. row0+rows-1)
    int light;               // Light Edge variant: no per-edge FiLM map; E is not read, dE = dE'
    int unnorm;              // unnormalised variant: the edge path reaches s' directly
    uint32_t prefetch_ahead;   // CTAs between this one and the one whose first tiles it prefetches
};

// 576 threads (18 warps): five warps share one of the four 16K-register sub-partitions,
// so at most 96 registers a thread
__global__ void __launch_bounds__(BS_THR, 1)
k_bwd_stream(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmDEp,
             const __grid_constant__ CUtensorMap tmDE, const __grid_constant__ CUtensorMap tmK,
             const __grid_constant__ CUtensorMap tmV, BwdStreamParams p) {
    using S = BsSmem;
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, W = tid >> 5, q = W & 3, hq = (W >> 2) & 3, t = tid & 31, c4 = t & 3, g8 = t >> 2;
    const int n = p.n, nch = (n + 31) / 32;
    // i0: the row block's first row in the graph; i0l: in the slab (E, dE', dE
    // rows); item: the row block's partials, (graph, row block of the graph)
    // the row block this CTA takes: longest first (k_row_block_order), so that
    // the short ones fill the last wave
    const int nrb = gridDim.x, ord = p.order[blockIdx.y * gridDim.x + blockIdx.x];
    const int b = ord / nrb, i0l = (ord % nrb) * TB, i0 = p.row0 + i0l;
    const int item = b * ((n + TB - 1) / TB) + i0 / TB;
    const uint32_t bars = sbase + S::BAR;
    auto bar = [&](int k) { return bars + 8 * k; };
    float *g = reinterpret_cast<float *>(sp + S::G);
    uint8_t *mj = sp + S::MJ;
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);

    // Block sparsity: a chunk holding no valid pair (live_chunk_mask) adds
    // nothing to any sum and its dE is its dE'.  The TMA warp loads iterations
    // it in order: pass 1 the nl live chunks, ascending; pass 2 the live
    // chunks, descending; then the copies of the dead ones (two dE' tiles
    // loaded and stored as dE).  The live iterations li = 0
    // .. 2 nl - 1 (pass 1, then pass 2's live chunks) are the ones the MMA and
    // compute warps see.  Tiles of a live iteration: E(s=0), E(s=1), dE'(s=0),
    // dE'(s=1), K, then V in pass 1 (and in pass 2 when S, dP are not kept).
    // The TMA warp places each tile in any free slot and records the slot in
    // table entry li % 4, which the other warps read after the load barrier.
    const bool keep = nch <= BS_KEEP_MAX_CHUNKS;
    const bool light = p.light != 0, unnorm = p.unnorm != 0;
    const int ns2 = keep ? 5 : 6;
    volatile uint8_t *stab = sp + S::STAB;
    auto slot_addr = [&](int li, int k) { return sbase + (uint32_t)stab[(li % BS_NFULL) * 8 + k] * BS_SLOT; };

    // ---------------- setup: barriers, TMEM, operands
    if (tid == 0) {
        for (int k = 0; k < BS_NFULL; ++k) mbar_init(bar(BB_FULL + k), 1);
        mbar_init(bar(BB_FILM_FULL), 1);
        mbar_init(bar(BB_FILM_FULL + 1), 1);
        mbar_init(bar(BB_FILM_EMPTY), NWARP);
        mbar_init(bar(BB_FILM_EMPTY + 1), NWARP);
        mbar_init(bar(BB_DF_FULL), NWARP);
        mbar_init(bar(BB_DE_FULL), 1);
        for (int k = 0; k < 4; ++k) mbar_init(bar(BB_STAGE_DONE + k), NWARP);
        mbar_init(bar(BB_MMA_FINAL), 1);
        mbar_init(bar(BB_WG_DONE), 1);
        mbar_init(bar(BB_WG_DONE + 1), 1);
        for (int k = 0; k < BS_NCOPY; ++k) mbar_init(bar(BB_COPY + k), 1);
        fence_mbar_init();
        *fail = 0;
    }
    if (W == 0) {
        tmem_alloc(sbase + S::TM, BS_TM_COLS);
        tmem_relinquish();
    }
    if (W == 1) {
        const uint32_t lm = live_chunk_mask(p.M, b, n, i0, t);
        if (t == 0) *reinterpret_cast<volatile uint32_t *>(sp + S::LIVE) = lm;
        const int below = __popc(lm & ((1u << t) - 1u));   // live chunks below chunk t
        if ((lm >> t) & 1u) sp[S::LC + below] = (uint8_t)t;
        else if (t < nch) sp[S::DC + t - below] = (uint8_t)t;
    }
    if (tid < 384) {
        const uint32_t img_off = (tid >> 7) == 0 ? IMG_WFE_T_SW : (tid >> 7) == 1 ? IMG_WE_SW : IMG_WFE_NS;
        reinterpret_cast<uint4 *>(sp + S::IMG)[tid] = reinterpret_cast<const uint4 *>(p.img)[(img_off >> 4) + (tid & 127)];
    }
    // [df | a] tiles: columns 24..31 (a of h >= 8) stay zero
    for (int e = tid; e < 16384 / 16; e += BS_THR) reinterpret_cast<uint4 *>(sp + S::DA)[e] = make_uint4(0, 0, 0, 0);
    if (tid < NF) g[tid] = p.g[(size_t)b * NF + tid];
    for (int j = tid; j < 32 * nch; j += BS_THR) mj[j] = j < n ? p.M[(size_t)b * n + j] : 0;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const uint32_t live = *reinterpret_cast<volatile uint32_t *>(sp + S::LIVE);
    const int nl = __popc(live), nit = 2 * nl, nload = nl + nch;
    const volatile uint8_t *lc = sp + S::LC;
    // chunk of live iteration li; chunk of load iteration it
    auto chunk_of_li = [&](int li) { return (int)lc[li < nl ? li : nit - 1 - li]; };
    // Load order: pass 1 (the live chunks, ascending), pass 2 (the live chunks,
    // descending), then the copies of the dead chunks, which stream at the CTA's
    // end while the last live chunks are computed (measured faster than copies
    // taken between the pass-1 chunks, which hold ring slots that pass 1 needs,
    // and than one copy after each pass-2 chunk: 0.147 against 0.141 ms on the
    // SBM batch).
    const volatile uint8_t *dc = sp + S::DC;
    auto is_live = [&](int it) { return it < nit; };
    auto chunk_of_it = [&](int it) { return it < nl ? (int)lc[it] : it < nit ? (int)lc[nit - 1 - it] : (int)dc[it - nit]; };

    if (W == NWARP) {
        // ================= MMA issuer
        if (t == 0) {
            const uint32_t idesc_f = idesc_bf16_f32(128, NF), idesc_d = idesc_bf16_f32(128, DE);
            const uint32_t idesc_w = idesc_bf16_f32_mn(128, 2 * NF);
            auto issue_fu = [&](int li) {
                tc_fence_after();
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const uint32_t ae = slot_addr(li, s), ad = slot_addr(li, 2 + s);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        if (!light)   // Light Edge: no FiLM product (its E tiles are not loaded)
                            mma_bf16_ss(tmem + BS_TM_FILM + 32 * (li & 1) + 16 * s,
                                        smem_desc(ae + kk * 32, 16, 1024, LAYOUT_SW128),
                                        smem_desc(sbase + S::IMG + kk * 32, 16, 1024, LAYOUT_SW128), idesc_f, kk > 0);
                        mma_bf16_ss(tmem + BS_TM_U + 32 * (li & 1) + 16 * s,
                                    smem_desc(ad + kk * 32, 16, 1024, LAYOUT_SW128),
                                    smem_desc(sbase + S::IMG + 2048 + kk * 32, 16, 1024, LAYOUT_SW128), idesc_f,
                                    kk > 0);
                    }
                }
                mma_commit(bar(BB_FILM_FULL + (li & 1)));
            };
            auto issue_de = [&](int li) {
                tc_fence_after();
                if (!light)   // Light Edge: df Wfe^T = 0, dE = dE'
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        mma_bf16_ss(tmem + BS_TM_DE + 64 * e,
                                    smem_desc(sbase + S::DA + e * 8192, 128, 512, LAYOUT_NONE),
                                    smem_desc(sbase + S::IMG + 4096, 128, 256, LAYOUT_NONE), idesc_d, 0);
                // dE alone is on the compute warps' path: its own completion
                mma_commit(bar(BB_DE_FULL));
                // [dWfe | .] and [. | dWe^T] in one product: A = the E tile and the dE' tile read
                // MN-major as the two 64-channel atoms of M = 128 (64 c per 128-byte swizzled row,
                // 8-row groups 1024 B apart; the second atom one slot distance further: the
                // TMA warp hands out slots in increasing order, so the dE' slot of a parity
                // half lies above its E slot); B = the [df | a] tile read MN-major (8 x 8 core
                // matrices: 128 B along N, 512 B along K); 16 pairs per MMA
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t te = slot_addr(li, e), td = slot_addr(li, 2 + e);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t acc = (li > nl || e > 0 || ks > 0) ? 1u : 0u;
                        mma_bf16_ss(tmem + BS_TM_W, smem_desc(te + ks * 2048, td - te, 1024, LAYOUT_SW128),
                                    smem_desc(sbase + S::DA + e * 8192 + ks * 1024, 512, 128, LAYOUT_NONE), idesc_w, acc);
                    }
                }
                // the tiles (E, dE', [df | a]) may be reused once these completed
                mma_commit(bar(BB_WG_DONE + ((li - nl) & 1)));
            };
            // issue whichever product is ready first: FiLM/u of the next chunk
            // (its tiles landed, its TMEM buffer released) or dE of the pass-2
            // chunk whose df the compute warps have written
            int next_fu = 0, next_de = nl;
            uint32_t polls = 0;
            while ((next_fu < nit || next_de < nit) && !*fail) {
                bool progressed = false;
                if (next_fu < nit && mbar_test_wait(bar(BB_FULL + next_fu % BS_NFULL), (next_fu / BS_NFULL) & 1) &&
                    (next_fu < 2 || mbar_test_wait(bar(BB_FILM_EMPTY + (next_fu & 1)), ((next_fu - 2) >> 1) & 1))) {
                    issue_fu(next_fu++);
                    progressed = true;
                }
                if (next_de < nit && next_de < next_fu && mbar_test_wait(bar(BB_DF_FULL), (next_de - nl) & 1)) {
                    issue_de(next_de);
                    ++next_de;
                    progressed = true;
                }
                // idle: back off after a few polls, so that this thread does not
                // take issue slots from the compute warps of its SM sub-partition;
                // a wait that makes no progress for 2^24 polls gives up
                if (progressed) {
                    polls = 0;
                } else {
                    if (++polls > (1u << 24)) {
                        *fail = 1;
                        flag_timeout(p.status);
                        break;
                    }
                    if (polls > 8) __nanosleep(64);
                }
            }
            // every product issued has completed before the tensor memory is freed
            mma_commit(bar(BB_MMA_FINAL));
            if (!mbar_wait(bar(BB_MMA_FINAL), 0)) flag_timeout(p.status);
        }
        __syncwarp();
        named_bar_sync(2, BS_THR);
    } else if (W == NWARP + 1) {
        // ================= TMA: loads into the slot ring, copies of dead chunks
        if (t == 0) {
            // E and dE' tiles loaded in pass 1 are read again in pass 2: keep
            // them in L2; pass-2 reads are not read again
            const uint64_t keep_l2 = l2_evict_last(), drop_l2 = l2_evict_first();
            volatile uint8_t *ctab = sp + S::CTAB;
            // a live chunk's slots are free once the compute warps are done with
            // it (and, in pass 2, its weight-gradient products have read the
            // tiles); a copy's once its store has read them
            uint32_t free_mask = (1u << BS_SLOTS) - 1u;
            auto take_slot = [&]() {
                const int sidx = __ffs(free_mask) - 1;
                free_mask &= free_mask - 1u;
                return (uint8_t)sidx;
            };
            // loads go out in iteration order; a live iteration waits for its
            // load barrier to be free (at most BS_NFULL live iterations in
            // flight), a copy likewise for its copy barrier
            int next_load = 0, load_li = 0, load_dk = 0, done_li = 0, done_dk = 0;
            auto issue_loads = [&]() {
                while (next_load < nload && !*fail) {
                    const int it = next_load, x0 = 32 * chunk_of_it(it);
                    const bool pass2 = it >= nl && it < nit;
                    if (is_live(it)) {
                        const int li = load_li, ns = pass2 ? ns2 : 6;
                        if (li >= done_li + BS_NFULL || __popc(free_mask) < ns) break;
                        // slots in increasing order: each dE' slot lies above the E slot of its parity
                        for (int k = 0; k < ns; ++k) stab[(li % BS_NFULL) * 8 + k] = take_slot();
                        const uint32_t fb = bar(BB_FULL + li % BS_NFULL);
                        // (Light Edge: the E tiles' slots are taken but not loaded)
                        mbar_expect_tx(fb, (ns - (light ? 2 : 0)) * BS_SLOT);   // releases the table entry too
                        const uint64_t pol = pass2 ? drop_l2 : keep_l2;
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            if (!light) tma_load_5d_hint(slot_addr(li, s), &tmE, fb, 0, i0l / 2, x0, s, b, pol);
                            tma_load_5d_hint(slot_addr(li, 2 + s), &tmDEp, fb, 0, i0l / 2, x0, s, b, pol);
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            tma_load_3d(slot_addr(li, 4) + k * 4096, &tmK, fb, 64 * k, x0, b);
                            if (!pass2 || !keep) tma_load_3d(slot_addr(li, 5) + k * 4096, &tmV, fb, 64 * k, x0, b);
                        }
                        ++load_li;
                    } else {
                        const int dk = load_dk;
                        if (dk >= done_dk + BS_NCOPY || __popc(free_mask) < 2) break;
                        const uint32_t cb = bar(BB_COPY + dk % BS_NCOPY);
                        mbar_expect_tx(cb, 2 * BS_SLOT);
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            const uint8_t sl = take_slot();
                            ctab[(dk % BS_NCOPY) * 2 + s] = sl;
                            tma_load_5d_hint(sbase + sl * BS_SLOT, &tmDEp, cb, 0, i0l / 2, x0, s, b, drop_l2);
                        }
                        ++load_dk;
                    }
                    ++next_load;
                }
            };
            issue_loads();
            uint32_t pend_mask = 0u;   // slots of the last dE store, not yet known to have read them
            for (int it = 0; it < nload; ++it) {
                if (it == nl && p.prefetch_ahead) {
                    // L2 prefetch of the first tiles of the CTA that runs about one wave later
                    const uint32_t cid = blockIdx.y * gridDim.x + blockIdx.x + p.prefetch_ahead;
                    if (cid < gridDim.x * gridDim.y) {
                        const int pord = p.order[cid], prb = pord % nrb, pb = pord / nrb;
                        for (int cc = 0; cc < nch && cc < 2; ++cc) {
                            if (!light) {
                                tma_prefetch_5d(&tmE, 0, prb * TB / 2, 32 * cc, 0, pb);
                                tma_prefetch_5d(&tmE, 0, prb * TB / 2, 32 * cc, 1, pb);
                            }
                            tma_prefetch_5d(&tmDEp, 0, prb * TB / 2, 32 * cc, 0, pb);
                            tma_prefetch_5d(&tmDEp, 0, prb * TB / 2, 32 * cc, 1, pb);
                        }
                    }
                }
                uint32_t s0, s1;   // the slots of the two dE tiles a store reads
                const bool pass2 = it >= nl && it < nit;
                if (is_live(it)) {
                    const int li = done_li++;
                    if (!cta_wait(bar(BB_STAGE_DONE + (li & 3)), (li >> 2) & 1, fail, p.status)) continue;
                    if (pass2) {
                        // the chunk's tiles are read by its weight-gradient products until these complete
                        const int p2 = li - nl;
                        if (!cta_wait(bar(BB_WG_DONE + (p2 & 1)), (p2 >> 1) & 1, fail, p.status)) continue;
                    }
                    // pass 2: the dE' tiles (now dE) are stored first; the other slots are free
                    for (int k = 0; k < (pass2 ? ns2 : 6); ++k)
                        if (!pass2 || (k != 2 && k != 3)) free_mask |= 1u << stab[(li % BS_NFULL) * 8 + k];
                    s0 = stab[(li % BS_NFULL) * 8 + 2];
                    s1 = stab[(li % BS_NFULL) * 8 + 3];
                } else {
                    const int dk = done_dk++;
                    if (!cta_wait(bar(BB_COPY + dk % BS_NCOPY), (dk / BS_NCOPY) & 1, fail, p.status)) continue;
                    s0 = ctab[(dk % BS_NCOPY) * 2];
                    s1 = ctab[(dk % BS_NCOPY) * 2 + 1];
                }
                if (pass2 || !is_live(it)) {
                    const int x0 = 32 * chunk_of_it(it);
                    tma_store_5d_hint(&tmDE, sbase + s0 * BS_SLOT, 0, i0l / 2, x0, 0, b, drop_l2);
                    tma_store_5d_hint(&tmDE, sbase + s1 * BS_SLOT, 0, i0l / 2, x0, 1, b, drop_l2);
                    tma_store_commit();
                    if (keep) {
                        // the previous store's slots are free once it has read them
                        if (pend_mask) {
                            tma_store_wait_read1();
                            free_mask |= pend_mask;
                        }
                        pend_mask = (1u << s0) | (1u << s1);
                    } else {
                        // six slots a pass-2 chunk: two chunks in flight only if this
                        // store's slots come back before the next loads
                        tma_store_wait_read0();
                        free_mask |= pend_mask | (1u << s0) | (1u << s1);
                        pend_mask = 0u;
                    }
                }
                issue_loads();
            }
            tma_store_wait_read0();
            if (*fail) {   // loads already issued land before the CTA's shared memory is released
                for (int li = max(load_li - BS_NFULL, 0); li < load_li; ++li)
                    mbar_wait(bar(BB_FULL + li % BS_NFULL), (li / BS_NFULL) & 1);
                for (int dk = max(load_dk - BS_NCOPY, 0); dk < load_dk; ++dk)
                    mbar_wait(bar(BB_COPY + dk % BS_NCOPY), (dk / BS_NCOPY) & 1);
            }
        }
        __syncwarp();
        named_bar_sync(2, BS_THR);   // the ring is drained: the compute warps may reuse it
    } else if (nl == 0) {
        // ================= compute warps of a row block without a valid pair: dq of
        // its rows and its weight-gradient partials are zero, no passes
        for (int x = tid; x < TB * HD / 8; x += NTHR) {
            const int il = x / (HD / 8), d = (x % (HD / 8)) * 8;
            if (i0 + il < n)
                *reinterpret_cast<uint4 *>(p.dQ + ((size_t)b * n + i0 + il) * HD + d) = make_uint4(0u, 0u, 0u, 0u);
        }
        float *rp = p.rparts + (size_t)item * RPART;
        for (int x = tid; x < RPART; x += NTHR) rp[x] = 0.f;
        named_bar_sync(2, BS_THR);   // the TMA warp has stored the copies
    } else {
        // ================= compute warps
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const float rs = rsqrtf((float)DH);
        const uint32_t L = 32 * q + t;
        bool mrow[2];            // the CTA's own nodes i0 + 2c4 + e: rows in passes 1-2, columns in pass 3
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = i0 + 2 * c4 + e;
            mrow[e] = i < n && p.M[(size_t)b * n + i] != 0;
        }
        {
            // ======== passes 1 and 2: the CTA's rows
            uint32_t qf[2][2][2], of[2][2][2];
            load_frags2(p.Q, b, n, i0, hq, g8, c4, qf);
            load_frags2(p.dO, b, n, i0, hq, g8, c4, of);
            float lse[2][2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int i = i0 + 2 * c4 + e;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) lse[e][hh] = i < n ? p.LSE[((size_t)b * NH + 2 * hq + hh) * n + i] : 0.f;
            }
            float dsum[2][2] = {{0.f, 0.f}, {0.f, 0.f}};     // running D partial, then the final D [e][hh]
            float qacc[2][2][4];
            float dgp[4] = {0.f, 0.f, 0.f, 0.f};              // dgamma h0, h1, dbeta h0, h1
#pragma unroll
            for (int x = 0; x < 4; ++x)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) qacc[hh][0][x] = qacc[hh][1][x] = 0.f;

            for (int li = 0; li < nit; ++li) {
                const int c = chunk_of_li(li), j0 = 32 * c;
                const bool pass2 = li >= nl;

                if (li == nl) {
                    // ---------------- D over lanes, then quadrants
                    tmem_st_wait();
                    float *wd = reinterpret_cast<float *>(sp + S::WD);
#pragma unroll
                    for (int e = 0; e < 2; ++e)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            float x = dsum[e][hh];
                            x += __shfl_xor_sync(0xffffffffu, x, 4);
                            x += __shfl_xor_sync(0xffffffffu, x, 8);
                            x += __shfl_xor_sync(0xffffffffu, x, 16);
                            if (g8 == 0) wd[(q * 8 + 2 * c4 + e) * 8 + 2 * hq + hh] = x;
                        }
                    named_bar_sync(1, NTHR);
#pragma unroll
                    for (int e = 0; e < 2; ++e)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int o = (2 * c4 + e) * 8 + 2 * hq + hh;
                            dsum[e][hh] = wd[o] + wd[64 + o] + wd[128 + o] + wd[192 + o];
                        }
                }

                cta_wait(bar(BB_FULL + li % BS_NFULL), (li / BS_NFULL) & 1, fail, p.status);
                // ---------------- S = Q K^T, dP = dO V^T (warp MMAs), or the kept ones
                float sv[2][4], da[2][4];
                const uint32_t kcol = tl + BS_TM_KEEP + 32 * c + 2 * hq;
                if (pass2 && keep) {
                    tmem_ld2(kcol, sv[0][0], sv[1][0]);
                    tmem_ld2(kcol + 8, sv[0][1], sv[1][1]);
                    tmem_ld2(kcol + 16, da[0][0], da[1][0]);
                    tmem_ld2(kcol + 24, da[0][1], da[1][1]);
                    tmem_ld_wait();
                } else {
                    warp_scores2<1>(slot_addr(li, 4), q, t, hq, qf, sv);
                    warp_scores2<1>(slot_addr(li, 5), q, t, hq, of, da);
                    if (keep) {
                        tmem_st2(kcol, sv[0][0], sv[1][0]);
                        tmem_st2(kcol + 8, sv[0][1], sv[1][1]);
                        tmem_st2(kcol + 16, da[0][0], da[1][0]);
                        tmem_st2(kcol + 24, da[0][1], da[1][1]);
                    }
                }

                // ---------------- FiLM and u from TMEM
                cta_wait(bar(BB_FILM_FULL + (li & 1)), (li >> 1) & 1, fail, p.status);
                tc_fence_after();
                float fg[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, fb[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, fu[2][2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const uint32_t fcol = BS_TM_FILM + 32 * (li & 1) + 16 * e, ucol = BS_TM_U + 32 * (li & 1) + 16 * e;
                    if (!light) {   // Light Edge: gamma, beta from y alone
                        tmem_ld2(tl + fcol + 2 * hq, fg[e][0], fg[e][1]);
                        tmem_ld2(tl + fcol + NH + 2 * hq, fb[e][0], fb[e][1]);
                    }
                    tmem_ld2(tl + ucol + 2 * hq, fu[e][0], fu[e][1]);
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (t == 0) mbar_arrive(bar(BB_FILM_EMPTY + (li & 1)));
                const bool mcol = mj[j0 + 8 * q + g8] != 0;
                // av: a; sv: s; gm: gamma; da: dA (the layer) or dP with the edge
                // term u in fu (the unnormalised variant: u enters dS' directly)
                // and the modulated score in fb (for dWe)
                float av[2][4], gm[2][4];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool valid = mcol && mrow[e];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int h = 2 * hq + hh;
                        const float s = sv[hh][e] * rs;
                        const float gam = fg[e][hh] + g[h], bet = fb[e][hh] + g[NH + h];
                        const float spv = s * (1.f + gam) + bet;
                        av[hh][e] = valid ? exp2f((spv - lse[e][hh]) * LOG2E) : 0.f;
                        sv[hh][e] = s;
                        gm[hh][e] = gam;
                        if (unnorm) {
                            fu[e][hh] = valid ? fu[e][hh] : 0.f;
                            fb[e][hh] = valid ? spv : 0.f;
                        } else {
                            da[hh][e] += fu[e][hh];
                        }
                    }
                }

                if (!pass2) {
#pragma unroll
                    for (int e = 0; e < 2; ++e)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) dsum[e][hh] += av[hh][e] * da[hh][e];
                    __syncwarp();
                    if (t == 0) mbar_arrive(bar(BB_STAGE_DONE + (li & 3)));
                    continue;
                }

                // ---------------- pass 2: dS', df and a tiles for the tensor cores / warp MMAs;
                // the previous chunk's weight-gradient products read the tile until they complete
                if (li > nl) cta_wait(bar(BB_WG_DONE + ((li - nl - 1) & 1)), ((li - nl - 1) >> 1) & 1, fail, p.status);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float dgam[2], dbet[2];
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float dsp = av[hh][e] * (da[hh][e] - dsum[e][hh]) + (unnorm ? fu[e][hh] : 0.f);
                        dgam[hh] = dsp * sv[hh][e];
                        dbet[hh] = dsp;
                        da[hh][e] = dsp * (1.f + gm[hh][e]);     // ds (unscaled)
                        dgp[hh] += dgam[hh];
                        dgp[2 + hh] += dbet[hh];
                    }
                    *reinterpret_cast<uint32_t *>(sp + S::DA + e * 8192 + ns32(L, 2 * hq)) = pack_bf16(dgam[0], dgam[1]);
                    *reinterpret_cast<uint32_t *>(sp + S::DA + e * 8192 + ns32(L, NH + 2 * hq)) = pack_bf16(dbet[0], dbet[1]);
                    // the coefficients the edge update used: a, or s' (unnormalised)
                    *reinterpret_cast<uint32_t *>(sp + S::DA + e * 8192 + ns32(L, NF + 2 * hq)) =
                        unnorm ? pack_bf16(fb[e][0], fb[e][1]) : pack_bf16(av[0][e], av[1][e]);
                }
                da[0][2] = da[0][3] = da[1][2] = da[1][3] = 0.f;
                // df and a of this warp's rows are in place: the MMA warp issues dE and
                // the weight-gradient products once all 16 warps have arrived
                fence_proxy_async_smem();
                __syncwarp();
                if (t == 0) mbar_arrive(bar(BB_DF_FULL));

                // ---------------- dq += ds K (warp MMAs; overlaps the tensor-core products)
                warp_contract2<1, true>(slot_addr(li, 4), q, t, hq, da, qacc);

                // ---------------- the row block's share of dk_j = sum_i ds_ij q_i and dv_j =
                // sum_i a_ij dO_i for the warp's 8 columns j (two heads): warp MMAs with M = j,
                // K = i (the 8 rows), N = 8 features.  A is the score tile's own fragment (row
                // j, columns i), B the transposed Q / dO fragment of the rows; the two lanes of
                // a pair (c4, c4 ^ 1) swap halves so that each adds four consecutive features
                // with one vector reduction: even lanes dk, odd lanes dv.
                {
                    const int j = j0 + 8 * q + g8;
                    const bool live = j < n && mj[j];        // masked columns get nothing
                    const bool even = (c4 & 1) == 0;
                    float *rowk = p.dK32 + ((size_t)b * n + (live ? j : 0)) * HD;
                    float *rowv = p.dV32 + ((size_t)b * n + (live ? j : 0)) * HD;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const uint32_t ak[4] = {pack_bf16(da[hh][0], da[hh][1]), 0u, 0u, 0u};
                        const uint32_t av4[4] = {pack_bf16(av[hh][0], av[hh][1]), 0u, 0u, 0u};
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                float ck[4] = {0.f, 0.f, 0.f, 0.f}, cv[4] = {0.f, 0.f, 0.f, 0.f};
                                mma16816(ck, ak, movmatrix_t(qf[hh][kk][half]), 0u);
                                mma16816(cv, av4, movmatrix_t(of[hh][kk][half]), 0u);
                                // lane holds features d0 + 2c4, +1 (d0 = the tile's first feature)
                                const float s0 = even ? cv[0] : ck[0], s1 = even ? cv[1] : ck[1];
                                const float r0 = __shfl_xor_sync(0xffffffffu, s0, 1);
                                const float r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
                                const int d0 = (2 * hq + hh) * DH + 16 * kk + 8 * half;
                                if (live) {
                                    if (even)
                                        atomicAdd(reinterpret_cast<float4 *>(rowk + d0 + 2 * c4),
                                                  make_float4(ck[0], ck[1], r0, r1));
                                    else
                                        atomicAdd(reinterpret_cast<float4 *>(rowv + d0 + 2 * c4 - 2),
                                                  make_float4(r0, r1, cv[0], cv[1]));
                                }
                            }
                    }
                }

                // ---------------- dE = dE' + df Wfe^T (Light Edge: dE = dE'), in place in the
                // dE' tile once this chunk's weight-gradient products (which read the tile)
                // have completed; the TMA warp stores it
                if (!light) {
                    cta_wait(bar(BB_DE_FULL), (li - nl) & 1, fail, p.status);
                    cta_wait(bar(BB_WG_DONE + ((li - nl) & 1)), ((li - nl) >> 1) & 1, fail, p.status);
                    tc_fence_after();
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float dv[16];
                        tmem_ld16(tl + BS_TM_DE + 64 * e + 16 * hq, dv);
                        tmem_ld_wait();
                        add_residual16(sp + (slot_addr(li, 2 + e) - sbase) + L * 128, L, hq, dv);
                    }
                    fence_proxy_async_smem();
                }
                tc_fence_before();
                __syncwarp();
                if (t == 0) mbar_arrive(bar(BB_STAGE_DONE + (li & 3)));
            }

            // the last chunk's weight-gradient products complete before the tile and the
            // accumulator are read
            if (nl > 0) cta_wait(bar(BB_WG_DONE + ((nl - 1) & 1)), ((nl - 1) >> 1) & 1, fail, p.status);
            // ---------------- row-block results: dq through the (now idle) DA tiles,
            // four heads at a time; dg and the weight-gradient partials
            float *part = reinterpret_cast<float *>(sp + S::DA);
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                if ((hq >> 1) == half) {
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int d = (2 * (hq & 1) + hh) * DH + mt * 16 + g8 + 8 * (e >> 1), il = 2 * c4 + (e & 1);
                                part[(q * TB + il) * 128 + d] = qacc[hh][mt][e];
                            }
                }
                named_bar_sync(1, NTHR);
                {
                    const int x = tid, il = (2 * x) / 128, d = (2 * x) % 128;   // 512 threads: 8 rows x 64 pairs
                    if (i0 + il < n) {
                        float o0 = 0.f, o1 = 0.f;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            o0 += part[(k * TB + il) * 128 + d];
                            o1 += part[(k * TB + il) * 128 + d + 1];
                        }
                        *reinterpret_cast<uint32_t *>(p.dQ + ((size_t)b * n + i0 + il) * HD + 128 * half + d) =
                            pack_bf16(o0 * rs, o1 * rs);
                    }
                }
                named_bar_sync(1, NTHR);
            }
            float *wdg = reinterpret_cast<float *>(sp + S::WDG);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float x = dgp[k];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (t == 0) wdg[W * 4 + k] = x;
            }
            named_bar_sync(1, NTHR);
            // weight-gradient partials of the row block: dWfe [c][k] from lanes 0..63,
            // columns 0..15 of the accumulator, dWe^T [c][h] from lanes 64..127,
            // columns 16..23; dg from the per-warp sums
            float *rp = p.rparts + (size_t)item * RPART;
            tc_fence_after();
            if (hq == 0) {
                float v[16];
                if (nl > 0) {
                    tmem_ld16(tl + BS_TM_W + (q < 2 ? 0 : NF), v);
                    tmem_ld_wait();
                } else {   // no live chunk: no product was accumulated
#pragma unroll
                    for (int k = 0; k < 16; ++k) v[k] = 0.f;
                }
                if (q < 2) {
                    const int c = 32 * q + t;
#pragma unroll
                    for (int k = 0; k < NF; ++k) rp[c * NF + k] = v[k];
                } else {
                    const int c = 32 * (q - 2) + t;
#pragma unroll
                    for (int h = 0; h < NH; ++h) rp[DE * NF + h * DE + c] = v[h];
                }
            }
            if (tid < NF) {
                const int which = tid >> 3, h = tid & 7, hq2 = h >> 1, hh = h & 1;
                float v = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) v += wdg[(4 * hq2 + k) * 4 + which * 2 + hh];
                rp[DE * NF + NH * DE + tid] = v;
            }
        }

        named_bar_sync(2, BS_THR);   // meets the MMA and TMA warps at their end
    }
    tc_fence_before();
    __syncthreads();
    if (W == 0) tmem_dealloc(tmem, BS_TM_COLS);
}

// ------------------------------------------------------------------ host side

cudaError_t launch_bwd_stream(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                              cudaStream_t st) {
    static std::atomic<uint32_t> attr_set{0};
    if (cudaError_t e = ensure_smem_attr(k_bwd_stream, BsSmem::BYTES, attr_set); e != cudaSuccess) return e;
    CUtensorMap mE, mDEp, mDE, mK, mV;
    const int rows = a.rows < 0 ? d.n : a.rows;
    if (!encode_pair_map(&mE, a.E, d.B, rows, d.n, 32, 1) || !encode_pair_map(&mDEp, a.dEout, d.B, rows, d.n, 32, 1) ||
        !encode_pair_map(&mDE, a.dE, d.B, rows, d.n, 32, 1) || !encode_node_map(&mK, a.K, d.B, d.n, 32) ||
        !encode_node_map(&mV, a.V, d.B, d.n, 32))
        return cudaErrorInvalidValue;
    BwdStreamParams p;
    p.order = reinterpret_cast<const int *>(ws + W.order);
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.dO = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dO);
    p.LSE = a.LSE;
    p.g = g;
    p.img = reinterpret_cast<const uint8_t *>(ws + W.img);
    p.M = a.M;
    p.dQ = reinterpret_cast<__nv_bfloat16 *>(ws + W.dQ);
    p.dE = static_cast<__nv_bfloat16 *>(a.dE);
    p.rparts = reinterpret_cast<float *>(ws + W.rparts);
    p.dK32 = reinterpret_cast<float *>(ws + W.dK32);
    p.dV32 = reinterpret_cast<float *>(ws + W.dV32);
    p.status = a.status;
    p.n = d.n;
    p.row0 = a.row0;
    p.rows = rows;
    p.light = a.variant == EAGA_VARIANT_LIGHT_EDGE;
    p.unnorm = a.variant == EAGA_VARIANT_UNNORMALISED;
    p.prefetch_ahead = (uint32_t)sm_count();
    return launch_pdl(k_bwd_stream, dim3((rows + TB - 1) / TB, d.B), dim3(BS_THR), BsSmem::BYTES, st, 1, mE, mDEp, mDE,
                      mK, mV, p);
}

}  // namespace fast
}  // namespace eaga
