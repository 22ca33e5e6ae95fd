// Forward pair kernel for de = 64, H = 8, dh = 32, bf16 storage (sm_100a).
//
// One CTA owns 8 query rows i of one graph and a range of at most 8 column
// chunks of 32 (256 pairs each: two 16 KB E tiles, the 16 KB K and V
// chunks), which it streams through shared memory twice, as the layer's two
// passes ("large graphs need two passes", AI-summary page, method paragraph):
//   pass 1: FiLM coefficients f = E Wfe on the tensor cores (tcgen05, fp32 in
//           TMEM), scores S = Q K^T with warp MMAs, s' = S(1+gamma)+beta,
//           running masked row max / sum per thread (online softmax); s' is
//           kept in TMEM (16 columns per chunk);
//   pass 2: s' from TMEM, normalised a, O += a V (warp MMAs), edge update
//           dE = a We on the tensor cores, E' = E + dE written in place and
//           stored with TMA.
// Pass 2 walks the chunks in reverse, so the E tiles it reads again are the
// ones pass 1 brought into L2 last: E leaves HBM once, E' is written once and
// the [B,H,n,n] map never leaves the chip.
//
// Two CTAs share an SM (320 threads, 112 KB of shared memory and 256 TMEM
// columns each), so that one CTA's setup, row-statistics merge and O
// reduction overlap the other's streaming.  A graph with more than 8 chunks
// (n > 256) splits each row block's columns over a cluster of CS = 2 or 4
// CTAs; they combine their partial row statistics (max, sum) and their
// partial O through distributed shared memory, and each CTA's slice (at most
// 8 x 256 pairs, 256 KB of E) stays small enough for pass 2 to find it in L2.
//
// Block sparsity (as a block mask lets FlexAttention skip whole blocks): a
// chunk with no valid pair (no node among the CTA's rows, or none among the
// chunk's columns: padding of a smaller graph) has a = 0 everywhere, so E' = E
// there.  Such a chunk is only copied by the TMA warp (loaded and stored back,
// bit for bit); the compute and MMA warps never see it.  The clusters take
// the row blocks longest first (most live chunks; k_row_block_order), so
// that short and copy-only row blocks fill the last wave.
//
// Warp roles.  Warps 0..7 compute (warp W reads TMEM quadrant q = W%4 and
// handles the four heads 4hp..4hp+3, hp = W/4).  Warp 8 (one thread) issues
// the FiLM MMAs as tiles land and the edge-update MMAs once the compute warps
// have written a.  Warp 9 (one thread) keeps a ring of six 16 KB slots
// filled with TMA loads and stores E'.  They meet only on mbarriers.
//
// Pair <-> lane mapping.  E tile s (i = 2ic + s) is loaded as [j][ic][c] so
// that its 128 rows, the M rows of FiLM MMA s, are the pairs (j = 8q + t/4,
// i = 2(t%4) + s) of lane t in the warps of quadrant q: the same pair those
// lanes hold in accumulator register s of their m16n8 score tile S^T[j,i].
// TMEM lane 32q+t therefore feeds lane t directly.
#include <math.h>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using namespace dev;

constexpr int FS_CW = 8;                  // compute warps
constexpr int FS_CTHR = 32 * FS_CW;       // compute threads
constexpr int FS_THR = FS_CTHR + 64;      // + the MMA warp and the TMA warp
constexpr int FS_SLOTS = 6;               // 16 KB slots of the load ring
constexpr uint32_t FS_SLOT = 16384;
constexpr int FS_NFULL = 4;               // load barriers of live iterations
constexpr int FS_NCOPY = 3;               // dead-chunk copies in flight
constexpr int FS_PF = 4;                  // pass-1 chunks prefetched into L2 beyond the loads
constexpr int FS_MAX_CPC = 8;             // chunks per CTA (their s' fills the upper half of TMEM)
constexpr int FS_MAX_CS = 4;              // CTAs per row block

// shared memory map (bytes from a 1024-aligned base)
struct FsSmem {
    static constexpr uint32_t WFE = FS_SLOTS * FS_SLOT;       // Wfe^T [16][64] swizzled (FiLM B)
    static constexpr uint32_t WE = WFE + 2048;                // We^T [64][16] no swizzle (edge-update B)
    static constexpr uint32_t A = WE + 2048;                  // 2 tiles [128][16] no swizzle (edge-update A);
                                                              // the per-quadrant statistics at the end of pass 1
    static constexpr uint32_t FIN = A + 8192;                 // row statistics [64 (i, h)][2]: (max, sum), then LSE
    static constexpr uint32_t XST = FIN + 512;                // the cluster's partial statistics [4 ranks][64][2]
    static constexpr uint32_t G = XST + 2048;                 // g_b [16]
    static constexpr uint32_t BAR = G + 64;                   // mbarriers, see below
    static constexpr uint32_t TM = BAR + 8 * 19;              // TMEM base address
    static constexpr uint32_t FAIL = TM + 8;                  // CTA failure flag (a wait ran out)
    static constexpr uint32_t STAB = TM + 16;                 // slot table [4 live iterations] u32
    static constexpr uint32_t CTAB = STAB + 16;               // slots of the copies [3][2] u8
    static constexpr uint32_t LIVE = CTAB + 8;                // live-chunk mask of the CTA's chunks
    static constexpr uint32_t LC = LIVE + 8;                  // the live chunks, ascending [8] u8 (+ slack)
    static constexpr uint32_t DC = LC + 32;                   // the dead chunks, ascending [8] u8 (+ slack)
    static constexpr uint32_t BYTES = DC + 32 + 1024;         // + alignment slack
    static constexpr uint32_t OPART = 0;                      // [4][8][256] f32 O partials (ring drained)
    static constexpr uint32_t OFIN = 32768;                   // [8][256] f32 the CTA's O (ring drained)
};
static_assert(FsSmem::BYTES <= 115712, "two CTAs per SM");
// mbarriers: full[4] (loads of live iterations), film_full[2], film_empty[2], a_full,
// edge_full, stage_done[4], mma_final, copy[3] (loads of dead chunks), stats (the
// cluster's partial row statistics have arrived)
constexpr int FB_FULL = 0, FB_FILM_FULL = 4, FB_FILM_EMPTY = 6, FB_A_FULL = 8, FB_EDGE_FULL = 9,
              FB_STAGE_DONE = 10, FB_MMA_FINAL = 14, FB_COPY = 15, FB_STATS = 18;

// TMEM columns: FiLM 0..63 (two buffers, pass 1), edge update 0..127 (pass 2),
// s' of the CTA's chunks 128..255 (16 per chunk)
constexpr uint32_t FS_TM_COLS = 256;
constexpr uint32_t FS_TM_FILM = 0, FS_TM_EDGE = 0, FS_TM_S = 128;

struct FwdParams {
    const int *order;        // [B * row blocks]: the row block each cluster takes, longest first (null: index order)
    const __nv_bfloat16 *Q;
    const uint8_t *img;      // operand images (IMG_*)
    const float *g;          // [B, 16] global FiLM term
    const uint8_t *M;
    __nv_bfloat16 *O;
    float *LSE;
    int *status;
    int n;
    int row0, rows;          // the slab of rows this call owns (E, E' hold rows row0 .. row0+rows-1)
    int cs;                  // CTAs per row block (a cluster when > 1)
    int light;               // Light Edge variant: no per-edge FiLM map, no E in pass 1, no FiLM products
    int unnorm;              // unnormalised variant: the edge update takes s' instead of a
    uint32_t prefetch_ahead; // CTAs between this one and the one whose first tiles it prefetches
};

// 320 threads, two CTAs per SM (20 warps: five share one of the four
// 16K-register sub-partitions, so at most 96 registers a thread)
__global__ void __launch_bounds__(FS_THR, 2)
k_fwd_stream(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmEo,
             const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, FwdParams p) {
    using S = FsSmem;
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, W = tid >> 5, t = tid & 31, c4 = t & 3, g8 = t >> 2;
    const int q = W & 3, hp = (W >> 2) & 1;   // TMEM quadrant, head quad (compute warps)
    const int n = p.n, nch = (n + 31) / 32, cs = p.cs;
    const int cpc = (nch + cs - 1) / cs;                        // chunks per CTA of the row block
    // i0: the row block's first row in the graph; i0l: in the slab (E, E' rows)
    // the row block of this CTA's cluster: longest first (k_row_block_order), so
    // that the short ones fill the last wave
    const int nrb = gridDim.x / cs, cl = blockIdx.y * nrb + blockIdx.x / cs, ord = p.order ? p.order[cl] : cl;
    const int rank = blockIdx.x % cs, b = ord / nrb, i0l = (ord % nrb) * TB, i0 = p.row0 + i0l;
    const int c_begin = rank * cpc, nchl = max(0, min(nch, c_begin + cpc) - c_begin);
    const uint32_t bars = sbase + S::BAR;
    auto bar = [&](int k) { return bars + 8 * k; };
    float *g = reinterpret_cast<float *>(sp + S::G);
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);

    // Block sparsity: a chunk holding no valid pair (live_chunk_mask) needs no
    // arithmetic, its E' is its E.  The TMA warp loads iterations it in order:
    // pass 1 the nl live chunks of the CTA, ascending; pass 2 the live chunks,
    // descending; then the copies of the dead ones (two E tiles loaded and
    // stored back).  The live iterations li = 0 .. 2 nl - 1 (pass 1, then pass
    // 2) are the ones the MMA and compute warps see.  Slots: pass 1 E(s=0),
    // E(s=1), K (Light Edge: K alone); pass 2 E(s=0), E(s=1), V; a copy E, E.
    // The TMA warp takes any free slots and records them in table entry li % 4
    // (load barrier li % 4), which the other warps read after that barrier.
    const bool light = p.light != 0;
    const int ns1 = light ? 1 : 3, ks1 = light ? 0 : 2;
    constexpr int ns2 = 3, vslot = 2;
    // the slots of live iteration li: one word of the table (slot k in byte k)
    volatile uint32_t *stab = reinterpret_cast<volatile uint32_t *>(sp + S::STAB);
    auto slot_word = [&](int li) { return stab[li % FS_NFULL]; };
    auto slot_at = [&](uint32_t sw, int k) { return sbase + ((sw >> (8 * k)) & 0xffu) * FS_SLOT; };

    // ---------------- setup: barriers, TMEM, operands
    if (tid == 0) {
        for (int k = 0; k < 4; ++k) mbar_init(bar(FB_FULL + k), 1);
        mbar_init(bar(FB_FILM_FULL), 1);
        mbar_init(bar(FB_FILM_FULL + 1), 1);
        mbar_init(bar(FB_FILM_EMPTY), FS_CW);
        mbar_init(bar(FB_FILM_EMPTY + 1), FS_CW);
        mbar_init(bar(FB_A_FULL), FS_CW);
        mbar_init(bar(FB_EDGE_FULL), 1);
        for (int k = 0; k < 4; ++k) mbar_init(bar(FB_STAGE_DONE + k), FS_CW);
        mbar_init(bar(FB_MMA_FINAL), 1);
        for (int k = 0; k < FS_NCOPY; ++k) mbar_init(bar(FB_COPY + k), 1);
        mbar_init(bar(FB_STATS), 64 * cs);
        fence_mbar_init();
        *fail = 0;
    }
    if (W == 0) {
        tmem_alloc(sbase + S::TM, FS_TM_COLS);
        tmem_relinquish();
    }
    if (W == 1) {
        // the CTA's chunks c_begin .. c_begin + nchl - 1, numbered from 0
        const uint32_t lm_all = live_chunk_mask(p.M, b, n, i0, t);
        const uint32_t lm = nchl > 0 ? (lm_all >> c_begin) & ((1u << nchl) - 1u) : 0u;
        if (t == 0) *reinterpret_cast<volatile uint32_t *>(sp + S::LIVE) = lm;
        const int below = __popc(lm & ((1u << t) - 1u));   // live chunks below chunk t
        if ((lm >> t) & 1u) sp[S::LC + below] = (uint8_t)t;
        else if (t < nchl) sp[S::DC + t - below] = (uint8_t)t;
    }
    // operand images: Wfe^T (FiLM B, swizzled) and We^T (edge-update B, no swizzle), 2 KB each
    if (tid < 256) reinterpret_cast<uint4 *>(sp + S::WFE)[tid] = reinterpret_cast<const uint4 *>(p.img)[tid];
    // edge-update A tiles: zero (the K half h >= 8 stays zero)
    for (int e = tid; e < 8192 / 16; e += FS_THR) reinterpret_cast<uint4 *>(sp + S::A)[e] = make_uint4(0, 0, 0, 0);
    if (tid < NF) g[tid] = p.g[(size_t)b * NF + tid];
    fence_proxy_async_smem();
    tc_fence_before();
    if (cs > 1)
        cluster_sync_all();   // every CTA of the cluster has its barriers before any remote arrival
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const uint32_t live = *reinterpret_cast<volatile uint32_t *>(sp + S::LIVE);
    const int nl = __popc(live), nit = 2 * nl, nload = nl + nchl;
    const volatile uint8_t *lc = sp + S::LC;
    const volatile uint8_t *dc = sp + S::DC;
    // chunk (of the CTA's) of live iteration li; of load iteration it
    auto chunk_of_li = [&](int li) { return (int)lc[li < nl ? li : nit - 1 - li]; };
    auto is_live = [&](int it) { return it < nit; };
    auto chunk_of_it = [&](int it) { return it < nl ? (int)lc[it] : it < nit ? (int)lc[nit - 1 - it] : (int)dc[it - nit]; };

    if (W == FS_CW) {
        // ================= MMA issuer: FiLM (pass 1) as tiles land, edge updates (pass 2) on demand
        if (t == 0) {
            const uint32_t idesc_f = idesc_bf16_f32(128, NF), idesc_e = idesc_bf16_f32(128, DE);
            auto issue_film = [&](int li) {   // into TMEM buffer li & 1
                tc_fence_after();
                const uint32_t sw = slot_word(li);
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const uint32_t a0 = slot_at(sw, s);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ss(tmem + FS_TM_FILM + 32 * (li & 1) + 16 * s,
                                    smem_desc(a0 + kk * 32, 16, 1024, LAYOUT_SW128),
                                    smem_desc(sbase + S::WFE + kk * 32, 16, 1024, LAYOUT_SW128), idesc_f, kk > 0);
                }
                mma_commit(bar(FB_FILM_FULL + (li & 1)));
            };
            auto issue_edge = [&]() {   // the a tiles -> the edge accumulator
                tc_fence_after();
#pragma unroll
                for (int e = 0; e < 2; ++e)
                    mma_bf16_ss(tmem + FS_TM_EDGE + 64 * e, smem_desc(sbase + S::A + e * 4096, 128, 256, LAYOUT_NONE),
                                smem_desc(sbase + S::WE, 128, 256, LAYOUT_NONE), idesc_e, 0);
                mma_commit(bar(FB_EDGE_FULL));
            };
            const int nfilm = light ? 0 : nl;   // Light Edge: no FiLM products
            int next_film = 0, next_edge = nl;
            uint32_t polls = 0;
            while ((next_film < nfilm || next_edge < nit) && !*fail) {
                bool progressed = false;
                if (next_film < nfilm &&
                    mbar_test_wait(bar(FB_FULL + next_film % FS_NFULL), (next_film / FS_NFULL) & 1) &&
                    (next_film < 2 ||
                     mbar_test_wait(bar(FB_FILM_EMPTY + (next_film & 1)), ((next_film - 2) >> 1) & 1))) {
                    issue_film(next_film++);
                    progressed = true;
                }
                if (next_edge < nit && mbar_test_wait(bar(FB_A_FULL), (next_edge - nl) & 1)) {
                    issue_edge();
                    ++next_edge;
                    progressed = true;
                }
                // idle: back off after a few polls; a wait that makes no progress
                // for 2^24 polls gives up
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
            mma_commit(bar(FB_MMA_FINAL));
            if (!mbar_wait(bar(FB_MMA_FINAL), 0)) flag_timeout(p.status);
        }
        __syncwarp();
        named_bar_sync(2, FS_THR);
    } else if (W == FS_CW + 1) {
        // ================= TMA: loads into the slot ring, E' stores, copies of dead chunks
        if (t == 0) {
            // E tiles loaded in pass 1 are read again in pass 2: keep them in L2;
            // pass-2 reads and the E' stores are not read again
            const uint64_t keep_l2 = l2_evict_last(), drop_l2 = l2_evict_first();
            volatile uint8_t *ctab = sp + S::CTAB;
            uint32_t free_mask = (1u << FS_SLOTS) - 1u;
            auto take_slot = [&]() {
                const int sidx = __ffs(free_mask) - 1;
                free_mask &= free_mask - 1u;
                return (uint8_t)sidx;
            };
            // loads go out in iteration order; a live iteration waits for its
            // load barrier to be free (at most FS_NFULL live iterations in
            // flight: a barrier is re-armed only after its previous iteration
            // was taken off the ring), a copy likewise for its copy barrier
            int next_load = 0, load_li = 0, load_dk = 0, done_li = 0, done_dk = 0;
            auto issue_loads = [&]() {
                while (next_load < nload && !*fail) {
                    const int it = next_load, j0 = 32 * (c_begin + chunk_of_it(it));
                    const bool pass2 = it >= nl && it < nit;
                    if (is_live(it)) {
                        const int li = load_li, ns = pass2 ? ns2 : ns1;
                        if (li >= done_li + FS_NFULL || __popc(free_mask) < ns) break;
                        uint32_t sw = 0;
                        for (int k = 0; k < ns; ++k) sw |= (uint32_t)take_slot() << (8 * k);
                        stab[li % FS_NFULL] = sw;
                        const uint32_t fb = bar(FB_FULL + li % FS_NFULL);
                        mbar_expect_tx(fb, ns * FS_SLOT);   // releases the table entry too
                        const uint64_t pol = pass2 ? drop_l2 : keep_l2;
                        if (pass2 || !light) {
                            tma_load_5d_hint(slot_at(sw, 0), &tmE, fb, 0, i0l / 2, j0, 0, b, pol);
                            tma_load_5d_hint(slot_at(sw, 1), &tmE, fb, 0, i0l / 2, j0, 1, b, pol);
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (!pass2) tma_load_3d(slot_at(sw, ks1) + k * 4096, &tmK, fb, 64 * k, j0, b);
                            else tma_load_3d(slot_at(sw, vslot) + k * 4096, &tmV, fb, 64 * k, j0, b);
                        }
                        if (!pass2 && !light && li + FS_PF < nl)
                            for (int s = 0; s < 2; ++s)
                                tma_prefetch_5d(&tmE, 0, i0l / 2, 32 * (c_begin + lc[li + FS_PF]), s, b);
                        ++load_li;
                    } else {
                        const int dk = load_dk;
                        if (dk >= done_dk + FS_NCOPY || __popc(free_mask) < 2) break;
                        const uint32_t cb = bar(FB_COPY + dk % FS_NCOPY);
                        mbar_expect_tx(cb, 2 * FS_SLOT);
#pragma unroll
                        for (int s = 0; s < 2; ++s) {
                            const uint8_t sl = take_slot();
                            ctab[(dk % FS_NCOPY) * 2 + s] = sl;
                            tma_load_5d_hint(sbase + sl * FS_SLOT, &tmE, cb, 0, i0l / 2, j0, s, b, drop_l2);
                        }
                        ++load_dk;
                    }
                    ++next_load;
                }
            };
            for (int c = 0; c < nl && c < FS_PF && !light; ++c)
                for (int s = 0; s < 2; ++s) tma_prefetch_5d(&tmE, 0, i0l / 2, 32 * (c_begin + lc[c]), s, b);
            issue_loads();
            // iterations are taken off the ring in order: a live one once the
            // compute warps are done with it (stage_done), a copy once its
            // tiles landed; the E tiles of a pass-2 chunk (E' in place) or of a
            // copy are stored, and their slots are free once the store has read them
            uint32_t pend_mask = 0u;   // slots of the last store, not yet known to have read them
            for (int it = 0; it < nload; ++it) {
                const bool pass2 = it >= nl && it < nit;
                if (it == nl && p.prefetch_ahead && !light) {
                    // L2 prefetch of the first tiles of the CTA that runs about one wave later
                    const uint32_t cid = blockIdx.y * gridDim.x + blockIdx.x + p.prefetch_ahead;
                    if (cid < gridDim.x * gridDim.y) {
                        const int pord = p.order ? p.order[cid / cs] : int(cid / cs), pb = pord / nrb,
                                  prb = pord % nrb;
                        const int pc0 = (cid % cs) * cpc;
                        for (int cc = pc0; cc < nch && cc < pc0 + 2; ++cc)
                            for (int s = 0; s < 2; ++s) tma_prefetch_5d(&tmE, 0, prb * TB / 2, 32 * cc, s, pb);
                    }
                }
                const int j0 = 32 * (c_begin + chunk_of_it(it));
                const bool lv = is_live(it);
                uint32_t s0, s1;        // the slots of the E tiles a store reads
                if (lv) {
                    const int li = done_li++;
                    if (!cta_wait(bar(FB_STAGE_DONE + (li & 3)), (li >> 2) & 1, fail, p.status)) continue;
                    const int ns = pass2 ? ns2 : ns1;
                    const uint32_t sw = slot_word(li);
                    for (int k = pass2 ? 2 : 0; k < ns; ++k) free_mask |= 1u << ((sw >> (8 * k)) & 0xffu);
                    s0 = sw & 0xffu;
                    s1 = (sw >> 8) & 0xffu;
                } else {
                    const int dk = done_dk++;
                    if (!cta_wait(bar(FB_COPY + dk % FS_NCOPY), (dk / FS_NCOPY) & 1, fail, p.status)) continue;
                    s0 = ctab[(dk % FS_NCOPY) * 2];
                    s1 = ctab[(dk % FS_NCOPY) * 2 + 1];
                }
                if (pass2 || !lv) {
                    tma_store_5d_hint(&tmEo, sbase + s0 * FS_SLOT, 0, i0l / 2, j0, 0, b, drop_l2);
                    tma_store_5d_hint(&tmEo, sbase + s1 * FS_SLOT, 0, i0l / 2, j0, 1, b, drop_l2);
                    tma_store_commit();
                    // the previous store's slots are free once it has read them
                    if (pend_mask) {
                        tma_store_wait_read1();
                        free_mask |= pend_mask;
                    }
                    pend_mask = (1u << s0) | (1u << s1);
                }
                issue_loads();
            }
            tma_store_wait_read0();
            if (*fail) {   // loads already issued land before the CTA's shared memory is released
                for (int li = max(load_li - FS_NFULL, 0); li < load_li; ++li)
                    mbar_wait(bar(FB_FULL + li % FS_NFULL), (li / FS_NFULL) & 1);
                for (int dk = max(load_dk - FS_NCOPY, 0); dk < load_dk; ++dk)
                    mbar_wait(bar(FB_COPY + dk % FS_NCOPY), (dk / FS_NCOPY) & 1);
            }
        }
        __syncwarp();
        named_bar_sync(2, FS_THR);   // the ring is drained
    } else if (nl == 0 && cs == 1) {
        // ================= compute warps of a row block without a valid pair: its
        // rows get LSE = -inf and O = 0 (what the passes would give), no passes
        for (int x = tid; x < TB * NH; x += FS_CTHR) {
            const int il = x >> 3, h = x & 7;
            if (i0 + il < n) p.LSE[((size_t)b * NH + h) * n + i0 + il] = -INFINITY;
        }
        for (int x = tid; x < TB * HD / 8; x += FS_CTHR) {
            const int il = x / (HD / 8), d = (x % (HD / 8)) * 8;
            if (i0 + il < n)
                *reinterpret_cast<uint4 *>(p.O + ((size_t)b * n + i0 + il) * HD + d) = make_uint4(0u, 0u, 0u, 0u);
        }
        named_bar_sync(2, FS_THR);   // the TMA warp has stored the copies
    } else {
        // ================= compute warps: quadrant q, heads 4hp..4hp+3
        const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
        const float rs = rsqrtf((float)DH);
        const uint32_t L = 32 * q + t;
        const int hqa = 2 * hp, hqb = 2 * hp + 1;     // the two head pairs (helpers take pairs)
        uint32_t qfa[2][2][2], qfb[2][2][2];
        load_frags2(p.Q, b, n, i0, hqa, g8, c4, qfa);
        load_frags2(p.Q, b, n, i0, hqb, g8, c4, qfb);
        // the thread's two rows i = i0 + 2c4 + e (e = 0, 1)
        const bool mrow[2] = {i0 + 2 * c4 < n && p.M[(size_t)b * n + i0 + 2 * c4] != 0,
                              i0 + 2 * c4 + 1 < n && p.M[(size_t)b * n + i0 + 2 * c4 + 1] != 0};

        // ======== pass 1: running (max, sum) per (row, head) over the CTA's live chunks
        float lse[2][4];        // after pass 1: the row statistics LSE = m + log l, per [e][k]
        {
            float rm[2][4], rl[2][4];
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    rm[e][k] = -INFINITY;
                    rl[e][k] = 0.f;
                }
            for (int li = 0; li < nl; ++li) {
                const int c = chunk_of_li(li), j = 32 * (c_begin + c) + 8 * q + g8;
                const bool mcol = j < n && p.M[(size_t)b * n + j] != 0;
                cta_wait(bar(FB_FULL + li % FS_NFULL), (li / FS_NFULL) & 1, fail, p.status);
                const uint32_t sw = slot_word(li);
                float sa[2][4], sb[2][4];
                const uint32_t ks = slot_at(sw, ks1);
                warp_scores2<1>(ks, q, t, hqa, qfa, sa);
                warp_scores2<1>(ks, q, t, hqb, qfb, sb);
                // FiLM of the pair: gamma, beta of the four heads
                float gm[2][4] = {}, bt[2][4] = {};
                if (!light) {
                    cta_wait(bar(FB_FILM_FULL + (li & 1)), (li >> 1) & 1, fail, p.status);
                    tc_fence_after();
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const uint32_t fcol = FS_TM_FILM + 32 * (li & 1) + 16 * e + 4 * hp;
                        tmem_ld2(tl + fcol, gm[e][0], gm[e][1]);
                        tmem_ld2(tl + fcol + 2, gm[e][2], gm[e][3]);
                        tmem_ld2(tl + fcol + NH, bt[e][0], bt[e][1]);
                        tmem_ld2(tl + fcol + NH + 2, bt[e][2], bt[e][3]);
                    }
                    tmem_ld_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (t == 0) mbar_arrive(bar(FB_FILM_EMPTY + (li & 1)));
                }
                float sx[4][2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool valid = mcol && mrow[e];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int h = 4 * hp + k;
                        const float raw = k < 2 ? sa[k][e] : sb[k - 2][e];
                        const float sv = raw * rs * (1.f + gm[e][k] + g[h]) + bt[e][k] + g[NH + h];
                        sx[k][e] = valid ? sv : -INFINITY;
                        const float x = sx[k][e];
                        const float mn = fmaxf(rm[e][k], x);
                        if (mn != -INFINITY) {
                            rl[e][k] = rl[e][k] * exp2f((rm[e][k] - mn) * LOG2E) + exp2f((x - mn) * LOG2E);
                            rm[e][k] = mn;
                        }
                    }
                }
                // s' for pass 2 (-inf where invalid)
                const uint32_t scol = tl + FS_TM_S + 16 * c;
                tmem_st2(scol + 2 * hqa, sx[0][0], sx[1][0]);
                tmem_st2(scol + 2 * hqa + 8, sx[0][1], sx[1][1]);
                tmem_st2(scol + 2 * hqb, sx[2][0], sx[3][0]);
                tmem_st2(scol + 2 * hqb + 8, sx[2][1], sx[3][1]);
                __syncwarp();
                if (t == 0) mbar_arrive(bar(FB_STAGE_DONE + (li & 3)));
            }
            tmem_st_wait();
            // ---------------- end of pass 1: statistics over lanes, then quadrants
            // (in the idle a tiles), then over the cluster's CTAs
            float *wst = reinterpret_cast<float *>(sp + S::A);
            float *fin = reinterpret_cast<float *>(sp + S::FIN);
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    float m = rm[e][k], l = rl[e][k];
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) {
                        const float mo = __shfl_xor_sync(0xffffffffu, m, o);
                        const float lo = __shfl_xor_sync(0xffffffffu, l, o);
                        const float mn = fmaxf(m, mo);
                        l = (mn == -INFINITY) ? 0.f : l * exp2f((m - mn) * LOG2E) + lo * exp2f((mo - mn) * LOG2E);
                        m = mn;
                    }
                    if (g8 == 0) {
                        const int il = 2 * c4 + e, h = 4 * hp + k;
                        wst[((q * 8 + il) * 8 + h) * 2 + 0] = m;
                        wst[((q * 8 + il) * 8 + h) * 2 + 1] = l;
                    }
                }
            named_bar_sync(1, FS_CTHR);
            // (max, sum) of (row, head) tid over the quadrants, in a fixed order
            auto combine = [](float &m, float &l, float mk, float lk) {
                const float mn = fmaxf(m, mk);
                if (mn != -INFINITY) {
                    l = (m == -INFINITY ? 0.f : l * exp2f((m - mn) * LOG2E)) +
                        (mk == -INFINITY ? 0.f : lk * exp2f((mk - mn) * LOG2E));
                    m = mn;
                }
            };
            if (tid < 64) {
                float m = -INFINITY, l = 0.f;
#pragma unroll
                for (int k = 0; k < 4; ++k) combine(m, l, wst[(k * 64 + tid) * 2], wst[(k * 64 + tid) * 2 + 1]);
                if (cs > 1) {
                    // to every CTA of the cluster (itself included): slot `rank` of its table
                    const uint32_t src = sbase + S::XST + (uint32_t)(rank * 64 + tid) * 8;
                    for (int r = 0; r < cs; ++r) {
                        st_cluster_f32x2(cluster_map(src, r), m, l);
                        mbar_arrive_cluster(cluster_map(bar(FB_STATS), r));
                    }
                } else {
                    fin[2 * tid] = m;
                    fin[2 * tid + 1] = l;
                }
            }
            if (cs > 1) {
                // the partial statistics of all CTAs of the row block (bounded wait)
                bool ok = !*fail;
                for (uint32_t it = 0; ok && !mbar_try_wait_cluster(bar(FB_STATS), 0); ++it)
                    if (it > (1u << 24) || ((it & 255u) == 255u && *fail)) {
                        if (!*fail) {
                            *fail = 1;
                            flag_timeout(p.status);
                        }
                        ok = false;
                    }
                if (tid < 64) {
                    const float *xst = reinterpret_cast<const float *>(sp + S::XST);
                    float m = -INFINITY, l = 0.f;
                    for (int r = 0; r < cs; ++r) combine(m, l, xst[(r * 64 + tid) * 2], xst[(r * 64 + tid) * 2 + 1]);
                    fin[2 * tid] = m;
                    fin[2 * tid + 1] = l;
                }
            }
            if (tid < 64) {
                const float m = fin[2 * tid], l = fin[2 * tid + 1];
                const float v = (m == -INFINITY) ? -INFINITY : m + logf(l);
                const int il = tid >> 3, h = tid & 7;
                if (rank == 0 && i0 + il < n) p.LSE[((size_t)b * NH + h) * n + i0 + il] = v;
                fin[2 * tid] = v;
            }
            named_bar_sync(1, FS_CTHR);
#pragma unroll
            for (int e = 0; e < 2; ++e)
#pragma unroll
                for (int k = 0; k < 4; ++k) lse[e][k] = fin[2 * ((2 * c4 + e) * 8 + 4 * hp + k)];
            // the a tiles again: the statistics overwrote their first 2 KB
            reinterpret_cast<uint2 *>(sp + S::A)[tid] = make_uint2(0u, 0u);
        }

        // ======== pass 2: normalised a, O += a V, the edge update, E' = E + a We
        float oa[2][2][4], ob[2][2][4];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int x = 0; x < 4; ++x) oa[hh][mt][x] = ob[hh][mt][x] = 0.f;
        for (int li = nl; li < nit; ++li) {
            const int c = chunk_of_li(li), j = 32 * (c_begin + c) + 8 * q + g8;
            const bool mcol = j < n && p.M[(size_t)b * n + j] != 0;
            cta_wait(bar(FB_FULL + li % FS_NFULL), (li / FS_NFULL) & 1, fail, p.status);
            const uint32_t sw = slot_word(li);
            // s' as pass 1 left it in tensor memory (-inf where invalid)
            float sx[4][2];
            const uint32_t scol = tl + FS_TM_S + 16 * c;
            tmem_ld2(scol + 2 * hqa, sx[0][0], sx[1][0]);
            tmem_ld2(scol + 2 * hqa + 8, sx[0][1], sx[1][1]);
            tmem_ld2(scol + 2 * hqb, sx[2][0], sx[3][0]);
            tmem_ld2(scol + 2 * hqb + 8, sx[2][1], sx[3][1]);
            tmem_ld_wait();
            // a (for O) and the edge update's coefficient (a, or s' when unnormalised)
            float pa[2][4], pb[2][4];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const bool valid = mcol && mrow[e];
                float ce[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float a = valid ? exp2f((sx[k][e] - lse[e][k]) * LOG2E) : 0.f;
                    ce[k] = p.unnorm ? (valid ? sx[k][e] : 0.f) : a;
                    if (k < 2) pa[k][e] = a; else pb[k - 2][e] = a;
                }
                uint8_t *arow = sp + S::A + e * 4096;
                *reinterpret_cast<uint32_t *>(arow + ns16(L, 4 * hp)) = pack_bf16(ce[0], ce[1]);
                *reinterpret_cast<uint32_t *>(arow + ns16(L, 4 * hp + 2)) = pack_bf16(ce[2], ce[3]);
            }
            pa[0][2] = pa[0][3] = pa[1][2] = pa[1][3] = 0.f;
            pb[0][2] = pb[0][3] = pb[1][2] = pb[1][3] = 0.f;
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (t == 0) mbar_arrive(bar(FB_A_FULL));

            // O += a V on warp MMAs (overlaps the edge MMA)
            const uint32_t vs = slot_at(sw, vslot);
            warp_contract2<1, true>(vs, q, t, hqa, pa, oa);
            warp_contract2<1, true>(vs, q, t, hqb, pb, ob);

            // E' = E + (a We), in place (the TMA warp stores it)
            cta_wait(bar(FB_EDGE_FULL), (li - nl) & 1, fail, p.status);
            tc_fence_after();
#pragma unroll
            for (int e = 0; e < 2; ++e) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float dv[16];
                    tmem_ld16(tl + FS_TM_EDGE + 64 * e + 32 * hp + 16 * half, dv);
                    tmem_ld_wait();
                    add_residual16(sp + (slot_at(sw, e) - sbase) + L * 128, L, 2 * hp + half, dv);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (t == 0) mbar_arrive(bar(FB_STAGE_DONE + (li & 3)));
        }

        // ---------------- O: sum over the quadrant warps (in the drained ring)
        named_bar_sync(2, FS_THR);
        store_quadrant_part(sp, S::OPART, oa, q, hqa, t);
        store_quadrant_part(sp, S::OPART, ob, q, hqb, t);
        named_bar_sync(1, FS_CTHR);
        const float *part = reinterpret_cast<const float *>(sp + S::OPART);
        float *ofin = reinterpret_cast<float *>(sp + S::OFIN);
        for (int x = tid; x < TB * HD / 2; x += FS_CTHR) {
            const int il = (2 * x) / HD, d = (2 * x) % HD;
            float o0 = 0.f, o1 = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                o0 += part[k * TB * HD + il * HD + d];
                o1 += part[k * TB * HD + il * HD + d + 1];
            }
            if (cs > 1) {
                ofin[il * HD + d] = o0;
                ofin[il * HD + d + 1] = o1;
            } else if (i0 + il < n) {
                *reinterpret_cast<uint32_t *>(p.O + ((size_t)b * n + i0 + il) * HD + d) = pack_bf16(o0, o1);
            }
        }
    }
    if (cs > 1) {
        // O = the sum of the cluster's partial O (in rank order); CTA `rank`
        // writes features [rank * 256 / cs, (rank + 1) * 256 / cs) of the 8 rows
        cluster_sync_all();
        if (W < FS_CW) {
            const int fw = HD / cs;
            for (int x = tid; x < TB * fw / 2; x += FS_CTHR) {
                const int il = (2 * x) / fw, d = rank * fw + (2 * x) % fw;
                const uint32_t src = sbase + S::OFIN + (uint32_t)(il * HD + d) * 4;
                float o0 = 0.f, o1 = 0.f;
                for (int r = 0; r < cs; ++r) {
                    const float2 v = ld_cluster_f32x2(cluster_map(src, r));
                    o0 += v.x;
                    o1 += v.y;
                }
                if (i0 + il < n)
                    *reinterpret_cast<uint32_t *>(p.O + ((size_t)b * n + i0 + il) * HD + d) = pack_bf16(o0, o1);
            }
        }
        cluster_sync_all();   // no CTA leaves while another reads its shared memory
    }
    tc_fence_before();
    __syncthreads();
    if (W == 0) tmem_dealloc(tmem, FS_TM_COLS);
}

// ------------------------------------------------------------------ host side

// CTAs per row block: enough that each takes at most FS_MAX_CPC chunks.
static int fwd_cluster_size(int n) {
    const int nch = (n + 31) / 32;
    int cs = 1;
    while ((nch + cs - 1) / cs > FS_MAX_CPC) cs *= 2;
    return cs;
}

cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, const uint8_t *img, const int *order, const float *g,
                             cudaStream_t st) {
    static std::atomic<uint32_t> attr_set{0}, carveout_set{0};
    if (cudaError_t e = ensure_smem_attr(k_fwd_stream, FsSmem::BYTES, attr_set); e != cudaSuccess) return e;
    {   // the whole shared-memory carveout, so that two CTAs fit on an SM
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && dev < 32 && !(carveout_set.load() & (1u << dev))) {
            if (cudaError_t e = cudaFuncSetAttribute(k_fwd_stream, cudaFuncAttributePreferredSharedMemoryCarveout,
                                                     (int)cudaSharedmemCarveoutMaxShared);
                e != cudaSuccess)
                return e;
            carveout_set.fetch_or(1u << dev);
        }
    }
    CUtensorMap mE, mEo, mK, mV;
    const int rows = a.rows < 0 ? d.n : a.rows;
    if (!encode_pair_map(&mE, a.E, d.B, rows, d.n, 32, 1) || !encode_pair_map(&mEo, a.Eout, d.B, rows, d.n, 32, 1) ||
        !encode_node_map(&mK, a.K, d.B, d.n, 32) || !encode_node_map(&mV, a.V, d.B, d.n, 32))
        return cudaErrorInvalidValue;
    const int cs = fwd_cluster_size(d.n);
    if (cs > FS_MAX_CS) return cudaErrorInvalidValue;
    FwdParams p;
    p.order = order;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.img = img;
    p.g = g;
    p.M = a.M;
    p.O = static_cast<__nv_bfloat16 *>(a.O);
    p.LSE = a.LSE;
    p.status = a.status;
    p.n = d.n;
    p.row0 = a.row0;
    p.rows = rows;
    p.cs = cs;
    p.light = a.variant == EAGA_VARIANT_LIGHT_EDGE;
    p.unnorm = a.variant == EAGA_VARIANT_UNNORMALISED;
    p.prefetch_ahead = (uint32_t)(2 * sm_count());   // two CTAs per SM
    const dim3 grid(((rows + TB - 1) / TB) * cs, d.B);
    return launch_pdl(k_fwd_stream, grid, dim3(FS_THR), FsSmem::BYTES, st, cs, mE, mEo, mK, mV, p);
}

}  // namespace fast
}  // namespace eaga
