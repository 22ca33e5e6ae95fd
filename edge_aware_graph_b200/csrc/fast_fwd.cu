// Forward pair kernel for de = 64, H = 8, dh = 32, bf16 storage (sm_100a).
//
// One CTA owns the tile of 8 query rows i x 32NR key columns j of one graph
// (NR = 1 for n <= 512, so two CTAs share an SM; NR = 2 above); the CTAs
// that share the 8 rows form a thread-block cluster.  Each CTA loads its E
// tile once with TMA and keeps it in shared memory for both passes of the
// layer ("large graphs need two passes", AI-summary page, method paragraph):
//   pass 1: FiLM coefficients f = E Wfe on the tensor cores (tcgen05, fp32 in
//           TMEM), scores S = Q K^T with warp MMAs, s' = S(1+gamma)+beta,
//           masked row max / sum over the CTA's columns;
//   cluster exchange of the (max, sum) pairs through distributed shared
//           memory gives every CTA the final softmax statistics;
//   pass 2: normalised a, O partial = a V (warp MMAs), edge update
//           dE = a We on the tensor cores, E' = E + dE written in place and
//           stored with TMA; O partials summed over the warps and the cluster.
// So E is read from HBM once and E' written once; the [B,H,n,n] map never
// leaves the chip.
//
// Pair <-> lane mapping.  The E tile is loaded as [s][j][ic][c] (i = 2ic+s)
// so that the 128 rows of FiLM MMA e = (r,s) are the pairs
// (j = 32r + 8q + t/4, i = 2(t%4) + s) of lane t in the warps of quadrant q:
// the same pair those lanes hold in accumulator register e of their m16n8
// score tile S^T[j,i].  TMEM lane 32q+t therefore feeds lane t directly.
// 16 warps: warp W reads quadrant q = W%4 and handles heads 2(W/4), 2(W/4)+1.
#include <math.h>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using namespace dev;

// shared memory map (bytes from a 1024-aligned base)
template <int NR>
struct FwdSmem {
    static constexpr uint32_t E = 0;                          // E tile [s 2][j 32NR][ic 4][c 64], swizzled rows
    static constexpr uint32_t K = NR * 32768;                 // K chunk: 4 boxes [j 32NR][d 64], swizzled
    static constexpr uint32_t V = K + NR * 16384;             // V chunk, same layout
    static constexpr uint32_t WFE = V + NR * 16384;           // Wfe^T [16][64] swizzled (FiLM B)
    static constexpr uint32_t WE = WFE + 2048;                // We^T [64][16] no swizzle (edge-update B)
    static constexpr uint32_t A = WE + 2048;                  // 2NR tiles [128][16] no swizzle (edge-update A)
    static constexpr uint32_t WST = A + 2 * NR * 4096;        // per-quadrant stats [4][8 i][8 h][2] f32
    static constexpr uint32_t CST = WST + 4 * 8 * 8 * 2 * 4;  // CTA stats [8][8][2] (read by peers)
    static constexpr uint32_t FIN = CST + 8 * 8 * 2 * 4;      // final m, 1/l [8][8][2] (m, l before inversion)
    static constexpr uint32_t G = FIN + 8 * 8 * 2 * 4;        // g_b [16]
    static constexpr uint32_t MI = G + 64;                    // mask of the 8 rows
    static constexpr uint32_t MJ = MI + 16;                   // mask of the 32NR columns
    static constexpr uint32_t BAR = MJ + 64;                  // 6 mbarriers
    static constexpr uint32_t TM = BAR + 48;                  // TMEM base address
    static constexpr uint32_t RST = TM + 16;                  // received softmax stats [16][64][2] f32
    static constexpr uint32_t RO = RST + RECV_ROWVALS_BYTES;  // received O partial slices
    static constexpr uint32_t BYTES = RO + recv_rows_bytes(1) + 1024;   // + alignment slack
    static constexpr uint32_t OPART = K;                      // 32 KB quadrant partials of O (K, V chunks are dead)
};

constexpr uint32_t TM_COLS = 256;            // FiLM: cols 0..32NR-1; edge update: cols 64..191
constexpr uint32_t TM_FILM = 0, TM_EDGE = 64;

struct FwdParams {
    const __nv_bfloat16 *Q;
    const uint8_t *img;      // operand images (IMG_*)
    const float *g;          // [B, 16] global FiLM term
    const uint8_t *M;
    __nv_bfloat16 *O;
    float *LSE;
    int *status;
    int n;
    uint32_t prefetch_ahead;   // CTAs between this one and the one whose tiles it prefetches (0: none)
};

template <int NR>
__global__ void __launch_bounds__(NTHR, NR == 1 ? 2 : 1)
k_fwd_pairs(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmEo,
            const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, FwdParams p) {
    using S = FwdSmem<NR>;
    constexpr int TCN = tile_cols(NR), NE = 2 * NR;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, W = tid >> 5, q = W & 3, hq = W >> 2, t = tid & 31, c4 = t & 3, g8 = t >> 2;
    const uint32_t rank = cluster_rank();
    const uint32_t nclu = gridDim.x;
    const int n = p.n;
    const int j0 = blockIdx.x * TCN, i0 = blockIdx.y * TB, b = blockIdx.z;
    const uint32_t bar_e = sbase + S::BAR, bar_kv = bar_e + 8, bar_film = bar_e + 16, bar_edge = bar_e + 24,
                   bar_st = bar_e + 32, bar_o = bar_e + 40;
    float *g = reinterpret_cast<float *>(sp + S::G);
    uint8_t *mi = sp + S::MI, *mj = sp + S::MJ;

    // ---------------- setup: barriers, TMA, TMEM, operands
    if (tid == 0) {
        mbar_init(bar_e, 1);
        mbar_init(bar_kv, 1);
        mbar_init(bar_film, 1);
        mbar_init(bar_edge, 1);
        mbar_init(bar_st, 1);
        mbar_init(bar_o, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_st, nclu * 64 * 8);
        mbar_expect_tx(bar_o, nclu * rows_slice(1, nclu, rank) * 16);
        mbar_expect_tx(bar_e, NR * 32768);
        tma_load_5d(sbase + S::E, &tmE, bar_e, 0, i0 / 2, j0, 0, b);
        mbar_expect_tx(bar_kv, NR * 32768);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            tma_load_3d(sbase + S::K + k * NR * 4096, &tmK, bar_kv, 64 * k, j0, b);
            tma_load_3d(sbase + S::V + k * NR * 4096, &tmV, bar_kv, 64 * k, j0, b);
        }        // L2 prefetch of the tiles of the CTA that runs about one wave later
        const uint32_t cid = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x + p.prefetch_ahead;
        if (p.prefetch_ahead && cid < gridDim.x * gridDim.y * gridDim.z) {
            const int px = cid % gridDim.x, py = (cid / gridDim.x) % gridDim.y, pz = cid / (gridDim.x * gridDim.y);
            tma_prefetch_5d(&tmE, 0, py * TB / 2, px * TCN, 0, pz);
            if (py == 0)
                for (int k = 0; k < 4; ++k) {
                    tma_prefetch_3d(&tmK, 64 * k, px * TCN, pz);
                    tma_prefetch_3d(&tmV, 64 * k, px * TCN, pz);
                }
        }
    }
    if (W == 0) {
        tmem_alloc(sbase + S::TM, TM_COLS);
        tmem_relinquish();
    }
    // operand images: Wfe^T (FiLM B, swizzled) and We^T (edge-update B, no swizzle), 2 KB each
    if (tid < 256) reinterpret_cast<uint4 *>(sp + S::WFE)[tid] = reinterpret_cast<const uint4 *>(p.img)[tid];
    // edge-update A tiles: zero (the K half h >= 8 stays zero)
    for (int e = tid; e < NE * 4096 / 16; e += NTHR) reinterpret_cast<uint4 *>(sp + S::A)[e] = make_uint4(0, 0, 0, 0);
    if (tid < NF) g[tid] = p.g[(size_t)b * NF + tid];
    if (tid >= 32 && tid < 32 + TB) mi[tid - 32] = (i0 + tid - 32 < n) ? p.M[(size_t)b * n + i0 + tid - 32] : 0;
    if (tid >= 64 && tid < 64 + TCN) mj[tid - 64] = (j0 + tid - 64 < n) ? p.M[(size_t)b * n + j0 + tid - 64] : 0;
    uint32_t qf[2][2][2];
    load_frags2(p.Q, b, n, i0, hq, g8, c4, qf);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
    cluster_arrive();   // receive barriers of this CTA are armed

    // ---------------- pass 1a: FiLM on the tensor cores (one thread issues)
    if (tid == 0) {
        if (!mbar_wait(bar_e, 0)) flag_timeout(p.status);
        tc_fence_after();
        issue_pair_products<NR>(sbase + S::E, sbase + S::WFE, tmem + TM_FILM);
        mma_commit(bar_film);
    }
    __syncwarp();

    // ---------------- pass 1b: scores S^T = K Q^T on warp MMAs (2 heads per warp)
    if (!mbar_wait(bar_kv, 0)) flag_timeout(p.status);
    float sacc[2][4];
    warp_scores2<NR>(sbase + S::K, q, t, hq, qf, sacc);

    // ---------------- combine with FiLM: s' = s(1+gamma)+beta, masked
    if (!mbar_wait(bar_film, 0)) flag_timeout(p.status);
    tc_fence_after();
    const float rs = rsqrtf((float)DH);
    bool valid[4] = {false, false, false, false};
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        const int jl = 32 * (e >> 1) + 8 * q + g8, il = 2 * c4 + (e & 1);
        valid[e] = mi[il] && mj[jl];
        float gm[2], bt[2];
        tmem_ld2(tl + TM_FILM + 16 * e + 2 * hq, gm[0], gm[1]);
        tmem_ld2(tl + TM_FILM + 16 * e + NH + 2 * hq, bt[0], bt[1]);
        tmem_ld_wait();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * hq + hh;
            const float gam = gm[hh] + g[h], bet = bt[hh] + g[NH + h];
            const float sv = sacc[hh][e] * rs * (1.f + gam) + bet;
            sacc[hh][e] = valid[e] ? sv : -INFINITY;
        }
    }

    // ---------------- row statistics: warp, CTA, cluster
    float *wst = reinterpret_cast<float *>(sp + S::WST);
    float *cst = reinterpret_cast<float *>(sp + S::CST);
    float *fin = reinterpret_cast<float *>(sp + S::FIN);
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float m = NR == 2 ? fmaxf(sacc[hh][s], sacc[hh][2 + s]) : sacc[hh][s];
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            float l = 0.f;
            if (m != -INFINITY) {
                l = exp2f((sacc[hh][s] - m) * LOG2E);
                if (NR == 2) l += exp2f((sacc[hh][2 + s] - m) * LOG2E);
            }
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (g8 == 0) {
                const int il = 2 * c4 + s, h = 2 * hq + hh;
                wst[((q * 8 + il) * 8 + h) * 2 + 0] = m;
                wst[((q * 8 + il) * 8 + h) * 2 + 1] = l;
            }
        }
    __syncthreads();
    if (tid < 64) {
        float m = -INFINITY;
#pragma unroll
        for (int k = 0; k < 4; ++k) m = fmaxf(m, wst[(k * 64 + tid) * 2]);
        float l = 0.f;
        if (m != -INFINITY)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float mk = wst[(k * 64 + tid) * 2];
                if (mk != -INFINITY) l += wst[(k * 64 + tid) * 2 + 1] * exp2f((mk - m) * LOG2E);
            }
        cst[tid * 2] = m;
        cst[tid * 2 + 1] = l;
    }
    __syncthreads();
    cluster_wait();     // every peer's receive barriers are armed
    push_rowvals(sp, sbase, S::CST, S::RST, bar_st, tid, rank, nclu);
    if (!mbar_wait(bar_st, 0)) flag_timeout(p.status);
    combine_rowvals<0>(sp, S::RST, S::FIN, tid, nclu);
    __syncthreads();
    if (tid < 64) {
        const float m = fin[tid * 2], l = fin[tid * 2 + 1];
        fin[tid * 2 + 1] = (l > 0.f) ? 1.f / l : 0.f;
        const int il = tid >> 3, h = tid & 7;
        if (rank == 0 && i0 + il < n)
            p.LSE[((size_t)b * NH + h) * n + i0 + il] = (m == -INFINITY) ? -INFINITY : m + logf(l);
    }
    __syncthreads();

    // ---------------- pass 2: normalised coefficients
    const uint32_t L = 32 * q + t;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (e >= NE) {
            sacc[0][e] = sacc[1][e] = 0.f;
            continue;
        }
        const int il = 2 * c4 + (e & 1);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * hq + hh;
            const float m = fin[(il * 8 + h) * 2], linv = fin[(il * 8 + h) * 2 + 1];
            sacc[hh][e] = valid[e] ? exp2f((sacc[hh][e] - m) * LOG2E) * linv : 0.f;
        }
        // edge-update A operand: row 32q+t of tile e, heads 2hq, 2hq+1
        *reinterpret_cast<uint32_t *>(sp + S::A + e * 4096 + ns16(L, 2 * hq)) = pack_bf16(sacc[0][e], sacc[1][e]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    const uint32_t idesc_e = idesc_bf16_f32(128, DE);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int e = 0; e < 2; ++e)
            mma_bf16_ss(tmem + TM_EDGE + 64 * e, smem_desc(sbase + S::A + e * 4096, 128, 256, LAYOUT_NONE),
                        smem_desc(sbase + S::WE, 128, 256, LAYOUT_NONE), idesc_e, 0);
        mma_commit(bar_edge);
    }
    __syncwarp();

    // ---------------- O partial = a V on warp MMAs (overlaps the edge MMAs)
    float oacc[2][2][4];
    warp_contract2<NR>(sbase + S::V, q, t, hq, sacc, oacc);

    // ---------------- E' = E + a We, NR rounds of two MMA tiles
    if (!mbar_wait(bar_e, 0)) flag_timeout(p.status);
    for (int round = 0; round < NR; ++round) {
        if (!mbar_wait(bar_edge, round)) flag_timeout(p.status);
        tc_fence_after();
#pragma unroll
        for (int ee = 0; ee < 2; ++ee) {
            const int e = 2 * round + ee;
            float dv[16];
            tmem_ld16(tl + TM_EDGE + 64 * ee + 16 * hq, dv);
            tmem_ld_wait();
            add_residual16(sp + S::E + tile_off<NR>(e) + L * 128, L, hq, dv);
        }
        if (round + 1 < NR) {
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ee = 0; ee < 2; ++ee)
                    mma_bf16_ss(tmem + TM_EDGE + 64 * ee,
                                smem_desc(sbase + S::A + (2 * (round + 1) + ee) * 4096, 128, 256, LAYOUT_NONE),
                                smem_desc(sbase + S::WE, 128, 256, LAYOUT_NONE), idesc_e, 0);
                mma_commit(bar_edge);
            }
            __syncwarp();
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tma_store_5d(&tmEo, sbase + S::E, 0, i0 / 2, j0, 0, b);
        tma_store_commit();
    }

    // ---------------- O: sum over the quadrant warps and the cluster
    store_quadrant_part(sp, S::OPART, oacc, q, hq, t);
    __syncthreads();
    {
        const uint32_t parts[1] = {S::OPART};
        push_rows_partials<1>(sp, sbase, parts, S::RO, bar_o, tid, rank, nclu);
        if (!mbar_wait(bar_o, 0)) flag_timeout(p.status);
        __nv_bfloat16 *const outs[1] = {p.O};
        const float sc[1] = {1.f};
        finish_rows_partials<1>(sp, S::RO, tid, rank, nclu, outs, b, n, i0, sc);
    }
    if (tid == 0) tma_store_wait_read0();
    tc_fence_before();
    __syncthreads();
    if (W == 0) tmem_dealloc(tmem, TM_COLS);
}

// ------------------------------------------------------------------ host side

template <int NR>
static cudaError_t launch_fwd_nr(const eaga_dims &d, const FwdArgs &a, const uint8_t *img, const float *g,
                                 cudaStream_t st) {
    constexpr int TCN = tile_cols(NR);
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(k_fwd_pairs<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             FwdSmem<NR>::BYTES);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_fwd_pairs<NR>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    CUtensorMap mE, mEo, mK, mV;
    if (!encode_pair_map(&mE, a.E, d.B, d.n, false, TCN) || !encode_pair_map(&mEo, a.Eout, d.B, d.n, false, TCN) ||
        !encode_node_map(&mK, a.K, d.B, d.n, TCN) || !encode_node_map(&mV, a.V, d.B, d.n, TCN))
        return cudaErrorInvalidValue;
    FwdParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.img = img;
    p.g = g;
    p.M = a.M;
    p.O = static_cast<__nv_bfloat16 *>(a.O);
    p.LSE = a.LSE;
    p.status = a.status;
    p.n = d.n;
    p.prefetch_ahead = (uint32_t)(sm_count() * (NR == 1 ? 2 : 1));
    const int nc = (d.n + TCN - 1) / TCN;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, (d.n + TB - 1) / TB, d.B);
    cfg.blockDim = dim3(NTHR);
    cfg.dynamicSmemBytes = FwdSmem<NR>::BYTES;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = nc;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_fwd_pairs<NR>, mE, mEo, mK, mV, p);
}

cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, const uint8_t *img, const float *g,
                             cudaStream_t st) {
    return pick_nr(d.n) == 1 ? launch_fwd_nr<1>(d, a, img, g, st) : launch_fwd_nr<2>(d, a, img, g, st);
}

}  // namespace fast
}  // namespace eaga
