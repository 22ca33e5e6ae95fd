// Forward pair kernel for de = 64, H = 8, dh = 32, bf16 storage (sm_100a).
//
// One CTA owns the tile of 8 query rows i x 64 key columns j of one graph; the
// ceil(n/64) CTAs that share the 8 rows form a thread-block cluster.  Each
// CTA loads its E tile (64 KB) once with TMA and keeps it in shared memory
// for both passes of the layer ("large graphs need two passes", AI-summary
// page, method paragraph):
//   pass 1: FiLM coefficients f = E Wfe on the tensor cores (tcgen05, fp32 in
//           TMEM), scores S = Q K^T with warp MMAs, s' = S(1+gamma)+beta,
//           masked row max / sum over the CTA's 64 columns;
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
// (j = 32r + 8w + t/4, i = 2(t%4) + s) of thread t in warp w: the same pair
// that thread holds in accumulator register e of its m16n8 score tile
// S^T[j,i].  TMEM lane 32w+t therefore feeds thread t directly.
#include <math.h>
#include "common.cuh"
#include "fast.h"
#include "sm100.cuh"

namespace eaga {
namespace fast {

using namespace sm100;

constexpr int DE = 64, NH = 8, DH = 32, HD = 256, NF = 16;
constexpr int IB = 8, JC = 64, NTHR = 128;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t S_E = 0;                  // E tile 64 KB: [s 2][j 64][ic 4][c 64] bf16, 128B-swizzled rows
constexpr uint32_t S_K = 65536;              // K chunk 32 KB: 4 boxes [j 64][d 64], 128B-swizzled
constexpr uint32_t S_V = 98304;              // V chunk 32 KB, same layout
constexpr uint32_t S_WFE = 131072;           // Wfe^T [16][64] bf16, 128B-swizzled (FiLM B operand)
constexpr uint32_t S_WE = S_WFE + 2048;      // We^T [64][16] bf16, no swizzle (edge-update B operand)
constexpr uint32_t S_A = S_WE + 2048;        // 4 tiles [128][16] bf16, no swizzle (edge-update A operand)
constexpr uint32_t S_WST = S_A + 4 * 4096;   // per-warp stats [4][8 i][8 h][2] f32
constexpr uint32_t S_CST = S_WST + 4 * 8 * 8 * 2 * 4;   // CTA stats [8][8][2] f32 (read by peers)
constexpr uint32_t S_FIN = S_CST + 8 * 8 * 2 * 4;       // final m, 1/l [8][8][2] f32
constexpr uint32_t S_G = S_FIN + 8 * 8 * 2 * 4;         // g_b [16] f32
constexpr uint32_t S_MI = S_G + 64;                     // mask of the 8 rows
constexpr uint32_t S_MJ = S_MI + 16;                    // mask of the 64 columns
constexpr uint32_t S_BAR = S_MJ + 64;                   // 4 mbarriers
constexpr uint32_t S_TM = S_BAR + 32;                   // TMEM base address
constexpr uint32_t S_END = S_TM + 16;
constexpr uint32_t SMEM_FWD = S_END + 1024;             // + alignment slack
// reused regions in pass 2
constexpr uint32_t S_OPART = S_K;            // [4 warps][8 i][256] f32 = 32 KB (K chunk is dead)
constexpr uint32_t S_OCTA = S_V;             // [8 i][256] f32 = 8 KB (V chunk is dead)

constexpr uint32_t TM_COLS = 256;            // FiLM: cols 0..63; edge update: cols 64..191
constexpr uint32_t TM_FILM = 0, TM_EDGE = 64;

struct FwdParams {
    const __nv_bfloat16 *Q, *Wfe, *We, *y, *Wfy, *bf;
    const uint8_t *M;
    __nv_bfloat16 *O;
    float *LSE;
    int *status;
    int n, dy;
    float log2e_over_sqrt_dh;   // unused (kept explicit below)
};

__device__ __forceinline__ void flag_timeout(int *status) { atomicExch(status, DEV_TIMEOUT); }

// byte offset of 16-byte chunk `ch` of row `row` inside a 128B-swizzled region
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t ch) { return row * 128u + ((ch ^ (row & 7u)) << 4); }

__global__ void __launch_bounds__(NTHR, 1)
k_fwd_pairs(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmEo,
            const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, FwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, w = tid >> 5, t = tid & 31, c4 = t & 3, g8 = t >> 2;
    const uint32_t rank = cluster_rank();
    const uint32_t nclu = gridDim.x;
    const int n = p.n;
    const int j0 = blockIdx.x * JC, i0 = blockIdx.y * IB, b = blockIdx.z;
    const uint32_t bar_e = sbase + S_BAR, bar_kv = bar_e + 8, bar_film = bar_e + 16, bar_edge = bar_e + 24;
    float *g = reinterpret_cast<float *>(sp + S_G);
    uint8_t *mi = sp + S_MI, *mj = sp + S_MJ;
    bool ok = true;

    // ---------------- setup: barriers, TMA, TMEM, operands
    if (tid == 0) {
        mbar_init(bar_e, 1);
        mbar_init(bar_kv, 1);
        mbar_init(bar_film, 1);
        mbar_init(bar_edge, 1);
        fence_mbar_init();
        prefetch_tmap(&tmE);
        mbar_expect_tx(bar_e, 65536);
        tma_load_5d(sbase + S_E, &tmE, bar_e, 0, i0 / 2, j0, 0, b);
        mbar_expect_tx(bar_kv, 65536);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            tma_load_3d(sbase + S_K + q * 8192, &tmK, bar_kv, 64 * q, j0, b);
            tma_load_3d(sbase + S_V + q * 8192, &tmV, bar_kv, 64 * q, j0, b);
        }
    }
    if (w == 0) {
        tmem_alloc(sbase + S_TM, TM_COLS);
        tmem_relinquish();
    }
    // Wfe^T (K-major, swizzled): element (k, c) of B[N=16][K=64]
    for (int e = tid; e < NF * DE; e += NTHR) {
        const int k = e / DE, c = e % DE;
        const __nv_bfloat16 v = p.Wfe[c * NF + k];
        *reinterpret_cast<__nv_bfloat16 *>(sp + S_WFE + sw128(k, c >> 3) + (c & 7) * 2) = v;
    }
    // We^T (K-major, no swizzle): element (n=c, k=h) of B[N=64][K=16], zero for h >= 8
    for (int e = tid; e < DE * 16; e += NTHR) {
        const int c = e / 16, h = e % 16;
        const __nv_bfloat16 v = h < NH ? p.We[h * DE + c] : __float2bfloat16_rn(0.f);
        *reinterpret_cast<__nv_bfloat16 *>(sp + S_WE + (c >> 3) * 256 + (h >> 3) * 128 + (c & 7) * 16 + (h & 7) * 2) =
            v;
    }
    // edge-update A tiles: zero (the K half h >= 8 stays zero)
    for (int e = tid; e < 4 * 4096 / 16; e += NTHR) reinterpret_cast<uint4 *>(sp + S_A)[e] = make_uint4(0, 0, 0, 0);
    if (tid < NF) {
        float acc = __bfloat162float(p.bf[tid]);
        for (int c = 0; c < p.dy; ++c)
            acc = fmaf(__bfloat162float(p.y[(size_t)b * p.dy + c]), __bfloat162float(p.Wfy[c * NF + tid]), acc);
        g[tid] = acc;
    }
    if (tid < IB) mi[tid] = (i0 + tid < n) ? p.M[(size_t)b * n + i0 + tid] : 0;
    if (tid < JC) mj[tid] = (j0 + tid < n) ? p.M[(size_t)b * n + j0 + tid] : 0;
    // Q fragments (B operand of S^T = K Q^T): rows i0 + g8
    uint32_t qf[NH][2][2];
    {
        const int qi = i0 + g8;
#pragma unroll
        for (int h = 0; h < NH; ++h)
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int d = h * DH + kk * 16 + 2 * c4;
                uint32_t lo = 0, hi = 0;
                if (qi < n) {
                    const __nv_bfloat16 *qrow = p.Q + ((size_t)b * n + qi) * HD;
                    lo = *reinterpret_cast<const uint32_t *>(qrow + d);
                    hi = *reinterpret_cast<const uint32_t *>(qrow + d + 8);
                }
                qf[h][kk][0] = lo;
                qf[h][kk][1] = hi;
            }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S_TM);

    // ---------------- pass 1a: FiLM on the tensor cores (one thread issues)
    if (tid == 0) {
        if (!mbar_wait(bar_e, 0)) { flag_timeout(p.status); ok = false; }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_f32(128, NF);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int r = e >> 1, s = e & 1;
            const uint32_t a0 = sbase + S_E + s * 32768 + r * 16384;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = smem_desc(a0 + kk * 32, 16, 1024, LAYOUT_SW128);
                const uint64_t bd = smem_desc(sbase + S_WFE + kk * 32, 16, 1024, LAYOUT_SW128);
                mma_bf16_ss(tmem + TM_FILM + 16 * e, ad, bd, idesc, kk > 0);
            }
        }
        mma_commit(bar_film);
    }
    __syncwarp();

    // ---------------- pass 1b: scores S^T = K Q^T on warp MMAs
    if (!mbar_wait(bar_kv, 0)) { flag_timeout(p.status); ok = false; }
    float sacc[NH][4];
    {
        // ldmatrix row addresses: matrix mi = t/8: rows j = (mi&1 ? 32 : 0) + 8w + t%8, chunk +(mi>>1)
        const int mrow = ((t >> 3) & 1 ? 32 : 0) + 8 * w + (t & 7);
        const int mch = t >> 4;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            sacc[h][0] = sacc[h][1] = sacc[h][2] = sacc[h][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int q = h >> 1;                               // box of d
                const int ch = ((h & 1) * 32 + kk * 16) / 8 + mch;  // 16-byte chunk in the 128-byte row
                uint32_t a[4];
                ldsm_x4(sbase + S_K + q * 8192 + sw128(mrow, ch), a);
                mma16816(sacc[h], a, qf[h][kk][0], qf[h][kk][1]);
            }
        }
    }

    // ---------------- combine with FiLM: s' = s(1+gamma)+beta, masked
    if (!mbar_wait(bar_film, 0)) { flag_timeout(p.status); ok = false; }
    tc_fence_after();
    const float rs = rsqrtf((float)DH);
    bool valid[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int r = e >> 1, s = e & 1;
        const int jl = 32 * r + 8 * w + g8, il = 2 * c4 + s;
        valid[e] = mi[il] && mj[jl];
        float f[16];
        tmem_ld16(tmem + ((uint32_t)(32 * w) << 16) + TM_FILM + 16 * e, f);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float gam = f[h] + g[h], bet = f[NH + h] + g[NH + h];
            const float sv = sacc[h][e] * rs * (1.f + gam) + bet;
            sacc[h][e] = valid[e] ? sv : -INFINITY;
        }
    }

    // ---------------- row statistics: warp, CTA, cluster
    float *wst = reinterpret_cast<float *>(sp + S_WST);
    float *cst = reinterpret_cast<float *>(sp + S_CST);
    float *fin = reinterpret_cast<float *>(sp + S_FIN);
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            float m = fmaxf(sacc[h][s], sacc[h][2 + s]);
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
            float l = 0.f;
            if (m != -INFINITY) {
                l = exp2f((sacc[h][s] - m) * 1.4426950408889634f) + exp2f((sacc[h][2 + s] - m) * 1.4426950408889634f);
            }
            l += __shfl_xor_sync(0xffffffffu, l, 4);
            l += __shfl_xor_sync(0xffffffffu, l, 8);
            l += __shfl_xor_sync(0xffffffffu, l, 16);
            if (g8 == 0) {
                const int il = 2 * c4 + s;
                wst[((w * 8 + il) * 8 + h) * 2 + 0] = m;
                wst[((w * 8 + il) * 8 + h) * 2 + 1] = l;
            }
        }
    __syncthreads();
    if (tid < 64) {
        float m = -INFINITY;
#pragma unroll
        for (int q = 0; q < 4; ++q) m = fmaxf(m, wst[(q * 64 + tid) * 2]);
        float l = 0.f;
        if (m != -INFINITY)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float mq = wst[(q * 64 + tid) * 2];
                if (mq != -INFINITY) l += wst[(q * 64 + tid) * 2 + 1] * exp2f((mq - m) * 1.4426950408889634f);
            }
        cst[tid * 2] = m;
        cst[tid * 2 + 1] = l;
    }
    cluster_sync();
    if (tid < 64) {
        float mp[16], lp[16];
        float m = -INFINITY;
        for (uint32_t q = 0; q < nclu; ++q) {
            const uint32_t a = map_peer(sbase + S_CST + tid * 8, q);
            mp[q] = ld_peer_f32(a);
            lp[q] = ld_peer_f32(a + 4);
            m = fmaxf(m, mp[q]);
        }
        float l = 0.f;
        if (m != -INFINITY)
            for (uint32_t q = 0; q < nclu; ++q)
                if (mp[q] != -INFINITY) l += lp[q] * exp2f((mp[q] - m) * 1.4426950408889634f);
        fin[tid * 2] = m;
        fin[tid * 2 + 1] = (l > 0.f) ? 1.f / l : 0.f;
        const int il = tid >> 3, h = tid & 7;
        if (rank == 0 && i0 + il < n)
            p.LSE[((size_t)b * NH + h) * n + i0 + il] = (m == -INFINITY) ? -INFINITY : m + logf(l);
    }
    __syncthreads();

    // ---------------- pass 2: normalised coefficients
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int il = 2 * c4 + (e & 1);
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const float m = fin[(il * 8 + h) * 2], il_ = fin[(il * 8 + h) * 2 + 1];
            sacc[h][e] = valid[e] ? exp2f((sacc[h][e] - m) * 1.4426950408889634f) * il_ : 0.f;
        }
    }
    // edge-update A operand: row 32w+t of tile e holds a[0..7] of this thread's pair e
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        uint4 v;
        v.x = pack_bf16(sacc[0][e], sacc[1][e]);
        v.y = pack_bf16(sacc[2][e], sacc[3][e]);
        v.z = pack_bf16(sacc[4][e], sacc[5][e]);
        v.w = pack_bf16(sacc[6][e], sacc[7][e]);
        const int L = 32 * w + t;
        *reinterpret_cast<uint4 *>(sp + S_A + e * 4096 + (L >> 3) * 256 + (L & 7) * 16) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    const uint32_t idesc_e = idesc_bf16_f32(128, DE);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const uint64_t ad = smem_desc(sbase + S_A + e * 4096, 128, 256, LAYOUT_NONE);
            const uint64_t bd = smem_desc(sbase + S_WE, 128, 256, LAYOUT_NONE);
            mma_bf16_ss(tmem + TM_EDGE + 64 * e, ad, bd, idesc_e, 0);
        }
        mma_commit(bar_edge);
    }

    // ---------------- O partial = a V on warp MMAs (overlaps the edge MMAs)
    float oacc[NH][2][4];
    {
        const int vrow = ((t >> 4) & 1 ? 32 : 0) + 8 * w + (t & 7);
        const int vch = (t >> 3) & 1;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
            const uint32_t lo = pack_bf16(sacc[h][0], sacc[h][1]);
            const uint32_t hi = pack_bf16(sacc[h][2], sacc[h][3]);
            const uint32_t b0 = movmatrix_t(lo), b1 = movmatrix_t(hi);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                oacc[h][mt][0] = oacc[h][mt][1] = oacc[h][mt][2] = oacc[h][mt][3] = 0.f;
                const int d0 = h * DH + mt * 16;
                const int q = d0 >> 6, ch = (d0 & 63) / 8 + vch;
                uint32_t a[4];
                ldsm_x4_t(sbase + S_V + q * 8192 + sw128(vrow, ch), a);
                mma16816(oacc[h][mt], a, b0, b1);
            }
        }
    }

    // ---------------- E' = E + a We for the 4 MMA tiles (two rounds of two)
    if (!mbar_wait(bar_e, 0)) { flag_timeout(p.status); ok = false; }
    for (int round = 0; round < 2; ++round) {
        if (!mbar_wait(bar_edge, round)) { flag_timeout(p.status); ok = false; }
        tc_fence_after();
#pragma unroll
        for (int ee = 0; ee < 2; ++ee) {
            const int e = 2 * round + ee, r = e >> 1, s = e & 1;
            const uint32_t L = 32 * w + t;
            const uint32_t row_base = S_E + s * 32768 + r * 16384 + L * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float dv[16];
                tmem_ld16(tmem + ((uint32_t)(32 * w) << 16) + TM_EDGE + 64 * ee + 16 * q, dv);
                tmem_ld_wait();
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t ch = 2 * q + hh;
                    uint4 *ptr = reinterpret_cast<uint4 *>(sp + row_base + ((ch ^ (L & 7u)) << 4));
                    uint4 ev = *ptr;
                    __nv_bfloat162 *e2 = reinterpret_cast<__nv_bfloat162 *>(&ev);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float2 x = __bfloat1622float2(e2[u]);
                        e2[u] = __floats2bfloat162_rn(x.x + dv[8 * hh + 2 * u], x.y + dv[8 * hh + 2 * u + 1]);
                    }
                    *ptr = ev;
                }
            }
        }
        if (round == 0) {
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ee = 0; ee < 2; ++ee) {
                    const uint64_t ad = smem_desc(sbase + S_A + (2 + ee) * 4096, 128, 256, LAYOUT_NONE);
                    const uint64_t bd = smem_desc(sbase + S_WE, 128, 256, LAYOUT_NONE);
                    mma_bf16_ss(tmem + TM_EDGE + 64 * ee, ad, bd, idesc_e, 0);
                }
                mma_commit(bar_edge);
            }
            __syncwarp();
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tma_store_5d(&tmEo, sbase + S_E, 0, i0 / 2, j0, 0, b);
        tma_store_commit();
    }

    // ---------------- O: sum over warps, then over the cluster
    float *opart = reinterpret_cast<float *>(sp + S_OPART);
#pragma unroll
    for (int h = 0; h < NH; ++h)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = h * DH + mt * 16 + g8 + 8 * (e >> 1), il = 2 * c4 + (e & 1);
                opart[(w * IB + il) * HD + d] = oacc[h][mt][e];
            }
    __syncthreads();
    float *octa = reinterpret_cast<float *>(sp + S_OCTA);
    for (int x = tid; x < IB * HD; x += NTHR)
        octa[x] = opart[x] + opart[IB * HD + x] + opart[2 * IB * HD + x] + opart[3 * IB * HD + x];
    cluster_sync();
    {
        const int per = (IB * HD / 4 + nclu - 1) / nclu;   // float4 groups per CTA
        for (int gq = rank * per + tid; gq < min((int)(rank + 1) * per, IB * HD / 4); gq += NTHR) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t q = 0; q < nclu; ++q) {
                const float4 v = ld_peer_f32x4(map_peer(sbase + S_OCTA + gq * 16, q));
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            const int il = (gq * 4) / HD, d = (gq * 4) % HD;
            if (i0 + il < n) {
                __nv_bfloat162 *o = reinterpret_cast<__nv_bfloat162 *>(p.O + ((size_t)b * n + i0 + il) * HD + d);
                o[0] = __floats2bfloat162_rn(acc.x, acc.y);
                o[1] = __floats2bfloat162_rn(acc.z, acc.w);
            }
        }
    }
    cluster_sync();
    if (tid == 0) tma_store_wait0();
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, TM_COLS);
    (void)ok;
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// E viewed as 5-D (c, ic, j, s, b) with i = 2ic + s; box (64, 4, 64, 2, 1).
bool encode_pair_map(CUtensorMap *m, const void *base, int B, int n) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[5] = {DE, (cuuint64_t)(n / 2), (cuuint64_t)n, 2, (cuuint64_t)B};
    const cuuint64_t rowb = DE * 2;
    const cuuint64_t strides[4] = {2 * (cuuint64_t)n * rowb, rowb, (cuuint64_t)n * rowb,
                                   (cuuint64_t)n * n * rowb};
    const cuuint32_t box[5] = {64, 4, 64, 2, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B, n, 256] node tensor; box (64 d, 64 rows, 1).
bool encode_node_map(CUtensorMap *m, const void *base, int B, int n) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {HD, (cuuint64_t)n, (cuuint64_t)B};
    const cuuint64_t strides[2] = {HD * 2, (cuuint64_t)n * HD * 2};
    const cuuint32_t box[3] = {64, 64, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, cudaStream_t st) {
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(k_fwd_pairs, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_FWD);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(k_fwd_pairs, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    CUtensorMap mE, mEo, mK, mV;
    if (!encode_pair_map(&mE, a.E, d.B, d.n) || !encode_pair_map(&mEo, a.Eout, d.B, d.n) ||
        !encode_node_map(&mK, a.K, d.B, d.n) || !encode_node_map(&mV, a.V, d.B, d.n))
        return cudaErrorInvalidValue;
    FwdParams p;
    p.Q = static_cast<const __nv_bfloat16 *>(a.Q);
    p.Wfe = static_cast<const __nv_bfloat16 *>(a.w[6]);
    p.Wfy = static_cast<const __nv_bfloat16 *>(a.w[7]);
    p.bf = static_cast<const __nv_bfloat16 *>(a.w[8]);
    p.We = static_cast<const __nv_bfloat16 *>(a.w[9]);
    p.y = static_cast<const __nv_bfloat16 *>(a.y);
    p.M = a.M;
    p.O = static_cast<__nv_bfloat16 *>(a.O);
    p.LSE = a.LSE;
    p.status = a.status;
    p.n = d.n;
    p.dy = d.dy;
    p.log2e_over_sqrt_dh = 0.f;
    const int nc = (d.n + JC - 1) / JC;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, (d.n + IB - 1) / IB, d.B);
    cfg.blockDim = dim3(NTHR);
    cfg.dynamicSmemBytes = SMEM_FWD;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = nc;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_fwd_pairs, mE, mEo, mK, mV, p);
}

}  // namespace fast
}  // namespace eaga
