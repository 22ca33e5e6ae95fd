// Node-side GEMMs on tcgen05: C[M, N] = sum_seg A_seg[M, K] B_seg[K, N], A
// K-major (row-major [M, K]); B either K-major (stored [N, K]) or MN-major
// (stored [K, N], one matrix per output when the outputs are several); 128B-swizzled tiles
// loaded by TMA through a 4-stage mbarrier pipeline, the 128 x BN fp32
// accumulator in TMEM, and the layer's epilogues fused:
//   QKV      [Q|K|V] = X [Wq|Wk|Wv] + b, masked rows zero   (B = Wq, Wk, Wv, MN-major)
//   out-proj X' = X + M (O Wo + bo)                         (B = Wo, MN-major)
//   dO       dO = M (dX' Wo^T)                              (Bt = Wo)
//   dX       dX = dX' + dQ Wq^T + dK Wk^T + dV Wv^T          (three segments, Bt = W)
// and the node FFN of the graph-transformer block around the layer:
//   FFN1     H = relu(A W1 + b1)                             (B = W1, MN-major)
//   FFN2     Z = R + H W2 + b2                               (B = W2, MN-major)
//   DRELU    dH = (dZ W2^T) [R > 0]   (R = H)                (Bt = W2)
// One thread issues TMA and MMAs; the four warps run the epilogue from TMEM.
// k_tc_wgrad computes the weight gradients A^T B over node rows (split-K fp32
// partials) with both operands read MN-major straight from the row-major
// node tensors.
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using dev::cta_wait;

constexpr int TBM = 128, TBK = 64, TTHR = 128;
// pipeline stages: 4 for 64-wide tiles, 3 for 128-wide (two CTAs fit an SM either way)
template <int BN> constexpr int tc_stages() { return BN == 128 ? 3 : 4; }
enum TcMode { TC_QKV = 0, TC_OUT = 1, TC_DO = 2, TC_DX = 3, TC_FFN1 = 4, TC_FFN2 = 5, TC_DRELU = 6 };

struct TcParams {
    const __nv_bfloat16 *bias[3];
    __nv_bfloat16 *C[3];
    const __nv_bfloat16 *R;      // residual [M, Nb]
    const uint8_t *mask;         // [M] (QKV, OUT, DO)
    int *status;
    int M, K, Nb, nseg, mode;
    int b_mn;                    // B stored [K, N] (MN-major), map chosen by output matrix
};

template <int BN, int TSTAGES = tc_stages<BN>()>
struct TcSmem {
    static constexpr uint32_t A_BYTES = TBM * TBK * 2, B_BYTES = BN * TBK * 2;
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr uint32_t BAR = TSTAGES * STAGE;        // full[S], empty[S], done
    static constexpr uint32_t TM = BAR + (2 * TSTAGES + 1) * 8;
    static constexpr uint32_t FAIL = TM + 4;                 // CTA failure flag (a wait ran out)
    static constexpr uint32_t BIAS = TM + 16;                // the tile's BN bias values, fp32
    static constexpr uint32_t BYTES = BIAS + BN * 4 + 1024;
};

template <int BN>
__global__ void __launch_bounds__(TTHR, 1)
k_tc_gemm(const __grid_constant__ CUtensorMap a0, const __grid_constant__ CUtensorMap a1,
          const __grid_constant__ CUtensorMap a2, const __grid_constant__ CUtensorMap b0,
          const __grid_constant__ CUtensorMap b1, const __grid_constant__ CUtensorMap b2, TcParams p) {
    using S = TcSmem<BN>;
    constexpr int TSTAGES = tc_stages<BN>();
    griddep_launch_dependents();
    griddep_wait();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, w = tid >> 5, t = tid & 31;
    const int n0 = blockIdx.x * BN, m0 = blockIdx.y * TBM;
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);
    const uint32_t bar0 = sbase + S::BAR;
    auto full = [&](int s) { return bar0 + 8 * s; };
    auto empty = [&](int s) { return bar0 + 8 * (TSTAGES + s); };
    const uint32_t done = bar0 + 16 * TSTAGES;
    const int kt_seg = p.K / TBK, nk = kt_seg * p.nseg;
    const int which_n = n0 / p.Nb, ncol0 = n0 % p.Nb;

    if (tid == 0) {
        for (int s = 0; s < TSTAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        *reinterpret_cast<volatile int *>(sp + S::FAIL) = 0;
    }
    if (w == 0) {
        tmem_alloc(sbase + S::TM, BN);
        tmem_relinquish();
    }
    float *sbias = reinterpret_cast<float *>(sp + S::BIAS);
    const bool has_bias = p.mode == TC_QKV || p.mode == TC_OUT || p.mode == TC_FFN1 || p.mode == TC_FFN2;
    for (int c = tid; c < BN; c += TTHR) {
        const int ng = n0 + c;
        sbias[c] = has_bias ? __bfloat162float(p.bias[ng / p.Nb][ng % p.Nb]) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);

    if (tid == 0) {
        auto issue_load = [&](int kt) {
            const int s = kt % TSTAGES, seg = kt / kt_seg, k0 = (kt % kt_seg) * TBK;
            const CUtensorMap *am = seg == 0 ? &a0 : seg == 1 ? &a1 : &a2;
            const int bsel = p.b_mn ? which_n : seg;
            const CUtensorMap *bm = bsel == 0 ? &b0 : bsel == 1 ? &b1 : &b2;
            const uint32_t st = sbase + s * S::STAGE;
            mbar_expect_tx(full(s), S::STAGE);
            tma_load_2d(st, am, full(s), k0, m0);
            if (p.b_mn) {
                // [64 k rows][64 n] boxes, 8 KB apart along N
#pragma unroll
                for (int h = 0; h < BN / 64; ++h) tma_load_2d(st + S::A_BYTES + h * 8192, bm, full(s), ncol0 + 64 * h, k0);
            } else {
                tma_load_2d(st + S::A_BYTES, bm, full(s), k0, n0);
            }
        };
        int issued = 0;
        for (; issued < TSTAGES && issued < nk; ++issued) issue_load(issued);
        const uint32_t idesc = idesc_bf16_f32(TBM, BN) | (p.b_mn ? (1u << 16) : 0u);
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % TSTAGES;
            const uint32_t ph = (kt / TSTAGES) & 1;
            if (!cta_wait(full(s), ph, fail, p.status)) break;
            tc_fence_after();
            const uint32_t st = sbase + s * S::STAGE;
#pragma unroll
            for (int kk = 0; kk < TBK / 16; ++kk)
                mma_bf16_ss(tmem, smem_desc(st + kk * 32, 16, 1024, LAYOUT_SW128),
                            p.b_mn ? smem_desc(st + S::A_BYTES + kk * 2048, 8192, 1024, LAYOUT_SW128)
                                   : smem_desc(st + S::A_BYTES + kk * 32, 16, 1024, LAYOUT_SW128),
                            idesc, (kt > 0 || kk > 0) ? 1u : 0u);
            mma_commit(empty(s));
            if (kt + TSTAGES < nk) {
                if (!cta_wait(empty(s), ph, fail, p.status)) break;
                issue_load(issued++);
            }
        }
        mma_commit(done);
        if (*fail) {   // what was issued completes before the CTA's memory is released
            for (int kt = max(issued - TSTAGES, 0); kt < issued; ++kt) mbar_wait(full(kt % TSTAGES), (kt / TSTAGES) & 1);
            mbar_wait(done, 0);
        }
    }
    __syncwarp();
    // epilogue: warp w holds rows m0 + 32w + t.  The residual row segment is
    // loaded into registers before the accumulator is ready.
    const int row = m0 + 32 * w + t;
    const bool in = row < p.M;
    const bool mk = in && (p.mask == nullptr || p.mask[in ? row : 0] != 0);
    const bool has_res = p.mode == TC_OUT || p.mode == TC_DX || p.mode == TC_FFN2 || p.mode == TC_DRELU;
    const int which0 = n0 / p.Nb, col0 = n0 % p.Nb;     // BN divides Nb: one output per tile
    const size_t obase = (size_t)(in ? row : 0) * p.Nb + col0;
    uint4 res[BN / 8];
#pragma unroll
    for (int u = 0; u < BN / 8; ++u)
        res[u] = (has_res && in) ? reinterpret_cast<const uint4 *>(p.R + obase)[u] : make_uint4(0, 0, 0, 0);
    cta_wait(done, 0, fail, p.status);
    tc_fence_after();
#pragma unroll
    for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * w) << 16) + c0, v);
        tmem_ld_wait();
        if (!in) continue;
#pragma unroll
        for (int u = 0; u < 16; ++u) v[u] += sbias[c0 + u];
        uint4 outv[2];
        __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(outv);
        if (p.mode == TC_QKV || p.mode == TC_DO) {
#pragma unroll
            for (int u = 0; u < 8; ++u)
                o2[u] = mk ? __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]) : __floats2bfloat162_rn(0.f, 0.f);
        } else if (p.mode == TC_FFN1) {
#pragma unroll
            for (int u = 0; u < 8; ++u) o2[u] = __floats2bfloat162_rn(fmaxf(v[2 * u], 0.f), fmaxf(v[2 * u + 1], 0.f));
        } else if (p.mode == TC_DRELU) {
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 r4 = res[c0 / 8 + (u >> 2)];
                const float2 h = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162 *>(&r4)[u & 3]);
                o2[u] = __floats2bfloat162_rn(h.x > 0.f ? v[2 * u] : 0.f, h.y > 0.f ? v[2 * u + 1] : 0.f);
            }
        } else {
            const bool add = p.mode == TC_DX || p.mode == TC_FFN2 || mk;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 r4 = res[c0 / 8 + (u >> 2)];
                const __nv_bfloat162 xr = reinterpret_cast<const __nv_bfloat162 *>(&r4)[u & 3];
                const float2 x = __bfloat1622float2(xr);
                o2[u] = add ? __floats2bfloat162_rn(x.x + v[2 * u], x.y + v[2 * u + 1]) : xr;
            }
        }
        uint4 *dst = reinterpret_cast<uint4 *>(p.C[which0] + obase + c0);
        dst[0] = outv[0];
        dst[1] = outv[1];
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, BN);
}

// ------------------------------------------------------------------ weight gradients
// P[z] = A[rows of split z]^T B[rows of split z]: A [K rows][M] and B [K rows][N]
// row-major (K = node rows), i.e. both MN-major for the product.  TMA boxes of
// 64 rows x 64 columns land as 64 swizzled 128-byte rows: one MN atom of 64
// elements by 8 atoms of 8 rows along K.  An M (or N) tile of 128 is two such
// boxes 8 KB apart (the descriptor's leading offset); 8-row groups are 1 KB
// apart (stride offset); each MMA consumes 16 rows.
struct WgParams {
    float *P[3];                 // [splits][M][Nb] fp32 per output matrix
    int *status;
    int M, K, Nb, kchunk;
};

template <int BN>
struct WgSmem {
    static constexpr uint32_t A_BYTES = TBM * TBK * 2, B_BYTES = BN * TBK * 2;
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr int ST = 3;
    static constexpr uint32_t BAR = ST * STAGE;
    static constexpr uint32_t TM = BAR + (2 * ST + 1) * 8;
    static constexpr uint32_t FAIL = TM + 4;                 // CTA failure flag (a wait ran out)
    static constexpr uint32_t BYTES = TM + 16 + 1024;
};

template <int BN>
__global__ void __launch_bounds__(TTHR, 1)
k_tc_wgrad(const __grid_constant__ CUtensorMap a0, const __grid_constant__ CUtensorMap b0,
           const __grid_constant__ CUtensorMap b1, const __grid_constant__ CUtensorMap b2, WgParams p) {
    using S = WgSmem<BN>;
    constexpr int ST = S::ST;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, w = tid >> 5, t = tid & 31;
    const int n0g = blockIdx.x * BN, m0 = blockIdx.y * TBM;
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);
    const int which = n0g / p.Nb, n0 = n0g % p.Nb;
    const int kbeg = blockIdx.z * p.kchunk, kend = min(p.K, kbeg + p.kchunk);
    const int nk = kend > kbeg ? (kend - kbeg + TBK - 1) / TBK : 0;
    const CUtensorMap *bm = which == 0 ? &b0 : which == 1 ? &b1 : &b2;
    const uint32_t bar0 = sbase + S::BAR;
    auto full = [&](int s) { return bar0 + 8 * s; };
    auto empty = [&](int s) { return bar0 + 8 * (ST + s); };
    const uint32_t done = bar0 + 16 * ST;

    if (tid == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        *reinterpret_cast<volatile int *>(sp + S::FAIL) = 0;
    }
    if (w == 0) {
        tmem_alloc(sbase + S::TM, BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);

    if (tid == 0) {
        auto issue_load = [&](int kt) {
            const int s = kt % ST, k0 = kbeg + kt * TBK;
            const uint32_t st = sbase + s * S::STAGE;
            mbar_expect_tx(full(s), S::STAGE);
#pragma unroll
            for (int h = 0; h < TBM / 64; ++h) tma_load_2d(st + h * 8192, &a0, full(s), m0 + 64 * h, k0);
#pragma unroll
            for (int h = 0; h < BN / 64; ++h) tma_load_2d(st + S::A_BYTES + h * 8192, bm, full(s), n0 + 64 * h, k0);
        };
        int issued = 0;
        for (; issued < ST && issued < nk; ++issued) issue_load(issued);
        const uint32_t idesc = idesc_bf16_f32_mn(TBM, BN);
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % ST;
            const uint32_t ph = (kt / ST) & 1;
            if (!cta_wait(full(s), ph, fail, p.status)) break;
            tc_fence_after();
            const uint32_t st = sbase + s * S::STAGE;
#pragma unroll
            for (int kk = 0; kk < TBK / 16; ++kk)
                mma_bf16_ss(tmem, smem_desc(st + kk * 2048, 8192, 1024, LAYOUT_SW128),
                            smem_desc(st + S::A_BYTES + kk * 2048, 8192, 1024, LAYOUT_SW128), idesc,
                            (kt > 0 || kk > 0) ? 1u : 0u);
            mma_commit(empty(s));
            if (kt + ST < nk) {
                if (!cta_wait(empty(s), ph, fail, p.status)) break;
                issue_load(issued++);
            }
        }
        mma_commit(done);
        if (*fail) {   // what was issued completes before the CTA's memory is released
            for (int kt = max(issued - ST, 0); kt < issued; ++kt) mbar_wait(full(kt % ST), (kt / ST) & 1);
            mbar_wait(done, 0);
        }
    }
    __syncwarp();
    cta_wait(done, 0, fail, p.status);
    tc_fence_after();
    const int row = m0 + 32 * w + t;
    float *P = p.P[which] + (size_t)blockIdx.z * p.M * p.Nb + (size_t)row * p.Nb + n0;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(32 * w) << 16) + c0, v);
        tmem_ld_wait();
        if (row >= p.M) continue;
        if (nk == 0) {
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] = 0.f;
        }
        float4 *dst = reinterpret_cast<float4 *>(P + c0);
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, BN);
}

// ------------------------------------------------------------------ host side

bool encode_2d(CUtensorMap *m, const void *base, int rows, int cols, int box_rows);

template <int BN>
static cudaError_t tc_launch(const CUtensorMap (&am)[3], const CUtensorMap (&bm)[3], const TcParams &p, int N,
                             cudaStream_t st) {
    static std::atomic<uint32_t> attr_set{0};
    if (cudaError_t e = ensure_smem_attr(k_tc_gemm<BN>, TcSmem<BN>::BYTES, attr_set); e != cudaSuccess) return e;
    dim3 grid(N / BN, (p.M + TBM - 1) / TBM);
    return launch_pdl(k_tc_gemm<BN>, grid, dim3(TTHR), TcSmem<BN>::BYTES, st, 1, am[0], am[1], am[2], bm[0], bm[1],
                      bm[2], p);
}

// Out = epilogue(sum_seg A[seg] B[seg]): A[seg] [M, K] row-major bf16; B[seg] stored
// [N, K] (b_mn = false), or, with b_mn, B[q] stored [K, Nb] for output matrix q.
cudaError_t tc_gemm(int mode, int M, int N, int K, int nseg, const void *const A[3], const void *const B[3],
                    const void *const bias[3], void *const C[3], int Nb, const void *R, const uint8_t *mask,
                    int *status, cudaStream_t st, bool b_mn) {
    CUtensorMap am[3], bm[3];
    // N is a multiple of 64; the wider tile only where it divides N (and each output)
    const int BN = (N >= 512 && N % 128 == 0 && Nb % 128 == 0) ? 128 : 64;
    const int nb_maps = b_mn ? N / Nb : nseg;
    for (int s = 0; s < 3; ++s) {
        const int sa = s < nseg ? s : 0, sb = s < nb_maps ? s : 0;
        if (!encode_2d(&am[s], A[sa], M, K, TBM)) return cudaErrorInvalidValue;
        if (!(b_mn ? encode_2d(&bm[s], B[sb], K, Nb, 64) : encode_2d(&bm[s], B[sb], N, K, BN)))
            return cudaErrorInvalidValue;
    }
    TcParams p = {};
    for (int s = 0; s < 3; ++s) {
        p.bias[s] = static_cast<const __nv_bfloat16 *>(bias ? bias[s] : nullptr);
        p.C[s] = static_cast<__nv_bfloat16 *>(C[s]);
    }
    p.R = static_cast<const __nv_bfloat16 *>(R);
    p.mask = mask;
    p.status = status;
    p.M = M; p.K = K; p.Nb = Nb; p.nseg = nseg; p.mode = mode; p.b_mn = b_mn ? 1 : 0;
    return BN == 128 ? tc_launch<128>(am, bm, p, N, st) : tc_launch<64>(am, bm, p, N, st);
}

// A [K][M] row-major with 64 x 64 boxes (one MN atom of 64 columns by 64 rows).
static bool encode_mn(CUtensorMap *m, const void *base, int rows, int cols) { return encode_2d(m, base, rows, cols, 64); }

template <int BN>
static cudaError_t wg_launch(const CUtensorMap &am, const CUtensorMap (&bm)[3], const WgParams &p, int N, int splits,
                             cudaStream_t st) {
    static std::atomic<uint32_t> attr_set{0};
    if (cudaError_t e = ensure_smem_attr(k_tc_wgrad<BN>, WgSmem<BN>::BYTES, attr_set); e != cudaSuccess) return e;
    dim3 grid(N / BN, (p.M + TBM - 1) / TBM, splits);
    k_tc_wgrad<BN><<<grid, TTHR, WgSmem<BN>::BYTES, st>>>(am, bm[0], bm[1], bm[2], p);
    return cudaGetLastError();
}

// Split-K weight-gradient partials P_q[z] = A[rows of split z]^T B_q[rows of split z]
// for q < nout: A [K][M], B_q [K][Nb] row-major bf16, outputs [splits][M][Nb] fp32.
cudaError_t tc_wgrad(int M, int Nb, int nout, int K, int splits, const void *A, const void *const B[3],
                     float *const P[3], int *status, cudaStream_t st) {
    CUtensorMap am, bm[3];
    if (!encode_mn(&am, A, K, M)) return cudaErrorInvalidValue;
    for (int q = 0; q < 3; ++q)
        if (!encode_mn(&bm[q], B[q < nout ? q : 0], K, Nb)) return cudaErrorInvalidValue;
    WgParams p = {};
    for (int q = 0; q < 3; ++q) p.P[q] = P[q < nout ? q : 0];
    p.status = status;
    p.M = M; p.K = K; p.Nb = Nb;
    p.kchunk = ((K + splits - 1) / splits + TBK - 1) / TBK * TBK;
    const int N = Nb * nout;
    const int BN = (N % 128 == 0 && Nb % 128 == 0) ? 128 : 64;
    return BN == 128 ? wg_launch<128>(am, bm, p, N, splits, st) : wg_launch<64>(am, bm, p, N, splits, st);
}

}  // namespace fast
}  // namespace eaga
