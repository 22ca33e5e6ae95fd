// Weight gradients of the node projections on warp MMAs (bf16 operands, fp32
// accumulation): X^T dQ, X^T dK, X^T dV and O^T dX' (O is zero on masked
// rows) as split-K fp32 partials over row chunks, summed in a fixed order by
// the finishing kernel.  64x64 output tile per CTA, 4 warps of 32x32, K (the
// node rows) in steps of 32 through a two-stage cp.async pipeline, 16-byte
// swizzled shared-memory rows.
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;

constexpr int GBM = 64, GBN = 64, GBK = 32, GTHR = 128;
struct GemmParams {
    const __nv_bfloat16 *A[3];       // per K-segment; [M,K] (or [K,M] when A is transposed)
    const __nv_bfloat16 *B[3];       // per output matrix
    float *P[3];                     // fp32 split-K partials [splits][M, Nb]
    int M, K, Nb, lda, ldb, nseg, kchunk;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred) {
    const int sz = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// [rows][32] bf16 tile (64 B rows): chunk c of row r
__device__ __forceinline__ uint32_t off64(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }
// [rows][64] bf16 tile (128 B rows): chunk c of row r
__device__ __forceinline__ uint32_t off128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// AT: A is stored [K, M] (row stride lda) and read transposed.  BT: B is stored [N, K].
template <bool AT, bool BT>
__global__ void __launch_bounds__(GTHR) k_node_gemm(GemmParams p) {
    __shared__ __align__(128) uint8_t sA[2][GBM * GBK * 2];
    __shared__ __align__(128) uint8_t sB[2][GBK * GBN * 2];
    const int tid = threadIdx.x, w = tid >> 5, t = tid & 31;
    const int n0g = blockIdx.x * GBN, m0 = blockIdx.y * GBM;
    const int which = n0g / p.Nb, n0 = n0g % p.Nb;
    const int wm = (w >> 1) * 32, wn = (w & 1) * 32;
    const int kbeg = blockIdx.z * p.kchunk;
    const int kend = min(p.K, kbeg + p.kchunk);
    float acc[2][4][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

    const int nseg = p.nseg;
    const int nk_seg = (kend - kbeg + GBK - 1) / GBK;
    const int nk = nk_seg * nseg;
    auto load = [&](int stage, int it) {
        const int seg = it / nk_seg, k0 = kbeg + (it % nk_seg) * GBK;
        const __nv_bfloat16 *A = p.A[nseg > 1 ? seg : 0];
        const __nv_bfloat16 *Bm = p.B[nseg > 1 ? seg : which];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = tid + q * GTHR;
            if (!AT) {   // [64 m][32 k]
                const int r = idx >> 2, c = idx & 3, gm = m0 + r, gk = k0 + c * 8;
                const bool ok = gm < p.M && gk < kend;
                cp_async16(smem_u32(sA[stage]) + off64(r, c), A + (ok ? (size_t)gm * p.lda + gk : 0), ok);
            } else {     // [32 k][64 m]
                const int r = idx >> 3, c = idx & 7, gk = k0 + r, gm = m0 + c * 8;
                const bool ok = gk < kend && gm < p.M;
                cp_async16(smem_u32(sA[stage]) + off128(r, c), A + (ok ? (size_t)gk * p.lda + gm : 0), ok);
            }
            if (!BT) {   // [32 k][64 n]
                const int r = idx >> 3, c = idx & 7, gk = k0 + r;
                const bool ok = gk < kend;
                cp_async16(smem_u32(sB[stage]) + off128(r, c), Bm + (ok ? (size_t)gk * p.ldb + n0 + c * 8 : 0), ok);
            } else {     // [64 n][32 k]
                const int r = idx >> 2, c = idx & 3, gk = k0 + c * 8;
                const bool ok = gk < kend;
                cp_async16(smem_u32(sB[stage]) + off64(r, c), Bm + (ok ? (size_t)(n0 + r) * p.ldb + gk : 0), ok);
            }
        }
        cp_async_commit();
    };

    if (nk > 0) load(0, 0);
    for (int it = 0; it < nk; ++it) {
        if (it + 1 < nk) {
            load((it + 1) & 1, it + 1);
            cp_async_wait1();
        } else {
            cp_async_wait0();
        }
        __syncthreads();
        const uint32_t a_s = smem_u32(sA[it & 1]), b_s = smem_u32(sB[it & 1]);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t af[2][4], bfr[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                if (!AT) {
                    // (m 0-7, k 0-7), (m 8-15, k 0-7), (m 0-7, k 8-15), (m 8-15, k 8-15)
                    const int r = wm + mt * 16 + (t & 7) + ((t >> 3) & 1) * 8;
                    ldsm_x4(a_s + off64(r, ks * 2 + (t >> 4)), af[mt]);
                } else {
                    // stored [k][m]: matrices as above via .trans of [k rows][m cols]
                    const int kr = ks * 16 + (t & 7) + ((t >> 4) & 1) * 8;
                    const int c = (wm + mt * 16) / 8 + ((t >> 3) & 1);
                    ldsm_x4_t(a_s + off128(kr, c), af[mt]);
                }
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                if (!BT) {
                    // (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
                    const int kr = ks * 16 + (t & 7) + ((t >> 3) & 1) * 8;
                    ldsm_x4_t(b_s + off128(kr, (wn + np * 16) / 8 + (t >> 4)), bfr[np]);
                } else {
                    // stored [n][k]: non-trans rows n
                    const int r = wn + np * 16 + (t & 7) + ((t >> 4) & 1) * 8;
                    ldsm_x4(b_s + off64(r, ks * 2 + ((t >> 3) & 1)), bfr[np]);
                }
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    mma16816(acc[mt][nt], af[mt], bfr[nt >> 1][(nt & 1) * 2], bfr[nt >> 1][(nt & 1) * 2 + 1]);
        }
        __syncthreads();
    }
    // epilogue
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + wm + mt * 16 + (t >> 2) + hh * 8;
                const int col = n0 + wn + nt * 8 + (t & 3) * 2;
                if (row >= p.M) continue;
                const size_t o = (size_t)row * p.Nb + col;
                float *P = p.P[which] + (size_t)blockIdx.z * p.M * p.Nb;
                *reinterpret_cast<float2 *>(P + o) = make_float2(acc[mt][nt][hh * 2], acc[mt][nt][hh * 2 + 1]);
            }
}

static inline const __nv_bfloat16 *bf(const void *p) { return static_cast<const __nv_bfloat16 *>(p); }

// Split-K weight-gradient partials: P_q[z] = (rows of chunk z of A)^T B_q.
//   X^T [dQ|dK|dV] -> 3 matrices [dx, 256];  O^T dX' -> [256, dx]
cudaError_t launch_wgrad(const eaga_dims &d, const BwdArgs &a, const __nv_bfloat16 *dN[3], float *parts,
                         int splits, cudaStream_t st) {
    const int rows = d.B * d.n, kchunk = ((rows + splits - 1) / splits + GBK - 1) / GBK * GBK;
    const size_t msz = (size_t)splits * d.dx * HD;
    GemmParams p = {};
    p.A[0] = bf(a.X);
    for (int q = 0; q < 3; ++q) {
        p.B[q] = dN[q];
        p.P[q] = parts + q * msz;
    }
    p.M = d.dx; p.K = rows; p.Nb = HD; p.lda = d.dx; p.ldb = HD; p.nseg = 1; p.kchunk = kchunk;
    k_node_gemm<true, false><<<dim3(3 * HD / GBN, (d.dx + GBM - 1) / GBM, splits), GTHR, 0, st>>>(p);
    GemmParams o = {};
    o.A[0] = bf(a.O);
    o.B[0] = bf(a.dXout);
    o.P[0] = parts + 3 * msz;
    o.M = HD; o.K = rows; o.Nb = d.dx; o.lda = HD; o.ldb = d.dx; o.nseg = 1; o.kchunk = kchunk;
    k_node_gemm<true, false><<<dim3(d.dx / GBN, HD / GBM, splits), GTHR, 0, st>>>(o);
    return cudaGetLastError();
}

}  // namespace fast
}  // namespace eaga
