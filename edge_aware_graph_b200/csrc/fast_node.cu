// Node-side GEMMs of the layer on the tensor cores (bf16 in, fp32 accumulate):
//   QKV:      [Q|K|V] = X [Wq|Wk|Wv] + b, rows of masked nodes written as zero
//   out-proj: X' = X + M (O Wo + bo)
// 64x64 output tile per CTA, 4 warps of 32x32, K in steps of 32 through a
// two-stage cp.async pipeline, 16-byte swizzled shared-memory rows.
#include "common.cuh"
#include "fast.h"
#include "sm100.cuh"

namespace eaga {
namespace fast {

using namespace sm100;

constexpr int GBM = 64, GBN = 64, GBK = 32, GTHR = 128;

struct GemmParams {
    const __nv_bfloat16 *A;          // [M, K]
    const __nv_bfloat16 *B[3];       // [K, Nb] each; output column tile n0 uses B[n0 / Nb]
    const __nv_bfloat16 *bias[3];    // [Nb]
    __nv_bfloat16 *C[3];             // [M, Nb]
    const __nv_bfloat16 *R;          // residual [M, Nb] (out-proj) or null
    const uint8_t *mask;             // [M]
    int M, K, Nb;
    int mode;                        // 0: QKV, 1: out-proj with residual
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred) {
    const int sz = pred ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// A tile [64 rows][32 k] (64 B rows): chunk c of row r at r*64 + ((c ^ ((r>>1)&3)) << 4)
__device__ __forceinline__ uint32_t a_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }
// B tile [32 k][64 n] (128 B rows): chunk c of row k at k*128 + ((c ^ (k&7)) << 4)
__device__ __forceinline__ uint32_t b_off(int k, int c) { return k * 128 + ((c ^ (k & 7)) << 4); }

__global__ void __launch_bounds__(GTHR) k_node_gemm(GemmParams p) {
    __shared__ __align__(128) uint8_t sA[2][GBM * GBK * 2];
    __shared__ __align__(128) uint8_t sB[2][GBK * GBN * 2];
    const int tid = threadIdx.x, w = tid >> 5, t = tid & 31;
    const int n0g = blockIdx.x * GBN, m0 = blockIdx.y * GBM;
    const int which = n0g / p.Nb, n0 = n0g % p.Nb;
    const __nv_bfloat16 *Bm = p.B[which];
    const int wm = (w >> 1) * 32, wn = (w & 1) * 32;
    float acc[2][4][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

    auto load = [&](int stage, int k0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int idx = tid + q * GTHR;      // 256 chunks of A: row idx/4, chunk idx%4
            const int r = idx >> 2, c = idx & 3;
            const int gm = m0 + r;
            cp_async16(smem_u32(sA[stage]) + a_off(r, c), p.A + (size_t)min(gm, p.M - 1) * p.K + k0 + c * 8, gm < p.M);
            const int kr = idx >> 3, cb = idx & 7;   // 256 chunks of B: row idx/8, chunk idx%8
            cp_async16(smem_u32(sB[stage]) + b_off(kr, cb), Bm + (size_t)(k0 + kr) * p.Nb + n0 + cb * 8, true);
        }
        cp_async_commit();
    };

    const int nk = p.K / GBK;
    load(0, 0);
    for (int kt = 0; kt < nk; ++kt) {
        if (kt + 1 < nk) {
            load((kt + 1) & 1, (kt + 1) * GBK);
            cp_async_wait1();
        } else {
            cp_async_wait0();
        }
        __syncthreads();
        const uint32_t a_s = smem_u32(sA[kt & 1]), b_s = smem_u32(sB[kt & 1]);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t af[2][4], bfr[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                // matrices: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
                const int r = wm + mt * 16 + (t & 7) + ((t >> 3) & 1) * 8;
                const int c = ks * 2 + (t >> 4);
                ldsm_x4(a_s + a_off(r, c), af[mt]);
            }
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                // matrices: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
                const int kr = ks * 16 + (t & 7) + ((t >> 3) & 1) * 8;
                const int c = (wn + np * 16) / 8 + (t >> 4);
                ldsm_x4_t(b_s + b_off(kr, c), bfr[np]);
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
    const __nv_bfloat16 *bias = p.bias[which];
    __nv_bfloat16 *C = p.C[which];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int row = m0 + wm + mt * 16 + (t >> 2) + hh * 8;
                const int col = n0 + wn + nt * 8 + (t & 3) * 2;
                if (row >= p.M) continue;
                const float2 bb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(bias + col));
                const bool mk = p.mask[row] != 0;
                float v0 = acc[mt][nt][hh * 2] + bb.x, v1 = acc[mt][nt][hh * 2 + 1] + bb.y;
                __nv_bfloat162 out;
                if (p.mode == 0) {
                    out = mk ? __floats2bfloat162_rn(v0, v1) : __floats2bfloat162_rn(0.f, 0.f);
                } else {
                    const __nv_bfloat162 rr = *reinterpret_cast<const __nv_bfloat162 *>(p.R + (size_t)row * p.Nb + col);
                    if (mk) {
                        const float2 x = __bfloat1622float2(rr);
                        out = __floats2bfloat162_rn(x.x + v0, x.y + v1);
                    } else {
                        out = rr;
                    }
                }
                *reinterpret_cast<__nv_bfloat162 *>(C + (size_t)row * p.Nb + col) = out;
            }
}

cudaError_t launch_qkv(const eaga_dims &d, const FwdArgs &a, cudaStream_t st) {
    GemmParams p;
    p.A = static_cast<const __nv_bfloat16 *>(a.X);
    for (int q = 0; q < 3; ++q) {
        p.B[q] = static_cast<const __nv_bfloat16 *>(a.w[2 * q]);
        p.bias[q] = static_cast<const __nv_bfloat16 *>(a.w[2 * q + 1]);
    }
    p.C[0] = static_cast<__nv_bfloat16 *>(a.Q);
    p.C[1] = static_cast<__nv_bfloat16 *>(a.K);
    p.C[2] = static_cast<__nv_bfloat16 *>(a.V);
    p.R = nullptr;
    p.mask = a.M;
    p.M = d.B * d.n;
    p.K = d.dx;
    p.Nb = d.H * d.dh;
    p.mode = 0;
    dim3 grid(3 * p.Nb / GBN, (p.M + GBM - 1) / GBM);
    k_node_gemm<<<grid, GTHR, 0, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_out_proj(const eaga_dims &d, const FwdArgs &a, cudaStream_t st) {
    GemmParams p;
    p.A = static_cast<const __nv_bfloat16 *>(a.O);
    p.B[0] = p.B[1] = p.B[2] = static_cast<const __nv_bfloat16 *>(a.w[10]);
    p.bias[0] = p.bias[1] = p.bias[2] = static_cast<const __nv_bfloat16 *>(a.w[11]);
    p.C[0] = p.C[1] = p.C[2] = static_cast<__nv_bfloat16 *>(a.Xout);
    p.R = static_cast<const __nv_bfloat16 *>(a.X);
    p.mask = a.M;
    p.M = d.B * d.n;
    p.K = d.H * d.dh;
    p.Nb = d.dx;
    p.mode = 1;
    dim3 grid(p.Nb / GBN, (p.M + GBM - 1) / GBM);
    k_node_gemm<<<grid, GTHR, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace fast
}  // namespace eaga
