// Node and global parts of the graph-transformer block around the layer, the
// reductions of the block's weight gradients, and the block's launch sequence
// on the specialised sm_100a path (the edge part is in fast_block_edge.cu).
//
// The pages place the layer inside DeFoG's graph-transformer backbone, which
// updates node, edge and global features jointly (AI-summary page, method
// paragraph; paper index page, abstract), and print none of the block's
// equations.  The block computed here is the plain post-norm reading:
//   pX_b = sum_i M_bi X'_bi / max(cnt_b, 1),  pE_b = sum_ij valid E'_bij / max(cnt_b^2, 1)
//   y1_b = y_b + pX_b Wyx + pE_b Wye + by
//   for Z in (X', E', y1):  Za = LN(Z; g1, s1),  Zz = Za + relu(Za W1 + b1) W2 + b2,
//                           Zo = LN(Zz; g2, s2)
//   Xout = M Xo,  Eout = valid Eo,  yout = yo
// Node FFN products run on the tcgen05 GEMM (fast_gemm_tc.cu) with fused
// bias / relu / residual epilogues; LayerNorms and the global sub-block (a few
// hundred values per graph) run on CUDA cores.  Every reduction over rows or
// graphs runs in a fixed order.
#include "fast.h"
#include "fast_common.cuh"
#include "fast_block.h"

namespace eaga {
namespace fast {

cudaError_t tc_gemm(int mode, int M, int N, int K, int nseg, const void *const A[3], const void *const B[3],
                    const void *const bias[3], void *const C[3], int Nb, const void *R, const uint8_t *mask,
                    int *status, cudaStream_t st, bool b_mn);
cudaError_t tc_wgrad(int M, int Nb, int nout, int K, int splits, const void *A, const void *const B[3],
                     float *const P[3], int *status, cudaStream_t st);

namespace blk {

constexpr float LN_EPS = 1e-5f;
constexpr int LN_WARPS = 8;

__device__ __forceinline__ float bf(const __nv_bfloat16 *p, size_t i) { return __bfloat162float(p[i]); }

// ------------------------------------------------------------------ node LayerNorms

// out = LN(Z; g, s) over D = 64 NQ features of each row (one warp a row; lane
// l holds features 64 q + 2 l, 64 q + 2 l + 1), zero on rows with mask 0 when
// a mask is given.
template <int NQ>
__global__ void __launch_bounds__(32 * LN_WARPS) k_ln_fwd(const __nv_bfloat16 *Z, const __nv_bfloat16 *g,
                                                          const __nv_bfloat16 *s, const uint8_t *mask,
                                                          __nv_bfloat16 *out, int R) {
    constexpr int D = 64 * NQ;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * LN_WARPS + (threadIdx.x >> 5);
    if (row >= R) return;
    float v[2 * NQ];
    const __nv_bfloat162 *z2 = reinterpret_cast<const __nv_bfloat162 *>(Z + (size_t)row * D);
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const float2 f = __bfloat1622float2(z2[32 * q + lane]);
        v[2 * q] = f.x;
        v[2 * q + 1] = f.y;
        sum += f.x + f.y;
    }
    const float mean = warp_sum(sum) * (1.f / D);
    float sq = 0.f;
#pragma unroll
    for (int u = 0; u < 2 * NQ; ++u) {
        v[u] -= mean;
        sq = fmaf(v[u], v[u], sq);
    }
    const float rs = rsqrtf(warp_sum(sq) * (1.f / D) + LN_EPS);
    const bool keep = mask == nullptr || mask[row] != 0;
    __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(out + (size_t)row * D);
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int c = 64 * q + 2 * lane;
        const float a = keep ? fmaf(v[2 * q] * rs, bf(g, c), bf(s, c)) : 0.f;
        const float b = keep ? fmaf(v[2 * q + 1] * rs, bf(g, c + 1), bf(s, c + 1)) : 0.f;
        o2[32 * q + lane] = __floats2bfloat162_rn(a, b);
    }
}

// Chain rule of LN for each row: given the LN input Z and the output gradient
// dOut (zero on rows with mask 0 when a mask is given),
//   dZ = r (dOut g - mean(dOut g) - x mean(dOut g x)) [+ M_row add[b]]
// and the CTA's partial sums of dg = sum dOut x and ds = sum dOut into
// part[blockIdx][2 D] (features 0..D-1: dg, D..2D-1: ds).  `add` [B, D] fp32 is
// added on rows with addmask 1 (rows of graph b = row / n).
template <int NQ>
__global__ void __launch_bounds__(32 * LN_WARPS) k_ln_bwd(const __nv_bfloat16 *Z, const __nv_bfloat16 *dOut,
                                                          const __nv_bfloat16 *g, const uint8_t *mask,
                                                          const float *add, const uint8_t *addmask, int n,
                                                          __nv_bfloat16 *dZ, float *part, int R) {
    constexpr int D = 64 * NQ;
    __shared__ float red[LN_WARPS][2 * D];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float ag[2 * NQ], as[2 * NQ];
#pragma unroll
    for (int u = 0; u < 2 * NQ; ++u) ag[u] = as[u] = 0.f;
    for (int row = blockIdx.x * LN_WARPS + w; row < R; row += gridDim.x * LN_WARPS) {
        float x[2 * NQ], d[2 * NQ];
        const __nv_bfloat162 *z2 = reinterpret_cast<const __nv_bfloat162 *>(Z + (size_t)row * D);
        const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(dOut + (size_t)row * D);
        const bool keep = mask == nullptr || mask[row] != 0;
        float sum = 0.f;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            const float2 f = __bfloat1622float2(z2[32 * q + lane]);
            const float2 e = __bfloat1622float2(d2[32 * q + lane]);
            x[2 * q] = f.x;
            x[2 * q + 1] = f.y;
            d[2 * q] = keep ? e.x : 0.f;
            d[2 * q + 1] = keep ? e.y : 0.f;
            sum += f.x + f.y;
        }
        const float mean = warp_sum(sum) * (1.f / D);
        float sq = 0.f;
#pragma unroll
        for (int u = 0; u < 2 * NQ; ++u) {
            x[u] -= mean;
            sq = fmaf(x[u], x[u], sq);
        }
        const float rs = rsqrtf(warp_sum(sq) * (1.f / D) + LN_EPS);
        float m1 = 0.f, m2 = 0.f;
#pragma unroll
        for (int q = 0; q < NQ; ++q)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int u = 2 * q + e, c = 64 * q + 2 * lane + e;
                x[u] *= rs;
                ag[u] = fmaf(d[u], x[u], ag[u]);
                as[u] += d[u];
                d[u] *= bf(g, c);
                m1 += d[u];
                m2 = fmaf(d[u], x[u], m2);
            }
        m1 = warp_sum(m1) * (1.f / D);
        m2 = warp_sum(m2) * (1.f / D);
        const bool addrow = add != nullptr && addmask[row] != 0;
        const float *ad = add ? add + (size_t)(row / n) * D : nullptr;
        __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(dZ + (size_t)row * D);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            const int c = 64 * q + 2 * lane;
            float a = rs * (d[2 * q] - m1 - x[2 * q] * m2);
            float b = rs * (d[2 * q + 1] - m1 - x[2 * q + 1] * m2);
            if (addrow) {
                a += ad[c];
                b += ad[c + 1];
            }
            o2[32 * q + lane] = __floats2bfloat162_rn(a, b);
        }
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = 64 * q + 2 * lane + e;
            red[w][c] = ag[2 * q + e];
            red[w][D + c] = as[2 * q + e];
        }
    __syncthreads();
    for (int c = threadIdx.x; c < 2 * D; c += blockDim.x) {
        float t = 0.f;
#pragma unroll
        for (int k = 0; k < LN_WARPS; ++k) t += red[k][c];
        part[(size_t)blockIdx.x * 2 * D + c] = t;
    }
}

// Column sums of A [R, C] bf16: part[blockIdx][C] over the CTA's range of rows.
__global__ void __launch_bounds__(256) k_colsum(const __nv_bfloat16 *A, float *part, int R, int C, int rows_per) {
    const int r0 = blockIdx.x * rows_per, r1 = min(R, r0 + rows_per);
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        float t = 0.f;
        for (int r = r0; r < r1; ++r) t += __bfloat162float(A[(size_t)r * C + c]);
        part[(size_t)blockIdx.x * C + c] = t;
    }
}

// ------------------------------------------------------------------ global sub-block

// Block-wide sum over the CTA (blockDim a multiple of 32, at most 1024).
__device__ __forceinline__ float block_sum(float v, float *scratch) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) scratch[w] = v;
    __syncthreads();
    float t = 0.f;
    for (int k = 0; k < nw; ++k) t += scratch[k];
    return t;
}

// LN over dy values in shared memory: xh <- normalised z, returns 1/sqrt(var + eps).
__device__ __forceinline__ float block_ln(const float *z, float *xh, int dy, float *scratch) {
    float s = 0.f;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) s += z[o];
    const float mean = block_sum(s, scratch) / dy;
    float q = 0.f;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        const float c = z[o] - mean;
        q = fmaf(c, c, q);
    }
    const float rs = rsqrtf(block_sum(q, scratch) / dy + LN_EPS);
    for (int o = threadIdx.x; o < dy; o += blockDim.x) xh[o] = (z[o] - mean) * rs;
    __syncthreads();
    return rs;
}

// out[o] = init(o) + sum_k in[k] w(k, o) for o < nout <= blockDim.x, by every
// thread of the CTA: the k range split into blockDim.x / nout parts whose
// partial sums (in `part`, blockDim.x floats) are added in part order.
template <class W, class Init>
__device__ __forceinline__ void block_matvec(const float *in, int K, int nout, W w, Init init, float *out,
                                             float *part) {
    const int P = blockDim.x / nout;
    const int t = threadIdx.x, o = t % nout, pi = t / nout;
    if (pi < P) {
        const int k0 = pi * K / P, k1 = (pi + 1) * K / P;
        float a = 0.f;
#pragma unroll 8
        for (int k = k0; k < k1; ++k) a = fmaf(in[k], w(k, o), a);
        part[pi * nout + o] = a;
    }
    __syncthreads();
    for (int q = t; q < nout; q += blockDim.x) {
        float a = init(q);
        for (int pp = 0; pp < P; ++pp) a += part[pp * nout + q];
        out[q] = a;
    }
    __syncthreads();
}

// sum_k v[k] row[k] over a bf16 row of len values (len a multiple of 8, the
// row 16-byte aligned), read eight values a load, in k order.
__device__ __forceinline__ float row_dot(const float *v, const __nv_bfloat16 *row, int len) {
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
    float a = 0.f;
#pragma unroll 4
    for (int c = 0; c < len / 8; ++c) {
        const uint4 u = r4[c];
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float2 f = __bfloat1622float2(h2[j]);
            a = fmaf(v[8 * c + 2 * j], f.x, a);
            a = fmaf(v[8 * c + 2 * j + 1], f.y, a);
        }
    }
    return a;
}

// Recomputes the global sub-block of graph b from y1 into shared memory:
// x1 (LN1 normalised), ya, hpre, h, x2 (LN2 normalised); returns r1, r2.
__device__ void y_sub_forward(const YParams &p, const float *y1, float *x1, float *ya, float *hpre, float *h,
                              float *yz, float *x2, float *scratch, float *part, float &r1, float &r2) {
    const int dy = p.dy, fy = 2 * p.dy;
    r1 = block_ln(y1, x1, dy, scratch);
    for (int o = threadIdx.x; o < dy; o += blockDim.x) ya[o] = fmaf(x1[o], bf(p.g1, o), bf(p.s1, o));
    __syncthreads();
    block_matvec(ya, dy, fy, [&](int k, int f) { return bf(p.W1, (size_t)k * fy + f); },
                 [&](int f) { return bf(p.b1, f); }, hpre, part);
    for (int f = threadIdx.x; f < fy; f += blockDim.x) h[f] = fmaxf(hpre[f], 0.f);
    __syncthreads();
    block_matvec(h, fy, dy, [&](int k, int o) { return bf(p.W2, (size_t)k * dy + o); },
                 [&](int o) { return ya[o] + bf(p.b2, o); }, yz, part);
    r2 = block_ln(yz, x2, dy, scratch);
}

// Sums of X' over the real nodes of each graph: CTA (b, 64-feature block,
// 64-row block), 8 warps of 8 rows, lane l features 2l, 2l+1; the CTA's sums
// are added to poolx [B, dx].
__global__ void __launch_bounds__(256) k_pool_x(const __nv_bfloat16 *X, const uint8_t *M, float *poolx, int n, int dx) {
    __shared__ float red[8][64];
    const int b = blockIdx.x, c0 = blockIdx.y * 64, i0 = blockIdx.z * 64;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    float a0 = 0.f, a1 = 0.f;
    for (int i = i0 + w; i < min(n, i0 + 64); i += 8) {
        if (!M[(size_t)b * n + i]) continue;
        const float2 f = __bfloat1622float2(
            reinterpret_cast<const __nv_bfloat162 *>(X + ((size_t)b * n + i) * dx + c0)[lane]);
        a0 += f.x;
        a1 += f.y;
    }
    red[w][2 * lane] = a0;
    red[w][2 * lane + 1] = a1;
    __syncthreads();
    if (threadIdx.x < 64) {
        float t = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) t += red[k][threadIdx.x];
        atomicAdd(poolx + (size_t)b * dx + c0 + threadIdx.x, t);
    }
}

// One CTA per graph: pX, pE (means over real nodes / valid pairs), y1, the
// global sub-block, yout.  Saves y1, pX and pE for the backward.
__global__ void __launch_bounds__(256) k_y_fwd(YParams p) {
    extern __shared__ float sm[];
    const int b = blockIdx.x, dx = p.dx, dy = p.dy, fy = 2 * p.dy, n = p.n;
    float *pX = sm, *pE = pX + dx, *y1 = pE + 64, *x1 = y1 + dy, *ya = x1 + dy, *hpre = ya + dy, *h = hpre + fy,
          *yz = h + fy, *x2 = yz + dy, *part = x2 + dy, *y1b = part + 256, *scratch = y1b + dy;
    float c = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) c += p.M[(size_t)b * n + i] ? 1.f : 0.f;
    const float cnt = block_sum(c, scratch);
    const float cx = fmaxf(cnt, 1.f), ce = fmaxf(cnt * cnt, 1.f);
    for (int k = threadIdx.x; k < dx; k += blockDim.x) {
        pX[k] = p.poolx[(size_t)b * dx + k] / cx;
        p.pX[(size_t)b * dx + k] = pX[k];
    }
    for (int k = threadIdx.x; k < 64; k += blockDim.x) {
        pE[k] = p.pool[(size_t)b * 64 + k] / ce;
        p.pE[(size_t)b * 64 + k] = pE[k];
    }
    __syncthreads();
    // y1 = y + pX Wyx + pE Wye + by
    block_matvec(pX, dx, dy, [&](int k, int o) { return bf(p.Wyx, (size_t)k * dy + o); },
                 [&](int o) { return bf(p.y, (size_t)b * dy + o) + bf(p.by, o); }, y1b, part);
    block_matvec(pE, 64, dy, [&](int k, int o) { return bf(p.Wye, (size_t)k * dy + o); },
                 [&](int o) { return y1b[o]; }, y1, part);
    for (int o = threadIdx.x; o < dy; o += blockDim.x) p.y1[(size_t)b * dy + o] = y1[o];
    __syncthreads();
    float r1, r2;
    y_sub_forward(p, y1, x1, ya, hpre, h, yz, x2, scratch, part, r1, r2);
    for (int o = threadIdx.x; o < dy; o += blockDim.x)
        p.yout[(size_t)b * dy + o] = __float2bfloat16_rn(fmaf(x2[o], bf(p.g2, o), bf(p.s2, o)));
}

// One CTA per graph: the chain rule of the global sub-block and of y1 from
// the saved y1.  Writes dy1, dpX = dy1 Wyx^T / cnt, dpE = dy1 Wye^T / cnt^2
// and the per-graph vectors k_y_wgrad sums over graphs.
__global__ void __launch_bounds__(256) k_y_bwd(YParams p) {
    extern __shared__ float sm[];
    const int b = blockIdx.x, dx = p.dx, dy = p.dy, fy = 2 * p.dy, n = p.n;
    float *y1 = sm, *x1 = y1 + dy, *ya = x1 + dy, *hpre = ya + dy, *h = hpre + fy, *yz = h + fy, *x2 = yz + dy,
          *dyz = x2 + dy, *dh = dyz + dy, *dya = dh + fy, *dy1 = dya + dy, *part = dy1 + dy, *scratch = part + 256;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) y1[o] = p.y1[(size_t)b * dy + o];
    __syncthreads();
    float r1, r2;
    y_sub_forward(p, y1, x1, ya, hpre, h, yz, x2, scratch, part, r1, r2);
    // dyz = LN2^T(dyout)
    float m1 = 0.f, m2 = 0.f;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        const float dg = bf(p.dyout, (size_t)b * dy + o) * bf(p.g2, o);
        m1 += dg;
        m2 = fmaf(dg, x2[o], m2);
    }
    m1 = block_sum(m1, scratch) / dy;
    m2 = block_sum(m2, scratch) / dy;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        const float dg = bf(p.dyout, (size_t)b * dy + o) * bf(p.g2, o);
        dyz[o] = r2 * (dg - m1 - x2[o] * m2);
    }
    __syncthreads();
    // dh = dyz W2^T [hpre > 0]: row f of W2 per output
    for (int f = threadIdx.x; f < fy; f += blockDim.x)
        dh[f] = hpre[f] > 0.f ? row_dot(dyz, p.W2 + (size_t)f * dy, dy) : 0.f;
    __syncthreads();
    // dya = dyz + dh W1^T: row o of W1 per output
    for (int o = threadIdx.x; o < dy; o += blockDim.x) dya[o] = dyz[o] + row_dot(dh, p.W1 + (size_t)o * fy, fy);
    __syncthreads();
    m1 = 0.f;
    m2 = 0.f;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        const float dg = dya[o] * bf(p.g1, o);
        m1 += dg;
        m2 = fmaf(dg, x1[o], m2);
    }
    m1 = block_sum(m1, scratch) / dy;
    m2 = block_sum(m2, scratch) / dy;
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        const float v = r1 * (dya[o] * bf(p.g1, o) - m1 - x1[o] * m2);
        dy1[o] = v;
        p.dy1[(size_t)b * dy + o] = v;
    }
    __syncthreads();
    float c = 0.f;
    for (int i = threadIdx.x; i < n; i += blockDim.x) c += p.M[(size_t)b * n + i] ? 1.f : 0.f;
    const float cnt = block_sum(c, scratch);
    const float cx = fmaxf(cnt, 1.f), ce = fmaxf(cnt * cnt, 1.f);
    for (int k = threadIdx.x; k < dx; k += blockDim.x) p.dpX[(size_t)b * dx + k] = row_dot(dy1, p.Wyx + (size_t)k * dy, dy) / cx;
    for (int k = threadIdx.x; k < 64; k += blockDim.x) p.dpE[(size_t)b * 64 + k] = row_dot(dy1, p.Wye + (size_t)k * dy, dy) / ce;
    // per-graph vectors: h, dh [fy]; ya, dyz, x1, dya, x2 [dy]
    float *v = p.yv + (size_t)b * YV_PER_DY * dy;
    for (int f = threadIdx.x; f < fy; f += blockDim.x) {
        v[f] = h[f];
        v[fy + f] = dh[f];
    }
    for (int o = threadIdx.x; o < dy; o += blockDim.x) {
        v[2 * fy + o] = ya[o];
        v[2 * fy + dy + o] = dyz[o];
        v[2 * fy + 2 * dy + o] = x1[o];
        v[2 * fy + 3 * dy + o] = dya[o];
        v[2 * fy + 4 * dy + o] = x2[o];
    }
}

// The global sub-block's weight gradients and those of the pooling maps: one
// thread per entry, summed over the graphs in order (each region of entries a
// plain loop over the graphs, so the loads of consecutive graphs overlap).
__global__ void __launch_bounds__(256) k_y_wgrad(YParams p, YGrads gr) {
    const int dy = p.dy, fy = 2 * p.dy, dx = p.dx, B = p.B;
    const int nW1 = dy * fy, nW2 = fy * dy, nyx = dx * dy, nye = 64 * dy;
    const int total = nW1 + nW2 + nyx + nye + fy + 6 * dy;
    const size_t vs = (size_t)YV_PER_DY * dy;                 // per-graph vector stride
    const float *v0 = p.yv;
    // offsets inside a graph's vectors: h, dh [fy]; ya, dyz, x1, dya, x2 [dy]
    const int oh = 0, odh = fy, oya = 2 * fy, odyz = 2 * fy + dy, ox1 = 2 * fy + 2 * dy, odya = 2 * fy + 3 * dy,
              ox2 = 2 * fy + 4 * dy;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < total; e += gridDim.x * blockDim.x) {
        float a = 0.f;
        int q = e;
        if (q < nW1) {
            const int o = q / fy, f = q % fy;
#pragma unroll 4
            for (int b = 0; b < B; ++b) a = fmaf(v0[b * vs + oya + o], v0[b * vs + odh + f], a);
            gr.W1[q] = a;
            continue;
        }
        q -= nW1;
        if (q < nW2) {
            const int f = q / dy, o = q % dy;
#pragma unroll 4
            for (int b = 0; b < B; ++b) a = fmaf(v0[b * vs + oh + f], v0[b * vs + odyz + o], a);
            gr.W2[q] = a;
            continue;
        }
        q -= nW2;
        if (q < nyx) {
            const int k = q / dy, o = q % dy;
#pragma unroll 4
            for (int b = 0; b < B; ++b) a = fmaf(p.pX[(size_t)b * dx + k], p.dy1[(size_t)b * dy + o], a);
            gr.Wyx[q] = a;
            continue;
        }
        q -= nyx;
        if (q < nye) {
            const int k = q / dy, o = q % dy;
#pragma unroll 4
            for (int b = 0; b < B; ++b) a = fmaf(p.pE[(size_t)b * 64 + k], p.dy1[(size_t)b * dy + o], a);
            gr.Wye[q] = a;
            continue;
        }
        q -= nye;
        if (q < fy) {
#pragma unroll 4
            for (int b = 0; b < B; ++b) a += v0[b * vs + odh + q];
            gr.b1[q] = a;
            continue;
        }
        q -= fy;
        const int k = q / dy, o = q % dy;
#pragma unroll 4
        for (int b = 0; b < B; ++b) {
            const float *v = v0 + b * vs;
            const float up = bf(p.dyout, (size_t)b * dy + o);
            a += k == 0 ? v[odyz + o]                         // b2
               : k == 1 ? up * v[ox2 + o]                     // ln2 g
               : k == 2 ? up                                  // ln2 s
               : k == 3 ? v[odya + o] * v[ox1 + o]            // ln1 g
               : k == 4 ? v[odya + o]                         // ln1 s
                        : p.dy1[(size_t)b * dy + o];          // by
        }
        float *dst = k == 0 ? gr.b2 : k == 1 ? gr.g2 : k == 2 ? gr.s2 : k == 3 ? gr.g1 : k == 4 ? gr.s1 : gr.by;
        dst[o] = a;
    }
}

// ------------------------------------------------------------------ reductions

// dst = sum over parts of src (part k at src + k * stride); with trows > 0 the
// segment is the transpose of a [trows][count / trows] source.  The lanes of a
// warp take consecutive source entries, so every load is a coalesced 128-byte
// row of one part.  A segment of many parts (more than 16) gives 32 entries to
// a CTA whose eight warps split the parts; a segment of few parts gives 256
// entries to a CTA, each warp adding all parts of its 32.  Every entry is
// summed in the same order on every call.
__global__ void __launch_bounds__(256) k_sum_parts(SumSegs segs) {
    __shared__ float red[8][32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int item = blockIdx.x;
    for (int s = 0; s < segs.n; ++s) {
        const SumSeg &g = segs.seg[s];
        // a CTA: 32 consecutive source entries of a wide segment (more than 16
        // parts; warp w adds the parts k = w mod 8, then the eight sums are added
        // in warp order), or 256 of a narrow one (a warp 32, over every part)
        const bool wide = g.nparts > 16;
        const int per = wide ? 32 : 256;
        const int tiles = (g.count + per - 1) / per;
        if (item >= tiles) {
            item -= tiles;
            continue;
        }
        const int src = item * per + (wide ? 0 : 32 * w) + lane;   // consecutive lanes: consecutive addresses
        const bool in = src < g.count;
        float t = 0.f;
        if (wide) {
            if (in) {
#pragma unroll 4
                for (int k = w; k < g.nparts; k += 8) t += g.src[(size_t)k * g.stride + src];
            }
            red[w][lane] = t;
            __syncthreads();
            if (w != 0) return;
            t = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) t += red[k][lane];
        } else if (in) {
#pragma unroll 4
            for (int k = 0; k < g.nparts; ++k) t += g.src[(size_t)k * g.stride + src];
        }
        if (!in) return;
        int e = src;   // the destination entry: source [trows][cols] -> destination [cols][trows]
        if (g.trows > 0) {
            const int cols = g.count / g.trows;
            e = (src % cols) * g.trows + src / cols;
        }
        g.dst[e] = t;
        return;
    }
}

// dy += dy1 (bf16 storage, fp32 sum).
__global__ void k_add_dy(__nv_bfloat16 *dy, const float *dy1, int count) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < count) dy[e] = __float2bfloat16_rn(__bfloat162float(dy[e]) + dy1[e]);
}

// ------------------------------------------------------------------ host

namespace {
template <int NQ>
cudaError_t ln_fwd_nq(const void *Z, const void *g, const void *s, const uint8_t *mask, void *out, int R,
                      cudaStream_t st) {
    k_ln_fwd<NQ><<<(R + LN_WARPS - 1) / LN_WARPS, 32 * LN_WARPS, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(Z), static_cast<const __nv_bfloat16 *>(g),
        static_cast<const __nv_bfloat16 *>(s), mask, static_cast<__nv_bfloat16 *>(out), R);
    return cudaGetLastError();
}
cudaError_t ln_fwd(int D, const void *Z, const void *g, const void *s, const uint8_t *mask, void *out, int R,
                   cudaStream_t st) {
    switch (D) {
        case 256: return ln_fwd_nq<4>(Z, g, s, mask, out, R, st);
        case 512: return ln_fwd_nq<8>(Z, g, s, mask, out, R, st);
        case 1024: return ln_fwd_nq<16>(Z, g, s, mask, out, R, st);
        default: return cudaErrorInvalidValue;
    }
}
template <int NQ>
cudaError_t ln_bwd_nq(const void *Z, const void *dOut, const void *g, const uint8_t *mask, const float *add,
                      const uint8_t *addmask, int n, void *dZ, float *part, int R, int grid, cudaStream_t st) {
    k_ln_bwd<NQ><<<grid, 32 * LN_WARPS, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(Z), static_cast<const __nv_bfloat16 *>(dOut),
        static_cast<const __nv_bfloat16 *>(g), mask, add, addmask, n, static_cast<__nv_bfloat16 *>(dZ), part, R);
    return cudaGetLastError();
}
cudaError_t ln_bwd(int D, const void *Z, const void *dOut, const void *g, const uint8_t *mask, const float *add,
                   const uint8_t *addmask, int n, void *dZ, float *part, int R, int grid, cudaStream_t st) {
    switch (D) {
        case 256: return ln_bwd_nq<4>(Z, dOut, g, mask, add, addmask, n, dZ, part, R, grid, st);
        case 512: return ln_bwd_nq<8>(Z, dOut, g, mask, add, addmask, n, dZ, part, R, grid, st);
        default: return cudaErrorInvalidValue;     // 2 D floats of shared memory per warp
    }
}
#define BLK_TRY(x)                                   \
    do {                                             \
        cudaError_t e_ = (x);                        \
        if (e_ != cudaSuccess) return e_;            \
    } while (0)
}  // namespace

bool block_supports(int dx, int de, int dy) {
    return de == 64 && (dx == 256 || dx == 512) && dy % 32 == 0 && dy >= 32 && dy <= 128;
}

BlockSaved block_saved_layout(int B, int n, int dx, int dy, size_t base) {
    BlockSaved L;
    const size_t R = (size_t)B * n;
    size_t off = base;
    L.Xa = off; off = align256(off + R * dx * 2);
    L.Hx = off; off = align256(off + R * 2 * dx * 2);
    L.Xz = off; off = align256(off + R * dx * 2);
    L.y1 = off; off = align256(off + (size_t)B * dy * 4);
    L.pX = off; off = align256(off + (size_t)B * dx * 4);
    L.pE = off; off = align256(off + (size_t)B * 64 * 4);
    L.total = off;
    return L;
}

BlockWs block_ws_layout(int B, int n, int dx, int dy, size_t base, int for_backward) {
    BlockWs L = {};
    const size_t R = (size_t)B * n;
    size_t off = base;
    L.pool = off; off = align256(off + (size_t)B * (64 + dx) * 4);    // E' sums [B][64], X' sums [B][dx]
    if (for_backward) {
        L.dXmid = off; off = align256(off + R * dx * 2);
        L.dXz = off; off = align256(off + R * dx * 2);
        L.dHx = off; off = align256(off + R * 2 * dx * 2);
        L.dXa = off; off = align256(off + R * dx * 2);
        L.dpX = off; off = align256(off + (size_t)B * dx * 4);
        L.dpE = off; off = align256(off + (size_t)B * 64 * 4);
        L.dy1 = off; off = align256(off + (size_t)B * dy * 4);
        L.yv = off; off = align256(off + (size_t)B * YV_PER_DY * dy * 4);
        L.ln_grid = 148;
        L.ln2 = off; off = align256(off + (size_t)L.ln_grid * 2 * dx * 4);
        L.ln1 = off; off = align256(off + (size_t)L.ln_grid * 2 * dx * 4);
        L.cs_rows = 16;
        L.cs_grid = (int)((R + L.cs_rows - 1) / L.cs_rows);
        L.cs1 = off; off = align256(off + (size_t)L.cs_grid * 2 * dx * 4);
        L.cs2 = off; off = align256(off + (size_t)L.cs_grid * dx * 4);
        int sp = (int)(R / 512);
        L.wsplits = sp < 1 ? 1 : (sp > 32 ? 32 : sp);
        L.wg1 = off; off = align256(off + (size_t)L.wsplits * dx * 2 * dx * 4);
        L.wg2 = off; off = align256(off + (size_t)L.wsplits * 2 * dx * dx * 4);
        L.ectas = edge_backward_ctas(B, n);
        L.eparts = off; off = align256(off + (size_t)L.ectas * EB_PART * 4);
        L.ewparts = off; off = align256(off + (size_t)L.ectas * 2 * 128 * 64 * 4);
    }
    L.total = off;
    return L;
}

int block_kernel_launches(int for_backward) {
    // forward: pool memset, edge, LN1, FFN1, FFN2, LN2, X' pooling, y
    // backward: y bwd, y wgrad, edge, LN2 bwd, DRELU, DX, LN1 bwd, 2 wgrad, 2 colsum, sum parts, add dy
    return for_backward ? 13 : 8;
}

YParams y_params(int B, int n, int dx, int dy, const void *const *wb, const uint8_t *M) {
    YParams p = {};
    p.B = B;
    p.n = n;
    p.dx = dx;
    p.dy = dy;
    p.M = M;
    auto w = [&](int i) { return static_cast<const __nv_bfloat16 *>(wb[i]); };
    p.g1 = w(BW_Y + 0);
    p.s1 = w(BW_Y + 1);
    p.W1 = w(BW_Y + 2);
    p.b1 = w(BW_Y + 3);
    p.W2 = w(BW_Y + 4);
    p.b2 = w(BW_Y + 5);
    p.g2 = w(BW_Y + 6);
    p.s2 = w(BW_Y + 7);
    p.Wyx = w(BW_YX);
    p.Wye = w(BW_YE);
    p.by = w(BW_BY);
    return p;
}

cudaError_t tail_forward(const TailFwd &a, char *ws, const BlockWs &W, char *saved, const BlockSaved &S,
                         cudaStream_t st) {
    return with_side_streams([&](const cudaStream_t *ss, const cudaEvent_t *ev) -> cudaError_t {
        cudaStream_t side = ss[2];
        cudaEvent_t e0 = ev[0], e1 = ev[1];
        const int R = a.B * a.n, dx = a.dx;
        float *pool = reinterpret_cast<float *>(ws + W.pool), *poolx = pool + (size_t)a.B * 64;
        BLK_TRY(cudaMemsetAsync(pool, 0, (size_t)a.B * (64 + dx) * 4, st));
        {   // edge sub-block (and the edge pooling sums)
            EdgeArgs e = {};
            e.B = a.B;
            e.n = a.n;
            e.Ein = a.Emid;
            e.Eout = a.Eout;
            e.W1 = a.wb[BW_E + 2];
            e.W2 = a.wb[BW_E + 4];
            EbParams &p = e.par;
            p.M = a.M;
            p.g1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 0]);
            p.s1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 1]);
            p.b1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 3]);
            p.b2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 5]);
            p.g2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 6]);
            p.s2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 7]);
            p.pool = pool;
            p.status = a.status;
            p.B = a.B;
            p.n = a.n;
            prof_mark(3, 0, st);
            BLK_TRY(edge_forward(e, st));
            prof_mark(3, 1, st);
        }
        // the global sub-block (its pooling of X' and its update) on a side stream,
        // beside the node sub-block: it needs the edge pooling sums and X' only
        BLK_TRY(cudaEventRecord(e0, st));
        BLK_TRY(cudaStreamWaitEvent(side, e0, 0));
        k_pool_x<<<dim3(a.B, dx / 64, (a.n + 63) / 64), 256, 0, side>>>(static_cast<const __nv_bfloat16 *>(a.Xmid),
                                                                        a.M, poolx, a.n, dx);
        BLK_TRY(cudaGetLastError());
        {   // global sub-block
            YParams p = y_params(a.B, a.n, a.dx, a.dy, a.wb, a.M);
            p.Xmid = static_cast<const __nv_bfloat16 *>(a.Xmid);
            p.y = static_cast<const __nv_bfloat16 *>(a.y);
            p.pool = pool;
            p.poolx = poolx;
            p.y1 = reinterpret_cast<float *>(saved + S.y1);
            p.pX = reinterpret_cast<float *>(saved + S.pX);
            p.pE = reinterpret_cast<float *>(saved + S.pE);
            p.yout = static_cast<__nv_bfloat16 *>(a.yout);
            const size_t smem = (size_t)(a.dx + 64 + 10 * a.dy + 256 + 32) * 4;
            k_y_fwd<<<a.B, 256, smem, side>>>(p);
            BLK_TRY(cudaGetLastError());
        }
        void *Xa = saved + S.Xa, *Hx = saved + S.Hx, *Xz = saved + S.Xz;
        BLK_TRY(ln_fwd(dx, a.Xmid, a.wb[BW_X + 0], a.wb[BW_X + 1], nullptr, Xa, R, st));
        {   // H = relu(Xa W1 + b1)
            const void *A[3] = {Xa, Xa, Xa}, *B[3] = {a.wb[BW_X + 2], a.wb[BW_X + 2], a.wb[BW_X + 2]};
            const void *bias[3] = {a.wb[BW_X + 3], a.wb[BW_X + 3], a.wb[BW_X + 3]};
            void *C[3] = {Hx, Hx, Hx};
            BLK_TRY(tc_gemm(4, R, 2 * dx, dx, 1, A, B, bias, C, 2 * dx, nullptr, nullptr, a.status, st, true));
        }
        {   // Xz = Xa + H W2 + b2
            const void *A[3] = {Hx, Hx, Hx}, *B[3] = {a.wb[BW_X + 4], a.wb[BW_X + 4], a.wb[BW_X + 4]};
            const void *bias[3] = {a.wb[BW_X + 5], a.wb[BW_X + 5], a.wb[BW_X + 5]};
            void *C[3] = {Xz, Xz, Xz};
            BLK_TRY(tc_gemm(5, R, dx, 2 * dx, 1, A, B, bias, C, dx, Xa, nullptr, a.status, st, true));
        }
        BLK_TRY(ln_fwd(dx, Xz, a.wb[BW_X + 6], a.wb[BW_X + 7], a.M, a.Xout, R, st));
        BLK_TRY(cudaEventRecord(e1, side));
        BLK_TRY(cudaStreamWaitEvent(st, e1, 0));
        return cudaSuccess;
    });
}

cudaError_t tail_backward(const TailBwd &a, char *ws, const BlockWs &W, const char *saved, const BlockSaved &S,
                          cudaStream_t st) {
    return with_side_streams([&](const cudaStream_t *ss, const cudaEvent_t *ev) -> cudaError_t {
        cudaStream_t side = ss[2];
        cudaEvent_t e0 = ev[0], e1 = ev[1];
        const int R = a.B * a.n, dx = a.dx;
        YParams yp = y_params(a.B, a.n, a.dx, a.dy, a.wb, a.M);
        yp.y1 = const_cast<float *>(reinterpret_cast<const float *>(saved + S.y1));
        yp.pX = const_cast<float *>(reinterpret_cast<const float *>(saved + S.pX));
        yp.pE = const_cast<float *>(reinterpret_cast<const float *>(saved + S.pE));
        yp.dyout = static_cast<const __nv_bfloat16 *>(a.dyout);
        yp.dy1 = reinterpret_cast<float *>(ws + W.dy1);
        yp.dpX = reinterpret_cast<float *>(ws + W.dpX);
        yp.dpE = reinterpret_cast<float *>(ws + W.dpE);
        yp.yv = reinterpret_cast<float *>(ws + W.yv);
        {
            const size_t smem = (size_t)(15 * a.dy + 256 + 32) * 4;
            k_y_bwd<<<a.B, 256, smem, st>>>(yp);
            BLK_TRY(cudaGetLastError());
        }
        {   // edge sub-block backward: dE' (+ the pooling's gradient), partial sums
            EdgeArgs e = {};
            e.B = a.B;
            e.n = a.n;
            e.Ein = a.Emid;
            e.dEout = a.dEout;
            e.dEin = a.dEmid;
            e.W1 = a.wb[BW_E + 2];
            e.W2 = a.wb[BW_E + 4];
            EbParams &p = e.par;
            p.M = a.M;
            p.g1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 0]);
            p.s1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 1]);
            p.b1 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 3]);
            p.b2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 5]);
            p.g2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 6]);
            p.s2 = static_cast<const __nv_bfloat16 *>(a.wb[BW_E + 7]);
            p.dpool = reinterpret_cast<const float *>(ws + W.dpE);
            p.parts = reinterpret_cast<float *>(ws + W.eparts);
            p.wparts = reinterpret_cast<float *>(ws + W.ewparts);
            p.status = a.status;
            p.B = a.B;
            p.n = a.n;
            prof_mark(4, 0, st);
            BLK_TRY(edge_backward(e, st));
            prof_mark(4, 1, st);
        }
        {   // the global sub-block's parameter gradients on a side stream, beside the
            // node sub-block (after the edge kernel, which fills the GPU)
            BLK_TRY(cudaEventRecord(e0, st));
            BLK_TRY(cudaStreamWaitEvent(side, e0, 0));
            YGrads g;
            auto d = [&](int i) { return a.dwb[i]; };
            g.g1 = d(BW_Y + 0); g.s1 = d(BW_Y + 1); g.W1 = d(BW_Y + 2); g.b1 = d(BW_Y + 3);
            g.W2 = d(BW_Y + 4); g.b2 = d(BW_Y + 5); g.g2 = d(BW_Y + 6); g.s2 = d(BW_Y + 7);
            g.Wyx = d(BW_YX); g.Wye = d(BW_YE); g.by = d(BW_BY);
            const int total = 4 * a.dy * a.dy + (dx + 64) * a.dy + 2 * a.dy + 6 * a.dy;
            k_y_wgrad<<<(total + 255) / 256, 256, 0, side>>>(yp, g);
            BLK_TRY(cudaGetLastError());
        }
        void *dXz = ws + W.dXz, *dHx = ws + W.dHx, *dXa = ws + W.dXa, *dXmid = ws + W.dXmid;
        const void *Xa = saved + S.Xa, *Hx = saved + S.Hx, *Xz = saved + S.Xz;
        float *ln2 = reinterpret_cast<float *>(ws + W.ln2), *ln1 = reinterpret_cast<float *>(ws + W.ln1);
        BLK_TRY(ln_bwd(dx, Xz, a.dXout, a.wb[BW_X + 6], a.M, nullptr, nullptr, a.n, dXz, ln2, R, W.ln_grid, st));
        {   // dH = (dXz W2^T) [H > 0]
            const void *A[3] = {dXz, dXz, dXz}, *Bt[3] = {a.wb[BW_X + 4], a.wb[BW_X + 4], a.wb[BW_X + 4]};
            void *C[3] = {dHx, dHx, dHx};
            BLK_TRY(tc_gemm(6, R, 2 * dx, dx, 1, A, Bt, nullptr, C, 2 * dx, Hx, nullptr, a.status, st, false));
        }
        // dW1 = Xa^T dH, dW2 = H^T dXz (split-K partials) and the column sums of
        // dH and dXz (the bias gradients) on two side streams, beside dXa and the
        // first LayerNorm's backward: they need dH and dXz only
        float *cs1 = reinterpret_cast<float *>(ws + W.cs1), *cs2 = reinterpret_cast<float *>(ws + W.cs2);
        BLK_TRY(cudaEventRecord(ev[2], st));
        BLK_TRY(cudaStreamWaitEvent(ss[0], ev[2], 0));
        BLK_TRY(cudaStreamWaitEvent(ss[1], ev[2], 0));
        {
            float *g1 = reinterpret_cast<float *>(ws + W.wg1), *g2 = reinterpret_cast<float *>(ws + W.wg2);
            const void *B1[3] = {dHx, dHx, dHx}, *B2[3] = {dXz, dXz, dXz};
            float *const P1[3] = {g1, g1, g1}, *const P2[3] = {g2, g2, g2};
            BLK_TRY(tc_wgrad(dx, 2 * dx, 1, R, W.wsplits, Xa, B1, P1, a.status, ss[0]));
            k_colsum<<<W.cs_grid, 256, 0, ss[0]>>>(static_cast<const __nv_bfloat16 *>(dHx), cs1, R, 2 * dx, W.cs_rows);
            BLK_TRY(cudaGetLastError());
            BLK_TRY(tc_wgrad(2 * dx, dx, 1, R, W.wsplits, Hx, B2, P2, a.status, ss[1]));
            k_colsum<<<W.cs_grid, 256, 0, ss[1]>>>(static_cast<const __nv_bfloat16 *>(dXz), cs2, R, dx, W.cs_rows);
            BLK_TRY(cudaGetLastError());
        }
        {   // dXa = dXz + dH W1^T
            const void *A[3] = {dHx, dHx, dHx}, *Bt[3] = {a.wb[BW_X + 2], a.wb[BW_X + 2], a.wb[BW_X + 2]};
            void *C[3] = {dXa, dXa, dXa};
            BLK_TRY(tc_gemm(3, R, dx, 2 * dx, 1, A, Bt, nullptr, C, dx, dXz, nullptr, a.status, st, false));
        }
        BLK_TRY(ln_bwd(dx, a.Xmid, dXa, a.wb[BW_X + 0], nullptr, reinterpret_cast<const float *>(ws + W.dpX), a.M,
                       a.n, dXmid, ln1, R, W.ln_grid, st));
        BLK_TRY(cudaEventRecord(ev[3], ss[0]));
        BLK_TRY(cudaEventRecord(ev[4], ss[1]));
        BLK_TRY(cudaStreamWaitEvent(st, ev[3], 0));
        BLK_TRY(cudaStreamWaitEvent(st, ev[4], 0));
        {
            SumSegs sg = {};
            auto add = [&](const float *src, float *dst, int nparts, int stride, int count, int trows) {
                SumSeg &q = sg.seg[sg.n++];
                q.src = src;
                q.dst = dst;
                q.nparts = nparts;
                q.stride = stride;
                q.count = count;
                q.trows = trows;
            };
            auto dw = [&](int i) { return a.dwb[i]; };
            add(ln2, dw(BW_X + 6), W.ln_grid, 2 * dx, dx, 0);
            add(ln2 + dx, dw(BW_X + 7), W.ln_grid, 2 * dx, dx, 0);
            add(ln1, dw(BW_X + 0), W.ln_grid, 2 * dx, dx, 0);
            add(ln1 + dx, dw(BW_X + 1), W.ln_grid, 2 * dx, dx, 0);
            add(cs1, dw(BW_X + 3), W.cs_grid, 2 * dx, 2 * dx, 0);
            add(cs2, dw(BW_X + 5), W.cs_grid, dx, dx, 0);
            add(reinterpret_cast<float *>(ws + W.wg1), dw(BW_X + 2), W.wsplits, dx * 2 * dx, dx * 2 * dx, 0);
            add(reinterpret_cast<float *>(ws + W.wg2), dw(BW_X + 4), W.wsplits, 2 * dx * dx, 2 * dx * dx, 0);
            const float *ep = reinterpret_cast<const float *>(ws + W.eparts);
            const int np = W.ectas;
            add(ep + 0, dw(BW_E + 6), np, EB_PART, 64, 0);      // dg2
            add(ep + 64, dw(BW_E + 7), np, EB_PART, 64, 0);     // ds2
            add(ep + 128, dw(BW_E + 5), np, EB_PART, 64, 0);    // db2
            add(ep + 192, dw(BW_E + 0), np, EB_PART, 64, 0);    // dg1
            add(ep + 256, dw(BW_E + 1), np, EB_PART, 64, 0);    // ds1
            add(ep + 320, dw(BW_E + 3), np, EB_PART, 128, 0);   // db1
            const float *ew = reinterpret_cast<const float *>(ws + W.ewparts);
            add(ew, dw(BW_E + 4), W.ectas, 2 * 128 * 64, 128 * 64, 0);            // dW2 [128][64]
            add(ew + 128 * 64, dw(BW_E + 2), W.ectas, 2 * 128 * 64, 128 * 64, 128);  // dW1 = (dW1^T)^T
            int ctas = 0;
            for (int s = 0; s < sg.n; ++s)
                ctas += sg.seg[s].nparts > 16 ? (sg.seg[s].count + 31) / 32 : (sg.seg[s].count + 255) / 256;
            k_sum_parts<<<ctas, 256, 0, st>>>(sg);
            BLK_TRY(cudaGetLastError());
        }
        BLK_TRY(cudaEventRecord(e1, side));
        BLK_TRY(cudaStreamWaitEvent(st, e1, 0));
        return cudaSuccess;
    });
}

cudaError_t add_dy(void *dy, const float *dy1, int count, cudaStream_t st) {
    k_add_dy<<<(count + 255) / 256, 256, 0, st>>>(static_cast<__nv_bfloat16 *>(dy), dy1, count);
    return cudaGetLastError();
}

}  // namespace blk
}  // namespace fast
}  // namespace eaga
