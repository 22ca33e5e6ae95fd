// Backward reductions of the specialised path (de = 64, H = 8, dh = 32, bf16
// storage), after the pair kernel (fast_bwd_stream.cu): bias gradients, the
// per-(graph, row block) dWfe / dWe / dg partials, the split-K
// weight-gradient partials, and the global FiLM term's dWfy, dbf, dy; all in
// a fixed order.
#include <math.h>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using namespace dev;

// ---------------------------------------------------------------- reductions
// All sums run in a fixed order (deterministic): first over segments of rows
// (or CTAs) in parallel blocks, then over the segments.

// Column sums of segment z of the rows: out[z][col].  Sources by column:
// [0,256) dQ, [256,512) dK, [512,768) dV, [768,768+dx) M-masked dX'.  Block
// (256-column strip, row segment): lane = 8 columns (one 16-byte load per
// row), warp = every 8th row of the segment, warps added in a fixed order.
__device__ __forceinline__ void bias_partial(const __nv_bfloat16 *dQ, const __nv_bfloat16 *dK,
                                             const __nv_bfloat16 *dV, const __nv_bfloat16 *dXo, const uint8_t *M,
                                             int rows, int dx, int seg_rows, float *out, int bx, int by) {
    __shared__ float red[8][256];
    const int w = threadIdx.x >> 5, t = threadIdx.x & 31;
    const int strip = bx, ncol = 3 * HD + dx;
    const bool masked = strip >= 3;
    const __nv_bfloat16 *src = strip == 0 ? dQ : strip == 1 ? dK : strip == 2 ? dV : dXo;
    const int ld = masked ? dx : HD, c0 = (masked ? (strip - 3) * 256 : 0) + 8 * t;
    const bool active = c0 < ld;
    const int r0 = by * seg_rows, r1 = min(rows, r0 + seg_rows);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
#pragma unroll 4
        for (int r = r0 + w; r < r1; r += 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + (size_t)r * ld + c0);
            const bool keep = !masked || M[r];
            const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(v2[u]);
                acc[2 * u] += keep ? f.x : 0.f;
                acc[2 * u + 1] += keep ? f.y : 0.f;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) red[w][8 * t + u] = acc[u];
    __syncthreads();
    const int col = threadIdx.x, gcol = strip * 256 + col;
    if (gcol < ncol && (!masked || (strip - 3) * 256 + col < dx)) {
        float x = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) x += red[k][col];
        out[(size_t)by * ncol + gcol] = x;
    }
}

// sum_{z < count} src[z * stride] with four independent accumulators (loads in
// flight together), combined in a fixed order: deterministic.
__device__ __forceinline__ float strided_sum(const float *src, int count, size_t stride) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int z = 0;
    for (; z + 4 <= count; z += 4) {
        a0 += src[(size_t)z * stride];
        a1 += src[(size_t)(z + 1) * stride];
        a2 += src[(size_t)(z + 2) * stride];
        a3 += src[(size_t)(z + 3) * stride];
    }
    for (; z < count; ++z) a0 += src[(size_t)z * stride];
    return (a0 + a1) + (a2 + a3);
}

// Row-kernel partials: out[z][e] = sum over CTAs of segment z of rparts[cta][e], e < dWfe+dWe
// (blockIdx.y = z < gridDim.y - 1); the last row of blocks sums each graph's
// dg_b = sum over its row blocks of their dg partials.
__device__ __forceinline__ void rparts_partial(const float *rparts, int ctas, int seg, float *out, float *dg, int B,
                                               int ctas_per_graph, int bx, int by, int gy) {
    const int e = bx * blockDim.x + threadIdx.x;
    constexpr int NE = DE * NF + NH * DE;
    if (by + 1 == gy) {
        if (e < B * NF) {
            const int b = e / NF, k = e % NF;
            dg[e] = strided_sum(rparts + (size_t)b * ctas_per_graph * RPART + NE + k, ctas_per_graph, RPART);
        }
        return;
    }
    if (e >= NE) return;
    const int c0 = by * seg, c1 = min(ctas, c0 + seg);
    out[(size_t)by * NE + e] = c1 > c0 ? strided_sum(rparts + (size_t)c0 * RPART + e, c1 - c0, RPART) : 0.f;
}

// The bias partials (CTA rows y < bsplits: column sums of dQ, dK, dV and the
// masked dX' over row segments) and the row-block partials (the other rows:
// sums of the pair kernel's per-row-block partials over CTA segments, and dg)
// in one launch; the two jobs are independent.
__global__ void __launch_bounds__(256) k_bwd_partials(const __nv_bfloat16 *dQ, const __nv_bfloat16 *dK,
                                                      const __nv_bfloat16 *dV, const __nv_bfloat16 *dXo,
                                                      const uint8_t *M, int rows, int dx, int seg_rows, float *bout,
                                                      int bias_x, int bsplits, const float *rparts, int ctas, int seg,
                                                      float *rout, float *dg, int B, int ctas_per_graph, int rp_x,
                                                      int rp_y) {
    if ((int)blockIdx.y < bsplits) {
        if ((int)blockIdx.x < bias_x) bias_partial(dQ, dK, dV, dXo, M, rows, dx, seg_rows, bout, blockIdx.x, blockIdx.y);
        return;
    }
    if ((int)blockIdx.x < rp_x)
        rparts_partial(rparts, ctas, seg, rout, dg, B, ctas_per_graph, blockIdx.x, blockIdx.y - bsplits, rp_y);
}

struct DWPtrs {
    float *p[12];
};

// Final sums: weight gradients of the four node projections (split-K
// partials), bias gradients, dWfe / dWe.
__global__ void k_bwd_finish(const float *wparts, int wsplits, const float *bparts, int bsplits,
                             const float *r2, int rsplits, int dx, DWPtrs dW, int zero_wfe, int e0, int e1) {
    const int e = e0 + blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= e1) return;
    const int msz = dx * HD;
    const int ncol = 3 * HD + dx;
    constexpr int NE = DE * NF + NH * DE;
    if (e < 4 * msz) {
        const int q = e / msz, o = e % msz;
        const float *src = wparts + (size_t)q * wsplits * msz + o;
        dW.p[q == 0 ? 0 : q == 1 ? 2 : q == 2 ? 4 : 10][o] = strided_sum(src, wsplits, msz);
        return;
    }
    int x = e - 4 * msz;
    if (x < ncol) {
        const float acc = strided_sum(bparts + x, bsplits, ncol);
        if (x < 3 * HD) dW.p[1 + 2 * (x / HD)][x % HD] = acc;
        else dW.p[11][x - 3 * HD] = acc;
        return;
    }
    x -= ncol;
    if (x < NE) {
        const float acc = strided_sum(r2 + x, rsplits, NE);
        // (Light Edge: Wfe is not a parameter, its gradient is zero)
        if (x < DE * NF) dW.p[6][x] = zero_wfe ? 0.f : acc; else dW.p[9][x - DE * NF] = acc;
    }
}

// dbf, dWfy, dy from dg (after k_bwd_partials).
__global__ void k_film_grads(const float *dg, int B, int dy, const __nv_bfloat16 *y, const __nv_bfloat16 *Wfy,
                             float *dbf, float *dWfy, __nv_bfloat16 *dyo) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < NF) {
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc += dg[b * NF + e];
        dbf[e] = acc;
    } else if (e < NF + dy * NF) {
        const int x = e - NF, c = x / NF, k = x % NF;
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc = fmaf(__bfloat162float(y[(size_t)b * dy + c]), dg[b * NF + k], acc);
        dWfy[x] = acc;
    } else if (e < NF + dy * NF + B * dy) {
        const int x = e - NF - dy * NF, b = x / dy, c = x % dy;
        float acc = 0.f;
        for (int k = 0; k < NF; ++k) acc = fmaf(dg[b * NF + k], __bfloat162float(Wfy[c * NF + k]), acc);
        dyo[x] = __float2bfloat16_rn(acc);
    }
}

// The order in which a pair kernel's CTAs take the row blocks: longest first
// (the most chunks with a valid pair), graph-major among equals, so that the
// short row blocks (few live chunks, or none: only copies) fill the last
// wave instead of leaving SMs idle behind a long one.  A row block's live
// chunks are the graph's chunks holding a node when one of its rows is a
// node, none otherwise (exactly live_chunk_mask's count).  One CTA: per
// graph the chunks holding a node (a warp a graph), per row block whether a
// row is a node, then a stable counting sort on the count (bin k: 32 - k live
// chunks).  Item = graph * row blocks of the slab + row block.
__global__ void __launch_bounds__(1024) k_row_block_order(const uint8_t *M, int B, int n, int row0, int rows,
                                                          int *order) {
    __shared__ uint8_t cost[ORDER_MAX_ITEMS];
    __shared__ uint8_t gcount[ORDER_MAX_ITEMS];
    __shared__ int bin_start[33];
    const int nrb = (rows + TB - 1) / TB, items = B * nrb;
    const int w = threadIdx.x >> 5, t = threadIdx.x & 31;
    if (items > ORDER_MAX_ITEMS) {
        for (int i = threadIdx.x; i < items; i += blockDim.x) order[i] = i;
        return;
    }
    if (threadIdx.x < 33) bin_start[threadIdx.x] = 0;
    for (int g = w; g < B; g += 32) {   // chunks of graph g holding a node (n even: 2-byte loads)
        const uint16_t *m2 = reinterpret_cast<const uint16_t *>(M + (size_t)g * n);
        uint32_t any = 0;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int j = 32 * t + 2 * k;
            if (j < n) any |= m2[j >> 1];
        }
        const uint32_t gm = __ballot_sync(0xffffffffu, any != 0);
        if (t == 0) gcount[g] = (uint8_t)__popc(gm);
    }
    __syncthreads();
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int b = it / nrb, i0 = row0 + (it % nrb) * TB;
        bool row = false;
        for (int k = 0; k < TB; ++k) row |= i0 + k < n && M[(size_t)b * n + i0 + k] != 0;
        const int c = row ? gcount[b] : 0;
        cost[it] = (uint8_t)c;
        atomicAdd(&bin_start[32 - c], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {   // counts -> where each bin starts
        int acc = 0;
        for (int k = 0; k < 33; ++k) {
            const int c = bin_start[k];
            bin_start[k] = acc;
            acc += c;
        }
    }
    __syncthreads();
    for (int k = w; k <= 32; k += 32) {
        int pos = bin_start[k];
        for (int base = 0; base < items; base += 32) {
            const int it = base + t;
            const bool mine = it < items && 32 - cost[it] == k;
            const uint32_t bal = __ballot_sync(0xffffffffu, mine);
            if (mine) order[pos + __popc(bal & ((1u << t) - 1u))] = it;
            pos += __popc(bal);
        }
    }
}

cudaError_t launch_row_block_order(const eaga_dims &d, const uint8_t *M, int row0, int rows, int *order,
                                   cudaStream_t st) {
    k_row_block_order<<<1, 1024, 0, st>>>(M, d.B, d.n, row0, rows, order);
    return cudaGetLastError();
}

// ---------------------------------------------------------------- host side

cudaError_t launch_bwd_stream(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                              cudaStream_t st);

// The backward pair kernel (profile point 2 brackets it alone).
cudaError_t launch_bwd_pairs(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                             cudaStream_t st) {
    prof_mark(2, 0, st);
    const cudaError_t e = launch_bwd_stream(d, a, W, ws, g, st);
    prof_mark(2, 1, st);
    return e;
}

// dK = bf16(dK32 / sqrt(dh)), dV = bf16(dV32): the pair kernel's fp32 sums over
// row blocks, for the node GEMMs and the bias sums (four features per thread).
__global__ void k_kv_convert(const float4 *dK32, const float4 *dV32, size_t n4, __nv_bfloat16 *dK,
                             __nv_bfloat16 *dV) {
    griddep_launch_dependents();
    griddep_wait();
    const float rs = rsqrtf((float)DH);
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < n4; x += (size_t)gridDim.x * blockDim.x) {
        const float4 k = dK32[x], v = dV32[x];
        uint2 ko, vo;
        ko.x = sm100::pack_bf16(k.x * rs, k.y * rs);
        ko.y = sm100::pack_bf16(k.z * rs, k.w * rs);
        vo.x = sm100::pack_bf16(v.x, v.y);
        vo.y = sm100::pack_bf16(v.z, v.w);
        reinterpret_cast<uint2 *>(dK)[x] = ko;
        reinterpret_cast<uint2 *>(dV)[x] = vo;
    }
}

cudaError_t launch_kv_convert(const eaga_dims &d, const FastWs &W, char *ws, cudaStream_t st) {
    const size_t n4 = (size_t)d.B * d.n * HD / 4;
    const int blocks = (int)std::min<size_t>((n4 + 255) / 256, (size_t)sm_count() * 8);
    return launch_pdl(k_kv_convert, dim3(blocks), dim3(256), 0, st, 1, reinterpret_cast<const float4 *>(ws + W.dK32),
                      reinterpret_cast<const float4 *>(ws + W.dV32), n4, reinterpret_cast<__nv_bfloat16 *>(ws + W.dK),
                      reinterpret_cast<__nv_bfloat16 *>(ws + W.dV));
}

// Column sums for the bias gradients and the first level of the row-block
// partials of dWfe / dWe (both read only what the pair kernels wrote).
cudaError_t launch_bwd_partials(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, cudaStream_t st) {
    const __nv_bfloat16 *dQ = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dQ);
    const __nv_bfloat16 *dK = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dK);
    const __nv_bfloat16 *dV = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dV);
    const int rows = d.B * d.n;
    float *bparts = reinterpret_cast<float *>(ws + W.bparts);
    const int seg_rows = (rows + W.bsplits - 1) / W.bsplits;
    const int bias_x = 3 + (d.dx + 255) / 256;
    float *r2 = reinterpret_cast<float *>(ws + W.r2);
    float *dg = reinterpret_cast<float *>(ws + W.dg);
    const int ctas = W.n_rparts, seg = (ctas + W.rsplits - 1) / W.rsplits;
    constexpr int NE = DE * NF + NH * DE;
    const float *rparts = reinterpret_cast<const float *>(ws + W.rparts);
    const int xblocks = (std::max(NE, d.B * NF) + 255) / 256;
    k_bwd_partials<<<dim3(std::max(bias_x, xblocks), W.bsplits + W.rsplits + 1), 256, 0, st>>>(
        dQ, dK, dV, static_cast<const __nv_bfloat16 *>(a.dXout), a.M, rows, d.dx, seg_rows, bparts, bias_x, W.bsplits,
        rparts, ctas, seg, r2, dg, d.B, (d.n + TB - 1) / TB, xblocks, W.rsplits + 1);
    return cudaGetLastError();
}

// dbf, dWfy, dy from dg (after launch_bwd_partials; off the path of dX and dW).
cudaError_t launch_film_grads(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, cudaStream_t st) {
    const float *dg = reinterpret_cast<const float *>(ws + W.dg);
    const int tf = NF + d.dy * NF + d.B * d.dy;
    k_film_grads<<<(tf + 255) / 256, 256, 0, st>>>(dg, d.B, d.dy, static_cast<const __nv_bfloat16 *>(a.y),
                                                   static_cast<const __nv_bfloat16 *>(a.w[7]), a.dW[8], a.dW[7],
                                                   static_cast<__nv_bfloat16 *>(a.dy));
    return cudaGetLastError();
}

// Final sums of the node projections' weight and bias gradients and of dWfe,
// dWe: entries [e0, e1) of dWq, dWk, dWv, dWo, the biases, dWfe, dWe (in that
// order; part 0 = dWq, dWk, dWv, part 1 = the rest), so that each part runs
// on the stream that produced its partials.
cudaError_t launch_bwd_final(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, int part,
                             cudaStream_t st) {
    const int ncol = 3 * HD + d.dx;
    constexpr int NE = DE * NF + NH * DE;
    DWPtrs dWdev;
    for (int q = 0; q < 12; ++q) dWdev.p[q] = a.dW[q];
    const int total = 4 * d.dx * HD + ncol + NE, split = 3 * d.dx * HD;
    const int e0 = part == 0 ? 0 : split, e1 = part == 0 ? split : total;
    k_bwd_finish<<<(e1 - e0 + 255) / 256, 256, 0, st>>>(
        reinterpret_cast<const float *>(ws + W.wparts), W.wsplits, reinterpret_cast<const float *>(ws + W.bparts),
        W.bsplits, reinterpret_cast<const float *>(ws + W.r2), W.rsplits, d.dx, dWdev,
        a.variant == EAGA_VARIANT_LIGHT_EDGE, e0, e1);
    return cudaGetLastError();
}

}  // namespace fast
}  // namespace eaga
