// TMA tensor maps of the specialised path and the per-call prologue kernel
// (global FiLM term g_b and the tensor-core operand images of the small weights).
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder, looked up once (a function-local static:
// its initialisation is thread-safe).
static EncodeTiledFn get_encode() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        return nullptr;
    }();
    return fn;
}

// A [B, rows, n, 64] bf16 pair tensor (rows = n for a whole graph, fewer for
// a slab of its rows) viewed as 5-D, dims (c, ic, j, s, b) with i = 2ic + s,
// and a box of 4 x box_rows pairs of one parity s (box_s = 1) or 8 x box_rows
// (box_s = 2), landing in shared memory as [s][j box_rows][ic 4][c 64].
// Requires rows even (i = 2ic + s stays inside the slab).
bool encode_pair_map(CUtensorMap *m, const void *base, int B, int rows, int n, int box_rows, int box_s) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t rowb = DE * 2;                       // one pair: 128 bytes
    const cuuint64_t dims[5] = {DE, (cuuint64_t)(rows / 2), (cuuint64_t)n, 2, (cuuint64_t)B};
    const cuuint64_t strides[4] = {2 * (cuuint64_t)n * rowb,          // ic -> two rows i
                                   rowb,                              // j
                                   (cuuint64_t)n * rowb,              // s -> one row i
                                   (cuuint64_t)rows * n * rowb};      // b
    const cuuint32_t box[5] = {64, 4, (cuuint32_t)box_rows, (cuuint32_t)box_s, 1};
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [B, n, 256] bf16 node tensor; box of 64 features x box_rows nodes, 128B-swizzled.
bool encode_node_map(CUtensorMap *m, const void *base, int B, int n, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[3] = {HD, (cuuint64_t)n, (cuuint64_t)B};
    const cuuint64_t strides[2] = {HD * 2, (cuuint64_t)n * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A row-major [rows, cols] bf16 matrix; box of 64 columns x box_rows rows, 128B-swizzled.
bool encode_2d(CUtensorMap *m, const void *base, int rows, int cols, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A [B, n, n, 64] bf16 pair tensor as 4-D (c, j, i, b) with a box of 4 rows i
// x 32 columns j (128 pairs, landing as [i 4][j 32][c 64], 128B-swizzled).
bool encode_tile_map(CUtensorMap *m, const void *base, int B, int n) {
    auto enc = get_encode();
    if (!enc) return false;
    const cuuint64_t rowb = DE * 2;
    const cuuint64_t dims[4] = {DE, (cuuint64_t)n, (cuuint64_t)n, (cuuint64_t)B};
    const cuuint64_t strides[3] = {rowb, (cuuint64_t)n * rowb, (cuuint64_t)n * n * rowb};
    const cuuint32_t box[4] = {64, 32, 4, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// g_b = y_b Wfy + bf (fp32) for every graph: one warp per graph, lanes split
// the dy terms and add their 16 sums with shuffles in a fixed order.  The last
// block writes the four operand images from Wfe and We staged in shared memory
// and zeroes `nzero` ints at `zero_ints` (the backward pair kernel's row-block
// flags and work-item counter).
__global__ void __launch_bounds__(256) k_prologue(const __nv_bfloat16 *y, const __nv_bfloat16 *Wfy,
                                                  const __nv_bfloat16 *bf, const __nv_bfloat16 *Wfe,
                                                  const __nv_bfloat16 *We, float *g, uint8_t *img, int B, int dy,
                                                  int *zero_ints, int nzero) {
    sm100::griddep_launch_dependents();   // the pair kernel behind it may become resident
    const int w = threadIdx.x >> 5, t = threadIdx.x & 31;
    if (blockIdx.x + 1 < gridDim.x) {
        const int b = blockIdx.x * 8 + w;
        if (b >= B) return;
        float acc[NF];
#pragma unroll
        for (int k = 0; k < NF; ++k) acc[k] = 0.f;
        for (int c = t; c < dy; c += 32) {
            const float yc = __bfloat162float(y[(size_t)b * dy + c]);
            const uint4 *wr = reinterpret_cast<const uint4 *>(Wfy + (size_t)c * NF);
#pragma unroll
            for (int hlf = 0; hlf < 2; ++hlf) {
                const uint4 v = wr[hlf];
                const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float2 f = __bfloat1622float2(v2[u]);
                    acc[8 * hlf + 2 * u] = fmaf(yc, f.x, acc[8 * hlf + 2 * u]);
                    acc[8 * hlf + 2 * u + 1] = fmaf(yc, f.y, acc[8 * hlf + 2 * u + 1]);
                }
            }
        }
#pragma unroll
        for (int k = 0; k < NF; ++k)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
        if (t < NF) {
            float v = acc[0];
#pragma unroll
            for (int k = 1; k < NF; ++k) v = t == k ? acc[k] : v;
            g[(size_t)b * NF + t] = v + __bfloat162float(bf[t]);
        }
        return;
    }
    for (int e = threadIdx.x; e < nzero; e += blockDim.x) zero_ints[e] = 0;
    __shared__ __nv_bfloat16 sWfe[DE * NF], sWe[NH * DE];
    for (int e = threadIdx.x; e < DE * NF / 8; e += blockDim.x)
        reinterpret_cast<uint4 *>(sWfe)[e] = reinterpret_cast<const uint4 *>(Wfe)[e];
    for (int e = threadIdx.x; e < NH * DE / 8; e += blockDim.x)
        reinterpret_cast<uint4 *>(sWe)[e] = reinterpret_cast<const uint4 *>(We)[e];
    __syncthreads();
    const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
    for (int e = threadIdx.x; e < NF * DE; e += blockDim.x) {
        // IMG_WFE_T_SW: row k (16), element c (64)
        {
            const int k = e / DE, c = e % DE;
            *reinterpret_cast<__nv_bfloat16 *>(img + IMG_WFE_T_SW + sw128(k, c >> 3) + (c & 7) * 2) = sWfe[c * NF + k];
        }
        // IMG_WE_SW: row h (16, zero for h >= 8), element c
        {
            const int h = e / DE, c = e % DE;
            *reinterpret_cast<__nv_bfloat16 *>(img + IMG_WE_SW + sw128(h, c >> 3) + (c & 7) * 2) =
                h < NH ? sWe[h * DE + c] : zero;
        }
        // IMG_WE_T_NS: row c (64), element h (16, zero for h >= 8)
        {
            const int c = e / NF, h = e % NF;
            *reinterpret_cast<__nv_bfloat16 *>(img + IMG_WE_T_NS + ns16(c, h)) = h < NH ? sWe[h * DE + c] : zero;
        }
        // IMG_WFE_NS: row c (64), element k (16)
        {
            const int c = e / NF, k = e % NF;
            *reinterpret_cast<__nv_bfloat16 *>(img + IMG_WFE_NS + ns16(c, k)) = sWfe[c * NF + k];
        }
    }
}

cudaError_t launch_prologue(const eaga_dims &d, const void *const w[12], const void *y, float *g, uint8_t *img,
                            int *zero, int nzero, cudaStream_t st) {
    const int blocks = (d.B + 7) / 8 + 1;
    k_prologue<<<blocks, 256, 0, st>>>(
        static_cast<const __nv_bfloat16 *>(y), static_cast<const __nv_bfloat16 *>(w[7]),
        static_cast<const __nv_bfloat16 *>(w[8]), static_cast<const __nv_bfloat16 *>(w[6]),
        static_cast<const __nv_bfloat16 *>(w[9]), g, img, d.B, d.dy, zero, nzero);
    return cudaGetLastError();
}

}  // namespace fast
}  // namespace eaga
