// Internal helpers shared by the CUDA translation units of libeaga.so.
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <atomic>
#include "eaga.h"

namespace eaga {

__device__ __forceinline__ float ldf(const float *p) { return *p; }
__device__ __forceinline__ float ldf(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
__device__ __forceinline__ void stf(float *p, float v) { *p = v; }
__device__ __forceinline__ void stf(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float warp_max(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// EAGA_ERR_INVALID_ARG for a null dims pointer, a non-positive dim or an
// unknown dtype; EAGA_ERR_UNSUPPORTED for dims outside the limits of eaga.h.
inline eaga_status check_dims(const eaga_dims *d) {
    if (!d) return EAGA_ERR_INVALID_ARG;
    if (d->B < 1 || d->n < 1 || d->dx < 1 || d->de < 1 || d->dy < 1 || d->H < 1 || d->dh < 1)
        return EAGA_ERR_INVALID_ARG;
    if (d->dtype != EAGA_FP32 && d->dtype != EAGA_BF16) return EAGA_ERR_INVALID_ARG;
    if (d->n > 1024 || d->H * d->dh > 256 || d->dh % 8 || d->de % 8 || d->de > 128 || d->dx % 8 ||
        d->dx > 1024 || d->dy % 8 || d->dy > 1024 || 2 * d->H > 32 || d->H * d->n > 8192)
        return EAGA_ERR_UNSUPPORTED;
    if ((size_t)d->B * d->n > (size_t)1 << 26) return EAGA_ERR_UNSUPPORTED;
    return EAGA_OK;
}

// Device address of the no-allocation forward's fixed scratch array on the
// current device (looked up once per device; eaga_noalloc.cu).  Its first
// int is that call's status word.
eaga_status noalloc_scratch_address(void **out);

// Byte layout of the forward's saved state and of the workspaces.
struct Layout {
    size_t lse, q, k, v, o, saved_total;        // offsets inside `saved`
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline Layout saved_layout(const eaga_dims &d) {
    const size_t es = d.dtype == EAGA_BF16 ? 2 : 4;
    const size_t rows = size_t(d.B) * d.n, hd = size_t(d.H) * d.dh;
    Layout L;
    size_t off = 0;
    L.lse = off; off = align256(off + size_t(d.B) * d.H * d.n * 4);
    L.q = off; off = align256(off + rows * hd * es);
    L.k = off; off = align256(off + rows * hd * es);
    L.v = off; off = align256(off + rows * hd * es);
    L.o = off; off = align256(off + rows * hd * es);
    L.saved_total = off;
    return L;
}

// Workspace: [status word (256 B)][g fp32 B*2H][forward: saved-equivalent if
// no saved buffer given][backward: dO, dQ, dK, dV fp32 rows*hd; D fp32 B*H*n;
// per-row parts fp32 rows*(de*2H + H*de + 2H); dg fp32 B*2H]
struct WsLayout {
    size_t status, g, fwd_saved, total_fwd;
    size_t dO, dQ, dK, dV, D, parts, dg, total_bwd;
    size_t part_stride;  // floats per row part
};

inline WsLayout ws_layout(const eaga_dims &d) {
    WsLayout W;
    const size_t rows = size_t(d.B) * d.n, hd = size_t(d.H) * d.dh, F = 2 * size_t(d.H);
    size_t off = 0;
    W.status = off; off = 256;
    W.g = off; off = align256(off + size_t(d.B) * F * 4);
    const size_t common = off;
    W.fwd_saved = off; off = align256(off + saved_layout(d).saved_total);
    W.total_fwd = off;
    off = common;
    W.dO = off; off = align256(off + rows * hd * 4);
    W.dQ = off; off = align256(off + rows * hd * 4);
    W.dK = off; off = align256(off + rows * hd * 4);
    W.dV = off; off = align256(off + rows * hd * 4);
    W.D = off; off = align256(off + size_t(d.B) * d.H * d.n * 4);
    W.part_stride = size_t(d.de) * F + size_t(d.H) * d.de + F;
    W.parts = off; off = align256(off + rows * W.part_stride * 4);
    W.dg = off; off = align256(off + size_t(d.B) * F * 4);
    W.total_bwd = off;
    return W;
}

// Optional profiling events around the pair kernels and the block's edge kernels
// (eaga_set_profile_events).
extern std::atomic<void *> g_prof_events[5][2];
inline void prof_mark(int point, int which, cudaStream_t st) {
    void *ev = g_prof_events[point][which].load(std::memory_order_acquire);
    if (ev) cudaEventRecord(static_cast<cudaEvent_t>(ev), st);
}

// Opt `kernel` in to `bytes` of dynamic shared memory on the current device,
// once per device (function attributes are per device).  `done` is the
// caller's per-kernel mask of devices already set; concurrent callers may both
// set the attribute, which is harmless.
template <typename K>
inline cudaError_t ensure_smem_attr(K kernel, int bytes, std::atomic<uint32_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint32_t bit = dev < 32 ? 1u << dev : 0u;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Byte extents of the layer's tensors for dims d: inputs in the storage
// dtype, weight gradients in fp32 (order of the eaga_weights fields).
struct Extents {
    size_t X, E, y, M, w[12], wgrad[12];
};
inline Extents tensor_extents(const eaga_dims &d) {
    const size_t s = d.dtype == EAGA_BF16 ? 2 : 4, hd = size_t(d.H) * d.dh, f = 2 * size_t(d.H);
    const size_t dx = d.dx, de = d.de, dy = d.dy;
    Extents x;
    x.X = size_t(d.B) * d.n * dx * s;
    x.E = size_t(d.B) * d.n * d.n * de * s;
    x.y = size_t(d.B) * dy * s;
    x.M = size_t(d.B) * d.n;
    const size_t count[12] = {dx * hd, hd, dx * hd, hd, dx * hd, hd, de * f, dy * f, f, size_t(d.H) * de, hd * dx, dx};
    for (int t = 0; t < 12; ++t) {
        x.w[t] = count[t] * s;
        x.wgrad[t] = count[t] * 4;
    }
    return x;
}

// A byte range [p, p + n) of device memory; n = 0 for an absent buffer.
struct Span {
    const void *p;
    size_t n;
};
inline bool spans_overlap(const Span &a, const Span &b) {
    const uintptr_t pa = reinterpret_cast<uintptr_t>(a.p), pb = reinterpret_cast<uintptr_t>(b.p);
    return a.n && b.n && pa < pb + b.n && pb < pa + a.n;
}
// EAGA_ERR_INVALID_ARG when an output range overlaps an input range or
// another output range (inputs may share memory: they are only read).
inline eaga_status check_no_alias(const Span *outs, int n_out, const Span *ins, int n_in) {
    for (int o = 0; o < n_out; ++o) {
        for (int i = 0; i < n_in; ++i)
            if (spans_overlap(outs[o], ins[i])) return EAGA_ERR_INVALID_ARG;
        for (int o2 = o + 1; o2 < n_out; ++o2)
            if (spans_overlap(outs[o], outs[o2])) return EAGA_ERR_INVALID_ARG;
    }
    return EAGA_OK;
}

// Device status word values (first int of the workspace).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1 };

}  // namespace eaga
