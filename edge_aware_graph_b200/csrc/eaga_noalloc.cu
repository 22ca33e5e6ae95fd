// eaga_forward_noalloc: the forward of the layer for callers that cannot hand
// the library a device workspace.
//
// Some callers have no way to allocate device memory for scratch: plain C
// clients that link this library but no device allocator, or code running
// under a framework whose memory pool must not be bypassed and that only
// hands out the tensors it owns (inputs, outputs, the saved state).  For them
// the forward's small scratch (the status word, the per-graph global FiLM
// term and the tensor-core operand images of the FiLM and edge weights) lives
// in a fixed device array inside this library instead of a caller buffer.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds NOALLOC_SCRATCH_BYTES of it until the process exits.  All
// calls on a device share it and it keeps the last call's contents; calls
// that overlap on the GPU (different streams, or different host threads on
// the same device) race on it and must be serialised by the caller.
#include <mutex>
#include "common.cuh"
#include "fast.h"
#include "generic.h"

using namespace eaga;

namespace {

constexpr size_t NOALLOC_SCRATCH_BYTES = 64 * 1024;   // status word + g [B,2H] fp32 + 8 KB of operand images
constexpr size_t NOALLOC_STATUS = 0, NOALLOC_G = 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_setup_mutex;
void *g_scratch_addr[MAX_DEVICES] = {};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace eaga {

// The device address of the array on the current device.  In host code the
// variable's name only stands for it, so the address is looked up once per
// device (with that device current) and cached.
eaga_status noalloc_scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return EAGA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return EAGA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return EAGA_OK;
}

}  // namespace eaga

extern "C" {

eaga_status eaga_forward_noalloc(const eaga_dims *d, const void *X, const void *E, const void *y, const uint8_t *M,
                                 const eaga_weights *w, void *Xout, void *Eout, void *saved, void *stream) {
    // The same argument checks as eaga_forward, with `saved` required: the
    // forward's saved state is as large as the node tensors and stays the
    // caller's buffer.
    const eaga_status ds = check_dims(d);
    if (ds != EAGA_OK) return ds;
    if (!w) return EAGA_ERR_INVALID_ARG;
    const void *ptrs[] = {X, E, y, M, Xout, Eout, saved, w->Wq, w->bq, w->Wk, w->bk, w->Wv,
                          w->bv, w->Wfe, w->Wfy, w->bf, w->We, w->Wo, w->bo};
    for (const void *p : ptrs) {
        if (!p) return EAGA_ERR_INVALID_ARG;
        if (!aligned16(p)) return EAGA_ERR_MISALIGNED;
    }
    const size_t g_bytes = align256(size_t(d->B) * 2 * d->H * sizeof(float));
    const bool fast_path = fast::supports(*d);
    const size_t images = fast_path ? fast::forward_scratch_bytes(*d, false) : 0;
    const size_t needed = NOALLOC_G + g_bytes + images;
    if (needed > NOALLOC_SCRATCH_BYTES) return EAGA_ERR_UNSUPPORTED;   // too large for the fixed array
    // the pair kernel's row-block order where it still fits (else index order)
    const bool with_order = fast_path && NOALLOC_G + g_bytes + fast::forward_scratch_bytes(*d) <= NOALLOC_SCRATCH_BYTES;
    {
        const Extents x = tensor_extents(*d);
        const Span outs[3] = {{Xout, x.X}, {Eout, x.E}, {saved, saved_layout(*d).saved_total}};
        Span ins[16] = {{X, x.X}, {E, x.E}, {y, x.y}, {M, x.M}};
        const void *wsrc[12] = {w->Wq, w->bq, w->Wk, w->bk, w->Wv, w->bv, w->Wfe, w->Wfy, w->bf, w->We, w->Wo, w->bo};
        for (int t = 0; t < 12; ++t) ins[4 + t] = {wsrc[t], x.w[t]};
        const eaga_status s = check_no_alias(outs, 3, ins, 16);
        if (s != EAGA_OK) return s;
    }

    void *base = nullptr;
    eaga_status s = noalloc_scratch_address(&base);
    if (s != EAGA_OK) return s;
    char *scratch = static_cast<char *>(base);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const Layout L = saved_layout(*d);
    char *sv = static_cast<char *>(saved);
    FwdArgs a;
    a.X = X; a.E = E; a.y = y; a.M = M;
    const void *wsrc[12] = {w->Wq, w->bq, w->Wk, w->bk, w->Wv, w->bv, w->Wfe, w->Wfy, w->bf, w->We, w->Wo, w->bo};
    for (int t = 0; t < 12; ++t) a.w[t] = wsrc[t];
    a.Xout = Xout; a.Eout = Eout;
    a.LSE = reinterpret_cast<float *>(sv + L.lse);
    a.Q = sv + L.q; a.K = sv + L.k; a.V = sv + L.v; a.O = sv + L.o;
    a.status = reinterpret_cast<int *>(scratch + NOALLOC_STATUS);
    a.g = reinterpret_cast<float *>(scratch + NOALLOC_G);
    // The status word must start at zero; g and the images are rewritten in full by every call.
    if (cudaMemsetAsync(a.status, 0, sizeof(int), st) != cudaSuccess) return EAGA_ERR_CUDA;
    cudaError_t e = fast_path ? fast::forward(*d, a, scratch + NOALLOC_G + g_bytes, st, with_order)
                                       : generic::forward(*d, a, st);
    return e == cudaSuccess ? EAGA_OK : EAGA_ERR_CUDA;
}

}  // extern "C"
