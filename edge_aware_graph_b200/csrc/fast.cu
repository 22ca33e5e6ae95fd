// Host glue of the specialised sm_100a path (de = 64, H = 8, dh = 32, bf16):
// which dims it covers, its workspace, its launch sequence and launch count.
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

cudaError_t launch_prologue(const eaga_dims &d, const void *const w[12], const void *y, float *g, uint8_t *img,
                            cudaStream_t st);
cudaError_t launch_qkv(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_out_proj(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, const uint8_t *img, const float *g,
                             cudaStream_t st);
cudaError_t launch_dO(const eaga_dims &d, const BwdArgs &a, __nv_bfloat16 *dO, cudaStream_t st);
cudaError_t launch_dX(const eaga_dims &d, const BwdArgs &a, const __nv_bfloat16 *dN[3], cudaStream_t st);
cudaError_t launch_wgrad(const eaga_dims &d, const BwdArgs &a, const __nv_bfloat16 *dN[3], float *parts,
                         int splits, cudaStream_t st);
cudaError_t launch_bwd_pairs(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                             cudaStream_t st);
cudaError_t launch_bwd_finish(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, float *dg,
                              cudaStream_t st);

bool supports(const eaga_dims &d) {
    return d.dtype == EAGA_BF16 && d.de == DE && d.H == NH && d.dh == DH && d.n % 2 == 0 && d.n >= 2 &&
           d.n <= 1024 && d.dx % 64 == 0 && d.dx >= 64;
}

// Forward: the operand images after the common workspace; backward: the whole FastWs.
size_t workspace_size(const eaga_dims &d, int for_backward, size_t common_fwd, size_t common_head) {
    if (!for_backward) return align256(common_fwd + IMG_BYTES);
    return fast_ws(d, common_head).total;
}

int kernel_launches(const eaga_dims &, int for_backward) {
    // forward: prologue, QKV, pairs, out-proj
    // backward: prologue, dO, rows, cols, dX, wgrad x2, bias partial, rparts partial, finish, film grads
    return for_backward ? 11 : 4;
}

#define FAST_TRY(x)                               \
    do {                                          \
        cudaError_t e_ = (x);                     \
        if (e_ != cudaSuccess) return e_;         \
    } while (0)

cudaError_t forward(const eaga_dims &d, const FwdArgs &a, char *ws_after_common, cudaStream_t st) {
    uint8_t *img = reinterpret_cast<uint8_t *>(ws_after_common);
    FAST_TRY(launch_prologue(d, a.w, a.y, a.g, img, st));
    FAST_TRY(launch_qkv(d, a, st));
    prof_mark(0, 0, st);
    FAST_TRY(launch_fwd_pairs(d, a, img, a.g, st));
    prof_mark(0, 1, st);
    return launch_out_proj(d, a, st);
}

cudaError_t backward(const eaga_dims &d, const BwdArgs &a, char *ws, size_t head, cudaStream_t st) {
    const FastWs W = fast_ws(d, head);
    uint8_t *img = reinterpret_cast<uint8_t *>(ws + W.img);
    __nv_bfloat16 *dO = reinterpret_cast<__nv_bfloat16 *>(ws + W.dO);
    FAST_TRY(launch_prologue(d, a.w, a.y, a.g, img, st));
    FAST_TRY(launch_dO(d, a, dO, st));
    prof_mark(1, 0, st);
    FAST_TRY(launch_bwd_pairs(d, a, W, ws, a.g, st));
    prof_mark(1, 1, st);
    const __nv_bfloat16 *dN[3] = {reinterpret_cast<const __nv_bfloat16 *>(ws + W.dQ),
                                  reinterpret_cast<const __nv_bfloat16 *>(ws + W.dK),
                                  reinterpret_cast<const __nv_bfloat16 *>(ws + W.dV)};
    FAST_TRY(launch_dX(d, a, dN, st));
    FAST_TRY(launch_wgrad(d, a, dN, reinterpret_cast<float *>(ws + W.wparts), W.wsplits, st));
    return launch_bwd_finish(d, a, W, ws, reinterpret_cast<float *>(ws + W.dg), st);
}

}  // namespace fast
}  // namespace eaga
