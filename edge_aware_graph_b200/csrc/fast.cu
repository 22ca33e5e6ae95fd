// Host glue of the specialised sm_100a path (de = 64, H = 8, dh = 32, bf16):
// which dims it covers, its launch sequence and its launch count.
#include "common.cuh"
#include "fast.h"

namespace eaga {
namespace fast {

cudaError_t launch_qkv(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_out_proj(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);
cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);

bool supports(const eaga_dims &d) {
    return d.dtype == EAGA_BF16 && d.de == 64 && d.H == 8 && d.dh == 32 && d.n % 2 == 0 && d.n >= 2 &&
           d.n <= 1024 && d.dx % 64 == 0 && d.dx >= 64;
}

size_t workspace_extra(const eaga_dims &, int) { return 0; }

int kernel_launches(const eaga_dims &d, int for_backward) {
    return for_backward ? generic::kernel_launches(d, 1) : 3;
}

cudaError_t forward(const eaga_dims &d, const FwdArgs &a, char *, cudaStream_t st) {
    cudaError_t e = launch_qkv(d, a, st);
    if (e != cudaSuccess) return e;
    prof_mark(0, 0, st);
    e = launch_fwd_pairs(d, a, st);
    prof_mark(0, 1, st);
    if (e != cudaSuccess) return e;
    return launch_out_proj(d, a, st);
}

cudaError_t backward(const eaga_dims &d, const BwdArgs &a, char *, cudaStream_t st) {
    return generic::backward(d, a, st);
}

}  // namespace fast
}  // namespace eaga
