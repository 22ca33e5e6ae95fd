// sm_100a kernels specialised for de = 64, H = 8, dh = 32, bf16 storage.
#pragma once
#include "generic.h"

namespace eaga {
namespace fast {
bool supports(const eaga_dims &d);
size_t workspace_extra(const eaga_dims &d, int for_backward);
int kernel_launches(const eaga_dims &d, int for_backward);
cudaError_t forward(const eaga_dims &d, const FwdArgs &a, char *ws_extra, cudaStream_t st);
cudaError_t backward(const eaga_dims &d, const BwdArgs &a, char *ws_extra, cudaStream_t st);
}  // namespace fast
}  // namespace eaga
