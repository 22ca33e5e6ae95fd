#include "fast.h"
namespace eaga {
namespace fast {
bool supports(const eaga_dims &) { return false; }
size_t workspace_extra(const eaga_dims &, int) { return 0; }
int kernel_launches(const eaga_dims &, int) { return 0; }
cudaError_t forward(const eaga_dims &, const FwdArgs &, char *, cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t backward(const eaga_dims &, const BwdArgs &, char *, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace fast
}  // namespace eaga
