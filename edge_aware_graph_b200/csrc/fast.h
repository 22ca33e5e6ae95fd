// sm_100a kernels specialised for de = 64, H = 8, dh = 32, bf16 storage.
#pragma once
#include <functional>
#include "generic.h"

namespace eaga {
namespace fast {
bool supports(const eaga_dims &d);
// common_fwd: end of the common forward workspace; common_head: end of the
// status word and g (start of the backward's own regions).
size_t workspace_size(const eaga_dims &d, int for_backward, size_t common_fwd, size_t common_head);
int kernel_launches(const eaga_dims &d, int for_backward);
// Bytes the forward uses after the common workspace (the FiLM and edge operand images).
// with_order: also the pair kernel's row-block order (without it the row
// blocks run in index order)
size_t forward_scratch_bytes(const eaga_dims &d, bool with_order = true);
cudaError_t forward(const eaga_dims &d, const FwdArgs &a, char *ws_after_common, cudaStream_t st,
                    bool with_order = true);
cudaError_t backward(const eaga_dims &d, const BwdArgs &a, char *ws, size_t head, cudaStream_t st);
// Runs `enqueue` with the current device's three auxiliary streams and five
// events of their own, the streams' enqueue lock held for the duration (the
// block around the layer runs its global sub-block and its node weight
// gradients there).
cudaError_t with_side_streams(const std::function<cudaError_t(const cudaStream_t *side, const cudaEvent_t *ev)> &enqueue);
}  // namespace fast
}  // namespace eaga
