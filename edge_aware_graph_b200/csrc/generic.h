// Launch arguments of the CUDA-core kernels (generic_kernels.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>
#include "eaga.h"

namespace eaga {

// Weight order everywhere: Wq bq Wk bk Wv bv Wfe Wfy bf We Wo bo.
// `variant` is an eaga_variant: the layer, Light Edge (no per-edge FiLM map)
// or the unnormalised edge update (from the modulated scores s').
// row0, rows: the slab of each graph's rows the call owns (rows < 0: the
// whole graph); E, Eout (dEout, dE) then hold those rows only, [B, rows, n, de].
struct FwdArgs {
    int variant = 0;
    int row0 = 0, rows = -1;
    const void *X, *E, *y;
    const uint8_t *M;
    const void *w[12];
    void *Xout, *Eout;
    void *Q, *K, *V, *O;     // saved (storage dtype) [B,n,H*dh]
    float *LSE;              // saved [B,H,n]
    float *g;                // workspace [B,2H]
    int *status;             // workspace status word
};

struct BwdArgs {
    int variant = 0;
    int row0 = 0, rows = -1;
    const void *X, *E, *y;
    const uint8_t *M;
    const void *w[12];
    const void *Q, *K, *V, *O;
    const float *LSE;
    const void *dXout, *dEout;
    void *dX, *dE, *dy;
    float *dW[12];
    float *g, *dO, *dQ, *dK, *dV, *D, *parts, *dg;
    size_t part_stride;
    int *status;
};

struct MapArgs {
    const void *E, *y, *Wfe, *Wfy, *bf;
    const uint8_t *M;
    const void *Q, *K;
    const float *LSE;
    float *g, *A;
};

namespace generic {
cudaError_t forward(const eaga_dims &d, const FwdArgs &a, cudaStream_t st);
cudaError_t backward(const eaga_dims &d, const BwdArgs &a, cudaStream_t st);
cudaError_t attention_map(const eaga_dims &d, const MapArgs &a, cudaStream_t st);
size_t max_dynamic_smem(const eaga_dims &d);
int kernel_launches(const eaga_dims &d, int for_backward);
}  // namespace generic
}  // namespace eaga
