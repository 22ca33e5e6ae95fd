// The graph-transformer block around the layer on the specialised sm_100a
// path (de = 64, H = 8, dh = 32, bf16 storage): launch helpers of its edge,
// node and global parts.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace eaga {
namespace fast {

bool encode_2d(CUtensorMap *m, const void *base, int rows, int cols, int box_rows);
bool encode_tile_map(CUtensorMap *m, const void *base, int B, int n);

namespace blk {

constexpr int EB_PART = 448;     // per-CTA channel sums of the edge backward: dg2, ds2, db2, dg1, ds1 [64], db1 [128]

// Parameters of the edge kernels (device pointers; bf16 parameters).
struct EbParams {
    const uint8_t *M;
    const __nv_bfloat16 *g1, *s1, *b1, *b2, *g2, *s2;
    float *pool;            // forward: [B, 64] sums of E' over valid pairs (added to)
    const float *dpool;     // backward: [B, 64] gradient of the edge pooling, divided by the pair count
    float *parts;           // backward: [CTAs][EB_PART]
    float *wparts;          // backward: [CTAs][2][128][64]: dW2, dW1^T
    int *status;
    int B, n, ti, tj;
};

struct EdgeArgs {
    int B, n;
    const void *Ein, *dEout;     // E' (the layer's output), dEout
    void *Eout, *dEin;           // Eout, dE'
    const void *W1, *W2;         // [64, 128], [128, 64]
    EbParams par;
};

// Block parameter order (the eaga_block_weights fields): node x, edge e and
// global y sub-blocks of ln1_g, ln1_s, W1, b1, W2, b2, ln2_g, ln2_s, then Wyx,
// Wye, by.
constexpr int BW_X = 0, BW_E = 8, BW_Y = 16, BW_YX = 24, BW_YE = 25, BW_BY = 26, BW_COUNT = 27;
constexpr int YV_PER_DY = 9;     // per-graph vectors of the global backward: h, dh [2 dy]; ya, dyz, x1, dya, x2 [dy]

struct YParams {
    int B, n, dx, dy;
    const uint8_t *M;
    const __nv_bfloat16 *g1, *s1, *W1, *b1, *W2, *b2, *g2, *s2, *Wyx, *Wye, *by;
    const __nv_bfloat16 *Xmid, *y, *dyout;
    const float *pool, *poolx;    // sums of E' over valid pairs [B, 64], of X' over real nodes [B, dx]
    float *y1, *pX, *pE;          // saved
    __nv_bfloat16 *yout;
    float *dy1, *dpX, *dpE, *yv;  // backward
};
struct YGrads {
    float *g1, *s1, *W1, *b1, *W2, *b2, *g2, *s2, *Wyx, *Wye, *by;
};

struct SumSeg {
    const float *src;
    float *dst;
    int nparts, stride, count, trows;
};
struct SumSegs {
    SumSeg seg[16];
    int n;
};

// Offsets (bytes) of the block's own saved state and workspace regions.
struct BlockSaved {
    size_t Xa, Hx, Xz, y1, pX, pE, total;
};
struct BlockWs {
    size_t pool, dXmid, dXz, dHx, dXa, dpX, dpE, dy1, yv, ln2, ln1, cs1, cs2, wg1, wg2, eparts, ewparts, total;
    int ln_grid, cs_grid, cs_rows, wsplits, ectas;
};

struct TailFwd {
    int B, n, dx, dy;
    const uint8_t *M;
    const void *y, *Xmid, *Emid;
    const void *const *wb;
    void *Xout, *Eout, *yout;
    int *status;
};
struct TailBwd {
    int B, n, dx, dy;
    const uint8_t *M;
    const void *Xmid, *Emid, *dXout, *dEout, *dyout;
    const void *const *wb;
    float *const *dwb;
    void *dEmid;
    int *status;
};

bool block_supports(int dx, int de, int dy);
BlockSaved block_saved_layout(int B, int n, int dx, int dy, size_t base);
BlockWs block_ws_layout(int B, int n, int dx, int dy, size_t base, int for_backward);
int block_kernel_launches(int for_backward);
YParams y_params(int B, int n, int dx, int dy, const void *const *wb, const uint8_t *M);
// b1-b4 after the layer: writes Xout, Eout, yout and the block's saved state.
cudaError_t tail_forward(const TailFwd &a, char *ws, const BlockWs &W, char *saved, const BlockSaved &S,
                         cudaStream_t st);
// Chain rule of b1-b4: writes dE' (a.dEmid), dX' (workspace dXmid), dy1
// (workspace) and every block parameter gradient.
cudaError_t tail_backward(const TailBwd &a, char *ws, const BlockWs &W, const char *saved, const BlockSaved &S,
                          cudaStream_t st);
cudaError_t add_dy(void *dy, const float *dy1, int count, cudaStream_t st);

cudaError_t edge_forward(const EdgeArgs &a, cudaStream_t st);
cudaError_t edge_backward(const EdgeArgs &a, cudaStream_t st);
int edge_backward_ctas(int B, int n);

}  // namespace blk
}  // namespace fast
}  // namespace eaga
