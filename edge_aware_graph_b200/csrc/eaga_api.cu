// C ABI of libeaga.so (declared in include/eaga.h): argument validation,
// saved-state and workspace layout, and the launch sequence on the caller's
// stream.  No device memory is allocated here.
#include <stdint.h>
#include <string.h>
#include "common.cuh"
#include "generic.h"
#include "fast.h"
#include "fast_block.h"
#include "sm100.cuh"
#include <nvtx3/nvToolsExt.h>

using namespace eaga;

namespace eaga {
std::atomic<void *> g_prof_events[5][2] = {};
}

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

eaga_status check_ptrs(std::initializer_list<const void *> ps) {
    for (const void *p : ps) {
        if (!p) return EAGA_ERR_INVALID_ARG;
        if (!aligned16(p)) return EAGA_ERR_MISALIGNED;
    }
    return EAGA_OK;
}

eaga_status check_weights(const eaga_weights *w) {
    if (!w) return EAGA_ERR_INVALID_ARG;
    return check_ptrs({w->Wq, w->bq, w->Wk, w->bk, w->Wv, w->bv, w->Wfe, w->Wfy, w->bf, w->We, w->Wo, w->bo});
}

void weight_array(const eaga_weights *w, const void *out[12]) {
    const void *src[12] = {w->Wq, w->bq, w->Wk, w->bk, w->Wv, w->bv, w->Wfe, w->Wfy, w->bf, w->We, w->Wo, w->bo};
    memcpy(out, src, sizeof(src));
}

// Appends the ranges of twelve weight (or weight-gradient) buffers, with
// extents `ext`, to `spans` at `k`.
int weight_spans(const void *const src[12], const size_t ext[12], Span *spans, int k) {
    for (int t = 0; t < 12; ++t) spans[k++] = {src[t], ext[t]};
    return k;
}

eaga_status launch_status(cudaError_t e) { return e == cudaSuccess ? EAGA_OK : EAGA_ERR_CUDA; }

}  // namespace

extern "C" {

size_t eaga_workspace_size(const eaga_dims *d, int for_backward) {
    if (check_dims(d) != EAGA_OK) return 0;
    const WsLayout W = ws_layout(*d);
    if (fast::supports(*d)) return fast::workspace_size(*d, for_backward, W.total_fwd, W.fwd_saved);
    return for_backward ? W.total_bwd : W.total_fwd;
}

size_t eaga_saved_size(const eaga_dims *d) {
    if (check_dims(d) != EAGA_OK) return 0;
    return saved_layout(*d).saved_total;
}

// NVTX range around an API call (visible to profilers that attach; inert otherwise).
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

static bool known_variant(int v) {
    return v == EAGA_VARIANT_LAYER || v == EAGA_VARIANT_LIGHT_EDGE || v == EAGA_VARIANT_UNNORMALISED;
}

// A slab of each graph's rows, row0 .. row0+rows-1 (rows < 0: the whole graph):
// the specialised path only; row0 and rows whole row blocks of 8 (the last
// slab may end at n).  Returns EAGA_OK or the reason it is refused.
static eaga_status check_slab(const eaga_dims &d, int row0, int rows) {
    if (rows < 0) return EAGA_OK;
    if (row0 < 0 || rows < 2 || (rows & 1) || row0 + rows > d.n || (row0 % 8) || ((rows % 8) && row0 + rows != d.n))
        return EAGA_ERR_INVALID_ARG;
    return fast::supports(d) ? EAGA_OK : EAGA_ERR_UNSUPPORTED;
}
// Bytes of an E-sized tensor of the slab.
static size_t slab_bytes(const eaga_dims &d, int rows) {
    const Extents x = tensor_extents(d);
    return rows < 0 ? x.E : x.E / d.n * rows;
}

static eaga_status forward_impl(const eaga_dims *d, int variant, int row0, int rows, const void *X, const void *E,
                                const void *y, const uint8_t *M, const eaga_weights *w, void *Xout, void *Eout,
                                void *saved, void *workspace, size_t ws_bytes, void *stream,
                                bool clear_status = true) {
    NvtxRange range("eaga_forward");
    eaga_status s = check_dims(d);
    if (s != EAGA_OK) return s;
    if (!known_variant(variant)) return EAGA_ERR_INVALID_ARG;
    if ((s = check_slab(*d, row0, rows)) != EAGA_OK) return s;
    if ((s = check_weights(w)) != EAGA_OK) return s;
    if ((s = check_ptrs({X, E, y, M, Xout, Eout, workspace})) != EAGA_OK) return s;
    if (saved && !aligned16(saved)) return EAGA_ERR_MISALIGNED;
    const Layout L = saved_layout(*d);
    {
        const Extents x = tensor_extents(*d);
        const size_t xe = slab_bytes(*d, rows);
        const Span outs[4] = {{Xout, x.X}, {Eout, xe}, {saved, saved ? L.saved_total : 0},
                              {workspace, eaga_workspace_size(d, 0)}};
        Span ins[16] = {{X, x.X}, {E, xe}, {y, x.y}, {M, x.M}};
        const void *wsrc[12];
        weight_array(w, wsrc);
        weight_spans(wsrc, x.w, ins, 4);
        if ((s = check_no_alias(outs, 4, ins, 16)) != EAGA_OK) return s;
    }
    if (ws_bytes < eaga_workspace_size(d, 0)) return EAGA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout W = ws_layout(*d);
    char *ws = static_cast<char *>(workspace);
    char *sv = saved ? static_cast<char *>(saved) : ws + W.fwd_saved;
    FwdArgs a;
    a.variant = variant;
    a.row0 = rows < 0 ? 0 : row0;
    a.rows = rows;
    a.X = X; a.E = E; a.y = y; a.M = M;
    weight_array(w, a.w);
    a.Xout = Xout; a.Eout = Eout;
    a.LSE = reinterpret_cast<float *>(sv + L.lse);
    a.Q = sv + L.q; a.K = sv + L.k; a.V = sv + L.v; a.O = sv + L.o;
    a.g = reinterpret_cast<float *>(ws + W.g);
    a.status = reinterpret_cast<int *>(ws + W.status);
    if (clear_status && cudaMemsetAsync(a.status, 0, sizeof(int), st) != cudaSuccess) return EAGA_ERR_CUDA;
    if (fast::supports(*d)) {
        return launch_status(fast::forward(*d, a, ws + W.total_fwd, st));
    }
    return launch_status(generic::forward(*d, a, st));
}

eaga_status eaga_forward_variant(const eaga_dims *d, int variant, const void *X, const void *E, const void *y,
                                 const uint8_t *M, const eaga_weights *w, void *Xout, void *Eout, void *saved,
                                 void *workspace, size_t ws_bytes, void *stream) {
    return forward_impl(d, variant, 0, -1, X, E, y, M, w, Xout, Eout, saved, workspace, ws_bytes, stream);
}

eaga_status eaga_forward_rows(const eaga_dims *d, int variant, int row0, int rows, const void *X, const void *E_rows,
                              const void *y, const uint8_t *M, const eaga_weights *w, void *Xout, void *Eout_rows,
                              void *saved, void *workspace, size_t ws_bytes, void *stream) {
    if (rows < 0) return EAGA_ERR_INVALID_ARG;
    return forward_impl(d, variant, row0, rows, X, E_rows, y, M, w, Xout, Eout_rows, saved, workspace, ws_bytes,
                        stream);
}

eaga_status eaga_forward(const eaga_dims *d, const void *X, const void *E, const void *y, const uint8_t *M,
                         const eaga_weights *w, void *Xout, void *Eout, void *saved, void *workspace,
                         size_t ws_bytes, void *stream) {
    return eaga_forward_variant(d, EAGA_VARIANT_LAYER, X, E, y, M, w, Xout, Eout, saved, workspace, ws_bytes,
                                stream);
}

static eaga_status backward_impl(const eaga_dims *d, int variant, int row0, int rows, const void *X, const void *E,
                                 const void *y, const uint8_t *M, const eaga_weights *w, const void *saved,
                                 const void *dXout, const void *dEout, void *dX, void *dE, void *dy,
                                 const eaga_weight_grads *dW, void *workspace, size_t ws_bytes, void *stream,
                                 bool clear_status = true) {
    NvtxRange range("eaga_backward");
    eaga_status s = check_dims(d);
    if (s != EAGA_OK) return s;
    if (!known_variant(variant)) return EAGA_ERR_INVALID_ARG;
    if ((s = check_slab(*d, row0, rows)) != EAGA_OK) return s;
    if ((s = check_weights(w)) != EAGA_OK) return s;
    if ((s = check_ptrs({X, E, y, M, saved, dXout, dEout, dX, dE, dy, workspace})) != EAGA_OK) return s;
    if (!dW) return EAGA_ERR_INVALID_ARG;
    if ((s = check_ptrs({dW->Wq, dW->bq, dW->Wk, dW->bk, dW->Wv, dW->bv, dW->Wfe, dW->Wfy, dW->bf, dW->We, dW->Wo,
                         dW->bo})) != EAGA_OK)
        return s;
    const Layout L = saved_layout(*d);
    {
        const Extents x = tensor_extents(*d);
        const size_t xe = slab_bytes(*d, rows);
        Span outs[16] = {{dX, x.X}, {dE, xe}, {dy, x.y}, {workspace, eaga_workspace_size(d, 1)}};
        const void *gsrc[12] = {dW->Wq, dW->bq, dW->Wk, dW->bk, dW->Wv, dW->bv,
                                dW->Wfe, dW->Wfy, dW->bf, dW->We, dW->Wo, dW->bo};
        weight_spans(gsrc, x.wgrad, outs, 4);
        Span ins[19] = {{X, x.X}, {E, xe}, {y, x.y}, {M, x.M}, {saved, L.saved_total}, {dXout, x.X}, {dEout, xe}};
        const void *wsrc[12];
        weight_array(w, wsrc);
        weight_spans(wsrc, x.w, ins, 7);
        if ((s = check_no_alias(outs, 16, ins, 19)) != EAGA_OK) return s;
    }
    if (ws_bytes < eaga_workspace_size(d, 1)) return EAGA_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const WsLayout W = ws_layout(*d);
    char *ws = static_cast<char *>(workspace);
    const char *sv = static_cast<const char *>(saved);
    BwdArgs a;
    a.variant = variant;
    a.row0 = rows < 0 ? 0 : row0;
    a.rows = rows;
    a.X = X; a.E = E; a.y = y; a.M = M;
    weight_array(w, a.w);
    a.Q = sv + L.q; a.K = sv + L.k; a.V = sv + L.v; a.O = sv + L.o;
    a.LSE = reinterpret_cast<const float *>(sv + L.lse);
    a.dXout = dXout; a.dEout = dEout;
    a.dX = dX; a.dE = dE; a.dy = dy;
    void *gsrc[12] = {dW->Wq, dW->bq, dW->Wk, dW->bk, dW->Wv, dW->bv, dW->Wfe, dW->Wfy, dW->bf, dW->We, dW->Wo, dW->bo};
    for (int t = 0; t < 12; ++t) a.dW[t] = static_cast<float *>(gsrc[t]);
    a.g = reinterpret_cast<float *>(ws + W.g);
    a.dO = reinterpret_cast<float *>(ws + W.dO);
    a.dQ = reinterpret_cast<float *>(ws + W.dQ);
    a.dK = reinterpret_cast<float *>(ws + W.dK);
    a.dV = reinterpret_cast<float *>(ws + W.dV);
    a.D = reinterpret_cast<float *>(ws + W.D);
    a.parts = reinterpret_cast<float *>(ws + W.parts);
    a.dg = reinterpret_cast<float *>(ws + W.dg);
    a.part_stride = W.part_stride;
    a.status = reinterpret_cast<int *>(ws + W.status);
    if (clear_status && cudaMemsetAsync(a.status, 0, sizeof(int), st) != cudaSuccess) return EAGA_ERR_CUDA;
    if (fast::supports(*d)) {
        return launch_status(fast::backward(*d, a, ws, W.fwd_saved, st));
    }
    return launch_status(generic::backward(*d, a, st));
}

eaga_status eaga_backward_variant(const eaga_dims *d, int variant, const void *X, const void *E, const void *y,
                                  const uint8_t *M, const eaga_weights *w, const void *saved, const void *dXout,
                                  const void *dEout, void *dX, void *dE, void *dy, const eaga_weight_grads *dW,
                                  void *workspace, size_t ws_bytes, void *stream) {
    return backward_impl(d, variant, 0, -1, X, E, y, M, w, saved, dXout, dEout, dX, dE, dy, dW, workspace, ws_bytes,
                         stream);
}

eaga_status eaga_backward_rows(const eaga_dims *d, int variant, int row0, int rows, const void *X, const void *E_rows,
                               const void *y, const uint8_t *M, const eaga_weights *w, const void *saved,
                               const void *dXout, const void *dEout_rows, void *dX, void *dE_rows, void *dy,
                               const eaga_weight_grads *dW, void *workspace, size_t ws_bytes, void *stream) {
    if (rows < 0) return EAGA_ERR_INVALID_ARG;
    return backward_impl(d, variant, row0, rows, X, E_rows, y, M, w, saved, dXout, dEout_rows, dX, dE_rows, dy, dW,
                         workspace, ws_bytes, stream);
}

eaga_status eaga_backward(const eaga_dims *d, const void *X, const void *E, const void *y, const uint8_t *M,
                          const eaga_weights *w, const void *saved, const void *dXout, const void *dEout,
                          void *dX, void *dE, void *dy, const eaga_weight_grads *dW, void *workspace,
                          size_t ws_bytes, void *stream) {
    return eaga_backward_variant(d, EAGA_VARIANT_LAYER, X, E, y, M, w, saved, dXout, dEout, dX, dE, dy, dW,
                                 workspace, ws_bytes, stream);
}

// ------------------------------------------------------------------ the block around the layer

static eaga_status check_block_dims(const eaga_dims *d) {
    eaga_status s = check_dims(d);
    if (s != EAGA_OK) return s;
    if (!fast::supports(*d) || !fast::blk::block_supports(d->dx, d->de, d->dy)) return EAGA_ERR_UNSUPPORTED;
    return EAGA_OK;
}
static size_t layer_saved_bytes(const eaga_dims &d) { return align256(saved_layout(d).saved_total); }

size_t eaga_block_saved_size(const eaga_dims *d) {
    if (check_block_dims(d) != EAGA_OK) return 0;
    return fast::blk::block_saved_layout(d->B, d->n, d->dx, d->dy, layer_saved_bytes(*d)).total;
}

size_t eaga_block_workspace_size(const eaga_dims *d, int for_backward) {
    if (check_block_dims(d) != EAGA_OK) return 0;
    const size_t base = align256(eaga_workspace_size(d, for_backward ? 1 : 0));
    return fast::blk::block_ws_layout(d->B, d->n, d->dx, d->dy, base, for_backward).total;
}

int eaga_block_kernel_launches(const eaga_dims *d, int for_backward) {
    if (check_block_dims(d) != EAGA_OK) return -1;
    return eaga_kernel_launches(d, for_backward) + fast::blk::block_kernel_launches(for_backward);
}

static eaga_status check_block_weights(const eaga_block_weights *wb, const void *out[27]) {
    if (!wb) return EAGA_ERR_INVALID_ARG;
    const void *src[27] = {wb->x_ln1_g, wb->x_ln1_s, wb->x_W1, wb->x_b1, wb->x_W2, wb->x_b2, wb->x_ln2_g,
                           wb->x_ln2_s, wb->e_ln1_g, wb->e_ln1_s, wb->e_W1, wb->e_b1, wb->e_W2, wb->e_b2,
                           wb->e_ln2_g, wb->e_ln2_s, wb->y_ln1_g, wb->y_ln1_s, wb->y_W1, wb->y_b1, wb->y_W2,
                           wb->y_b2, wb->y_ln2_g, wb->y_ln2_s, wb->Wyx, wb->Wye, wb->by};
    for (int k = 0; k < 27; ++k) {
        if (!src[k]) return EAGA_ERR_INVALID_ARG;
        if (!aligned16(src[k])) return EAGA_ERR_MISALIGNED;
        out[k] = src[k];
    }
    return EAGA_OK;
}

eaga_status eaga_block_forward(const eaga_dims *d, const void *X, const void *E, const void *y, const uint8_t *M,
                               const eaga_weights *w, const eaga_block_weights *wb, void *Xmid, void *Emid,
                               void *Xout, void *Eout, void *yout, void *saved, void *workspace, size_t ws_bytes,
                               void *stream) {
    NvtxRange range("eaga_block_forward");
    eaga_status s = check_block_dims(d);
    if (s != EAGA_OK) return s;
    const void *wbs[27];
    if ((s = check_block_weights(wb, wbs)) != EAGA_OK) return s;
    if ((s = check_ptrs({Xout, Eout, yout, saved, workspace})) != EAGA_OK) return s;
    if (ws_bytes < eaga_block_workspace_size(d, 0)) return EAGA_ERR_WORKSPACE;
    const fast::blk::BlockSaved S =
        fast::blk::block_saved_layout(d->B, d->n, d->dx, d->dy, layer_saved_bytes(*d));
    {
        const Extents x = tensor_extents(*d);
        const Span outs[4] = {{Xout, x.X}, {Eout, x.E}, {yout, x.y}, {saved, S.total}};
        const Span ins[7] = {{X, x.X}, {E, x.E}, {y, x.y}, {M, x.M}, {Xmid, x.X}, {Emid, x.E},
                             {workspace, eaga_block_workspace_size(d, 0)}};
        if ((s = check_no_alias(outs, 4, ins, 7)) != EAGA_OK) return s;
    }
    const size_t base = align256(eaga_workspace_size(d, 0));
    s = forward_impl(d, EAGA_VARIANT_LAYER, 0, -1, X, E, y, M, w, Xmid, Emid, saved, workspace, base, stream);
    if (s != EAGA_OK) return s;
    const fast::blk::BlockWs W = fast::blk::block_ws_layout(d->B, d->n, d->dx, d->dy, base, 0);
    char *ws = static_cast<char *>(workspace);
    fast::blk::TailFwd a = {};
    a.B = d->B; a.n = d->n; a.dx = d->dx; a.dy = d->dy;
    a.M = M; a.y = y; a.Xmid = Xmid; a.Emid = Emid; a.wb = wbs;
    a.Xout = Xout; a.Eout = Eout; a.yout = yout;
    a.status = reinterpret_cast<int *>(ws + ws_layout(*d).status);
    return launch_status(
        fast::blk::tail_forward(a, ws, W, static_cast<char *>(saved), S, static_cast<cudaStream_t>(stream)));
}

eaga_status eaga_block_backward(const eaga_dims *d, const void *X, const void *E, const void *y, const uint8_t *M,
                                const eaga_weights *w, const eaga_block_weights *wb, const void *Xmid,
                                const void *Emid, const void *saved, const void *dXout, const void *dEout,
                                const void *dyout, void *dEmid, void *dX, void *dE, void *dy,
                                const eaga_weight_grads *dW, const eaga_block_grads *dWb, void *workspace,
                                size_t ws_bytes, void *stream) {
    NvtxRange range("eaga_block_backward");
    eaga_status s = check_block_dims(d);
    if (s != EAGA_OK) return s;
    const void *wbs[27];
    if ((s = check_block_weights(wb, wbs)) != EAGA_OK) return s;
    if ((s = check_ptrs({Xmid, Emid, saved, dXout, dEout, dyout, dEmid, workspace})) != EAGA_OK) return s;
    if (!dWb) return EAGA_ERR_INVALID_ARG;
    float *dwb[27];
    {
        void *src[27] = {dWb->x_ln1_g, dWb->x_ln1_s, dWb->x_W1, dWb->x_b1, dWb->x_W2, dWb->x_b2, dWb->x_ln2_g,
                         dWb->x_ln2_s, dWb->e_ln1_g, dWb->e_ln1_s, dWb->e_W1, dWb->e_b1, dWb->e_W2, dWb->e_b2,
                         dWb->e_ln2_g, dWb->e_ln2_s, dWb->y_ln1_g, dWb->y_ln1_s, dWb->y_W1, dWb->y_b1, dWb->y_W2,
                         dWb->y_b2, dWb->y_ln2_g, dWb->y_ln2_s, dWb->Wyx, dWb->Wye, dWb->by};
        for (int k = 0; k < 27; ++k) {
            if (!src[k]) return EAGA_ERR_INVALID_ARG;
            if (!aligned16(src[k])) return EAGA_ERR_MISALIGNED;
            dwb[k] = static_cast<float *>(src[k]);
        }
    }
    if (ws_bytes < eaga_block_workspace_size(d, 1)) return EAGA_ERR_WORKSPACE;
    {
        const Extents x = tensor_extents(*d);
        const Span outs[2] = {{dEmid, x.E}, {workspace, eaga_block_workspace_size(d, 1)}};
        const Span ins[11] = {{X, x.X}, {E, x.E}, {y, x.y}, {M, x.M}, {Xmid, x.X}, {Emid, x.E},
                              {saved, eaga_block_saved_size(d)}, {dXout, x.X}, {dEout, x.E}, {dyout, x.y},
                              {dE, x.E}};
        if ((s = check_no_alias(outs, 2, ins, 11)) != EAGA_OK) return s;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t base = align256(eaga_workspace_size(d, 1));
    const fast::blk::BlockWs W = fast::blk::block_ws_layout(d->B, d->n, d->dx, d->dy, base, 1);
    const fast::blk::BlockSaved S =
        fast::blk::block_saved_layout(d->B, d->n, d->dx, d->dy, layer_saved_bytes(*d));
    char *ws = static_cast<char *>(workspace);
    int *status = reinterpret_cast<int *>(ws + ws_layout(*d).status);
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return EAGA_ERR_CUDA;
    fast::blk::TailBwd a = {};
    a.B = d->B; a.n = d->n; a.dx = d->dx; a.dy = d->dy;
    a.M = M; a.Xmid = Xmid; a.Emid = Emid; a.dXout = dXout; a.dEout = dEout; a.dyout = dyout;
    a.wb = wbs; a.dwb = dwb; a.dEmid = dEmid; a.status = status;
    if ((s = launch_status(fast::blk::tail_backward(a, ws, W, static_cast<const char *>(saved), S, st))) != EAGA_OK)
        return s;
    s = backward_impl(d, EAGA_VARIANT_LAYER, 0, -1, X, E, y, M, w, saved, ws + W.dXmid, dEmid, dX, dE, dy, dW,
                      workspace, base, stream, false);
    if (s != EAGA_OK) return s;
    return launch_status(fast::blk::add_dy(dy, reinterpret_cast<const float *>(ws + W.dy1), d->B * d->dy, st));
}

eaga_status eaga_debug_attention_map(const eaga_dims *d, const void *E, const uint8_t *M, const eaga_weights *w,
                                     const void *y, const void *saved, float *A, void *stream) {
    eaga_status s = check_dims(d);
    if (s != EAGA_OK) return s;
    if ((s = check_weights(w)) != EAGA_OK) return s;
    if ((s = check_ptrs({E, M, y, saved, A})) != EAGA_OK) return s;
    // g [B,2H] lives just past the A map the caller provides room for.
    const Layout L = saved_layout(*d);
    {
        const Extents x = tensor_extents(*d);
        const Span outs[1] = {{A, ((size_t)d->B * d->H * d->n * d->n + 2 * (size_t)d->B * d->H) * sizeof(float)}};
        Span ins[16] = {{E, x.E}, {M, x.M}, {y, x.y}, {saved, L.saved_total}};
        const void *wsrc[12];
        weight_array(w, wsrc);
        weight_spans(wsrc, x.w, ins, 4);
        if ((s = check_no_alias(outs, 1, ins, 16)) != EAGA_OK) return s;
    }
    const char *sv = static_cast<const char *>(saved);
    MapArgs a;
    a.E = E; a.y = y; a.Wfe = w->Wfe; a.Wfy = w->Wfy; a.bf = w->bf; a.M = M;
    a.Q = sv + L.q; a.K = sv + L.k;
    a.LSE = reinterpret_cast<const float *>(sv + L.lse);
    a.A = A;
    a.g = A + (size_t)d->B * d->H * d->n * d->n;
    return launch_status(generic::attention_map(*d, a, static_cast<cudaStream_t>(stream)));
}

// One thread waits, with the pair kernels' bounded poll loop, on phase 0 of an
// mbarrier that expects one arrival nobody makes.
__global__ void k_wait_probe(int *status, unsigned limit) {
    __shared__ __align__(8) unsigned long long bar;
    const uint32_t b = sm100::smem_u32(&bar);
    if (threadIdx.x == 0) {
        sm100::mbar_init(b, 1);
        sm100::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !sm100::mbar_wait(b, 0, limit)) atomicExch(status, DEV_TIMEOUT);
}

// The status word a call reports through: the workspace's first int, or, for
// workspace == NULL, that of the no-allocation forward's fixed scratch array
// on the current device.
static eaga_status status_word(void *workspace, int **out) {
    if (workspace) {
        if (reinterpret_cast<uintptr_t>(workspace) & 15u) return EAGA_ERR_MISALIGNED;
        *out = static_cast<int *>(workspace);
        return EAGA_OK;
    }
    void *base = nullptr;
    const eaga_status s = noalloc_scratch_address(&base);
    *out = static_cast<int *>(base);
    return s;
}

eaga_status eaga_debug_wait_probe(void *workspace, unsigned limit, void *stream) {
    if (limit < 1 || limit > (1u << 24)) return EAGA_ERR_INVALID_ARG;
    int *word = nullptr;
    const eaga_status s = status_word(workspace, &word);
    if (s != EAGA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    k_wait_probe<<<1, 32, 0, st>>>(word, limit);
    return cudaGetLastError() == cudaSuccess ? EAGA_OK : EAGA_ERR_CUDA;
}

eaga_status eaga_get_device_status(void *workspace, void *stream) {
    int *word = nullptr;
    const eaga_status s = status_word(workspace, &word);
    if (s != EAGA_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int h = 0;
    if (cudaMemcpyAsync(&h, word, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return EAGA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EAGA_ERR_CUDA;
    if (cudaMemsetAsync(word, 0, sizeof(int), st) != cudaSuccess) return EAGA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return EAGA_ERR_CUDA;
    return h == DEV_OK ? EAGA_OK : EAGA_ERR_TIMEOUT;
}

eaga_status eaga_set_profile_events(int point, void *before, void *after) {
    if (point < 0 || point > 4) return EAGA_ERR_INVALID_ARG;
    if ((before == nullptr) != (after == nullptr)) return EAGA_ERR_INVALID_ARG;
    g_prof_events[point][0].store(before, std::memory_order_release);
    g_prof_events[point][1].store(after, std::memory_order_release);
    return EAGA_OK;
}

int eaga_kernel_launches(const eaga_dims *d, int for_backward) {
    if (check_dims(d) != EAGA_OK) return -1;
    if (fast::supports(*d)) return fast::kernel_launches(*d, for_backward);
    return generic::kernel_launches(*d, for_backward);
}

const char *eaga_strerror(eaga_status s) {
    switch (s) {
    case EAGA_OK: return "ok";
    case EAGA_ERR_INVALID_ARG: return "invalid argument";
    case EAGA_ERR_UNSUPPORTED: return "unsupported dims";
    case EAGA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case EAGA_ERR_WORKSPACE: return "workspace too small";
    case EAGA_ERR_CUDA: return "CUDA error";
    case EAGA_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

}  // extern "C"
