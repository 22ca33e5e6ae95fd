// Host glue of the specialised sm_100a path (de = 64, H = 8, dh = 32, bf16):
// which dims it covers, its workspace, its launch sequence and launch count.
#include <mutex>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

cudaError_t launch_prologue(const eaga_dims &d, const void *const w[12], const void *y, float *g, uint8_t *img,
                            int *zero, int nzero, cudaStream_t st);
cudaError_t tc_gemm(int mode, int M, int N, int K, int nseg, const void *const A[3], const void *const B[3],
                    const void *const bias[3], void *const C[3], int Nb, const void *R, const uint8_t *mask,
                    int *status, cudaStream_t st, bool b_mn);
cudaError_t launch_fwd_pairs(const eaga_dims &d, const FwdArgs &a, const uint8_t *img, const int *order, const float *g,
                             cudaStream_t st);
cudaError_t tc_wgrad(int M, int Nb, int nout, int K, int splits, const void *A, const void *const B[3],
                     float *const P[3], int *status, cudaStream_t st);
cudaError_t launch_bwd_pairs(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                             cudaStream_t st);
cudaError_t launch_kv_convert(const eaga_dims &d, const FastWs &W, char *ws, cudaStream_t st);
cudaError_t launch_row_block_order(const eaga_dims &d, const uint8_t *M, int row0, int rows, int *order,
                                   cudaStream_t st);
cudaError_t launch_bwd_partials(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, cudaStream_t st);
cudaError_t launch_film_grads(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, cudaStream_t st);
cudaError_t launch_bwd_final(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, int part,
                             cudaStream_t st);

bool supports(const eaga_dims &d) {
    return d.dtype == EAGA_BF16 && d.de == DE && d.H == NH && d.dh == DH && d.n % 2 == 0 && d.n >= 2 &&
           d.n <= 1024 && d.dx % 64 == 0 && d.dx >= 64;
}

// Forward: the small operand images after the common workspace; backward:
// the whole FastWs.
// (the operand images, then the order of the row blocks for the pair kernel)
size_t forward_scratch_bytes(const eaga_dims &d, bool with_order) {
    return align256(IMG_BYTES) + (with_order ? align256(size_t(row_blocks(d)) * 4) : 0);
}
size_t workspace_size(const eaga_dims &d, int for_backward, size_t common_fwd, size_t common_head) {
    if (!for_backward) return align256(common_fwd) + forward_scratch_bytes(d);
    return fast_ws(d, common_head).total;
}

int kernel_launches(const eaga_dims &, int for_backward) {
    // forward: prologue, row-block order, QKV, pairs, out-proj
    // backward: prologue, dO, row-block order, pairs, dk/dv conversion, dX, wgrad x2, bias and
    // row-block partials, finish x2, film grads
    return for_backward ? 12 : 5;
}

#define FAST_TRY(x)                               \
    do {                                          \
        cudaError_t e_ = (x);                     \
        if (e_ != cudaSuccess) return e_;         \
    } while (0)

// Two auxiliary streams and a pool of events per device, created on first
// use: the forward and the backward run independent kernels side by side
// (fork / join on events), which a CUDA graph captured around the call keeps
// as parallel branches.  The lock is held while a call enqueues, so concurrent calls on
// one device never share an event between a record and its wait.
namespace {
constexpr int kMaxDevices = 64, kEvents = 16, kStreams = 3;
struct DeviceAux {
    std::mutex mu;
    bool ready = false;
    cudaStream_t s[kStreams] = {};
    cudaEvent_t ev[kEvents] = {};
};
DeviceAux g_aux[kMaxDevices];

cudaError_t device_aux(DeviceAux **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    *out = &g_aux[dev];
    return cudaSuccess;
}

cudaError_t aux_init(DeviceAux &x) {   // called with x.mu held
    if (x.ready) return cudaSuccess;
    cudaError_t e;
    for (int k = 0; k < kStreams; ++k)
        if ((e = cudaStreamCreateWithFlags(&x.s[k], cudaStreamNonBlocking)) != cudaSuccess) return e;
    for (int k = 0; k < kEvents; ++k)
        if ((e = cudaEventCreateWithFlags(&x.ev[k], cudaEventDisableTiming)) != cudaSuccess) return e;
    x.ready = true;
    return cudaSuccess;
}

// `to` waits for everything enqueued on `from` so far
cudaError_t stream_after(cudaStream_t to, cudaStream_t from, cudaEvent_t ev) {
    cudaError_t e = cudaEventRecord(ev, from);
    return e == cudaSuccess ? cudaStreamWaitEvent(to, ev, 0) : e;
}
}  // namespace

cudaError_t forward(const eaga_dims &d, const FwdArgs &a, char *ws_after_common, cudaStream_t st,
                    bool with_order) {
    uint8_t *img = reinterpret_cast<uint8_t *>(ws_after_common);
    int *order = with_order ? reinterpret_cast<int *>(ws_after_common + align256(IMG_BYTES)) : nullptr;
    const int rows = d.B * d.n;
    DeviceAux *aux = nullptr;
    FAST_TRY(device_aux(&aux));
    std::lock_guard<std::mutex> lock(aux->mu);
    FAST_TRY(aux_init(*aux));
    // the prologue (g, operand images) and the order of the row blocks for the
    // pair kernel (longest first) beside the QKV projection, each on a stream
    // of its own
    FAST_TRY(stream_after(aux->s[0], st, aux->ev[0]));
    FAST_TRY(launch_prologue(d, a.w, a.y, a.g, img, nullptr, 0, aux->s[0]));
    if (order) {
        FAST_TRY(stream_after(aux->s[1], st, aux->ev[2]));
        FAST_TRY(launch_row_block_order(d, a.M, a.row0, a.rows < 0 ? d.n : a.rows, order, aux->s[1]));
    }
    {   // [Q|K|V] = X [Wq|Wk|Wv] + b
        const void *A[3] = {a.X, a.X, a.X}, *B[3] = {a.w[0], a.w[2], a.w[4]};
        const void *bias[3] = {a.w[1], a.w[3], a.w[5]};
        void *C[3] = {a.Q, a.K, a.V};
        FAST_TRY(tc_gemm(0, rows, 3 * HD, d.dx, 1, A, B, bias, C, HD, nullptr, a.M, a.status, st, true));
    }
    FAST_TRY(stream_after(st, aux->s[0], aux->ev[1]));
    if (order) FAST_TRY(stream_after(st, aux->s[1], aux->ev[3]));
    // a slab of rows: O of the rows outside it is zero (the out-projection and,
    // in the backward, dWo read every row)
    if (a.rows >= 0 && a.rows < d.n) FAST_TRY(cudaMemsetAsync(a.O, 0, (size_t)rows * HD * 2, st));
    prof_mark(0, 0, st);
    FAST_TRY(launch_fwd_pairs(d, a, img, order, a.g, st));
    prof_mark(0, 1, st);
    {   // X' = X + M (O Wo + bo)
        const void *A[3] = {a.O, a.O, a.O}, *B[3] = {a.w[10], a.w[10], a.w[10]};
        const void *bias[3] = {a.w[11], a.w[11], a.w[11]};
        void *C[3] = {a.Xout, a.Xout, a.Xout};
        FAST_TRY(tc_gemm(1, rows, d.dx, HD, 1, A, B, bias, C, d.dx, a.X, a.M, a.status, st, true));
    }
    return cudaSuccess;
}

cudaError_t with_side_streams(const std::function<cudaError_t(const cudaStream_t *, const cudaEvent_t *)> &enqueue) {
    DeviceAux *aux = nullptr;
    FAST_TRY(device_aux(&aux));
    std::lock_guard<std::mutex> lock(aux->mu);
    FAST_TRY(aux_init(*aux));
    return enqueue(aux->s, aux->ev + 11);   // events 11..15 are the caller's
}

cudaError_t backward(const eaga_dims &d, const BwdArgs &a, char *ws, size_t head, cudaStream_t st) {
    const FastWs W = fast_ws(d, head);
    uint8_t *img = reinterpret_cast<uint8_t *>(ws + W.img);
    __nv_bfloat16 *dO = reinterpret_cast<__nv_bfloat16 *>(ws + W.dO);
    const int rows = d.B * d.n;
    DeviceAux *aux = nullptr;
    FAST_TRY(device_aux(&aux));
    std::lock_guard<std::mutex> lock(aux->mu);
    FAST_TRY(aux_init(*aux));
    cudaStream_t s1 = aux->s[0], s2 = aux->s[1], s3 = aux->s[2];
    cudaEvent_t *ev = aux->ev;

    // prologue (g, operand images) beside dO = M (dX' Wo^T)
    FAST_TRY(stream_after(s1, st, ev[0]));
    {
        const void *A[3] = {a.dXout, a.dXout, a.dXout}, *Bt[3] = {a.w[10], a.w[10], a.w[10]};
        void *C[3] = {dO, dO, dO};
        FAST_TRY(tc_gemm(2, rows, HD, d.dx, 1, A, Bt, nullptr, C, HD, nullptr, a.M, a.status, s1, false));
    }
    // the dk, dv accumulators start at zero (beside dO on the auxiliary stream)
    FAST_TRY(cudaMemsetAsync(ws + W.dK32, 0, (size_t)rows * HD * 4 * 2, s1));
    if (a.rows >= 0 && a.rows < d.n) {   // a slab of rows: dq and the row-block partials of the other rows are zero
        FAST_TRY(cudaMemsetAsync(ws + W.dQ, 0, (size_t)rows * HD * 2, s1));
        FAST_TRY(cudaMemsetAsync(ws + W.rparts, 0, (size_t)W.n_rparts * RPART * 4, s1));
    }
    // the order of the row blocks for the pair kernel (longest first) on a
    // third stream and the prologue, beside dO
    FAST_TRY(stream_after(s3, st, ev[9]));
    FAST_TRY(launch_row_block_order(d, a.M, a.row0, a.rows < 0 ? d.n : a.rows, reinterpret_cast<int *>(ws + W.order),
                                    s3));
    FAST_TRY(launch_prologue(d, a.w, a.y, a.g, img, nullptr, 0, st));
    FAST_TRY(stream_after(st, s1, ev[1]));
    FAST_TRY(stream_after(st, s3, ev[10]));

    prof_mark(1, 0, st);
    FAST_TRY(launch_bwd_pairs(d, a, W, ws, a.g, st));
    prof_mark(1, 1, st);
    FAST_TRY(launch_kv_convert(d, W, ws, st));

    // dX, the weight-gradient partials and the reductions' first level side by side
    const __nv_bfloat16 *dN[3] = {reinterpret_cast<const __nv_bfloat16 *>(ws + W.dQ),
                                  reinterpret_cast<const __nv_bfloat16 *>(ws + W.dK),
                                  reinterpret_cast<const __nv_bfloat16 *>(ws + W.dV)};
    FAST_TRY(stream_after(s1, st, ev[2]));
    FAST_TRY(stream_after(s2, st, ev[3]));
    FAST_TRY(stream_after(s3, st, ev[6]));
    {   // dX = dX' + dQ Wq^T + dK Wk^T + dV Wv^T
        const void *A[3] = {dN[0], dN[1], dN[2]}, *Bt[3] = {a.w[0], a.w[2], a.w[4]};
        void *C[3] = {a.dX, a.dX, a.dX};
        FAST_TRY(tc_gemm(3, rows, d.dx, HD, 3, A, Bt, nullptr, C, d.dx, a.dXout, a.M, a.status, st, false));
    }
    {   // split-K partials of dW{q,k,v} = X^T d{Q,K,V} and dWo = O^T dX' (O is zero on masked rows)
        float *parts = reinterpret_cast<float *>(ws + W.wparts);
        const size_t msz = (size_t)W.wsplits * d.dx * HD;
        const void *Bq[3] = {dN[0], dN[1], dN[2]}, *Bo[3] = {a.dXout, a.dXout, a.dXout};
        float *const Pq[3] = {parts, parts + msz, parts + 2 * msz}, *const Po[3] = {parts + 3 * msz, nullptr, nullptr};
        // dW{q,k,v} and their final sums on one auxiliary stream; dWo, the
        // bias and row-block partials and the rest of the sums on the other
        FAST_TRY(tc_wgrad(d.dx, HD, 3, rows, W.wsplits, a.X, Bq, Pq, a.status, s1));
        FAST_TRY(launch_bwd_final(d, a, W, ws, 0, s1));
        FAST_TRY(tc_wgrad(HD, d.dx, 1, rows, W.wsplits, a.O, Bo, Po, a.status, s2));
    }
    // the bias and row-block partials beside dWo (they do not need it), then
    // dbf, dWfy, dy from dg beside the final sums of the rest
    FAST_TRY(launch_bwd_partials(d, a, W, ws, s3));
    FAST_TRY(stream_after(s2, s3, ev[7]));
    FAST_TRY(launch_film_grads(d, a, W, ws, s3));
    FAST_TRY(launch_bwd_final(d, a, W, ws, 1, s2));
    FAST_TRY(stream_after(st, s1, ev[4]));
    FAST_TRY(stream_after(st, s2, ev[5]));
    FAST_TRY(stream_after(st, s3, ev[8]));
    return cudaSuccess;
}

}  // namespace fast
}  // namespace eaga
