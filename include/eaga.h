/*
 * eaga.h — C ABI of the edge-aware graph attention layer (libeaga.so).
 *
 * The layer is the FlexAttentionGT edge-aware attention layer of "Efficient
 * Edge-aware Attention Network for Graph Generation": per-head scaled
 * dot-product attention over the nodes of dense padded graphs, whose scores
 * are modulated head-wise by a FiLM of the edge features E_ij and the graph's
 * global features y (AI-summary page, method paragraph; blog summary, "Design
 * Strategy of the Edge-aware Attention Layer"), restricted to real nodes by
 * the node mask, returning both the node aggregation and the normalised
 * attention coefficients in one pass, followed by a residual edge update from
 * those coefficients and a residual node update (AI-summary page, method
 * paragraph).  Per graph b, node i, j, head h:
 *
 *   Q,K,V   = X W{q,k,v} + b{q,k,v}                 head h = cols h*dh..h*dh+dh-1
 *   g_b     = y_b Wfy + bf                           [2H]
 *   f_bij   = E_bij Wfe + g_b;  gamma = f[h], beta = f[H+h]
 *   s'_ij   = (q_i . k_j / sqrt(dh)) (1 + gamma) + beta
 *   a_ij    = softmax over valid j of s'_ij          (valid: M_bi and M_bj; else 0)
 *   O_ih    = sum_j a_ij v_jh
 *   E'_bij  = E_bij + sum_h a^h_ij We[h,:]
 *   X'_bi   = X_bi + M_bi (O_bi Wo + bo)
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays,
 *     owned by the caller; the library never allocates device memory.
 *   - Storage dtype (dims.dtype) applies to X, E, y, weights, outputs X', E',
 *     the gradients dX, dE, dy, dX', dE' and the saved Q,K,V,O.  Arithmetic
 *     accumulates in fp32 in both modes.  Weight gradients are always fp32.
 *   - M is uint8 [B,n] with values 0/1 (any pattern, not only a prefix).
 *   - Weights are [in, out] (Y = X W): Wq,Wk,Wv [dx, H*dh]; bq,bk,bv [H*dh];
 *     Wfe [de, 2H]; Wfy [dy, 2H]; bf [2H] (first H columns gamma, next H
 *     beta); We [H, de] (no bias); Wo [H*dh, dx]; bo [dx].
 *   - Shapes: X, X', dX, dX' [B,n,dx]; E, E', dE, dE' [B,n,n,de]; y, dy [B,dy].
 *   - Every pointer must be 16-byte aligned (else EAGA_ERR_MISALIGNED).
 *     Outputs (including `saved` in the forward and the workspace) must not
 *     overlap an input or another output: the byte range of every buffer
 *     follows from the dims, and an overlap returns EAGA_ERR_INVALID_ARG
 *     before anything is launched.  Inputs may share memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  The return value reports host-side validation and
 *     launch errors only; device-side conditions (a bounded wait that ran out)
 *     are recorded in the workspace status word and read by
 *     eaga_get_device_status.
 *   - No global state besides per-device cached kernel attributes, the
 *     per-device auxiliary streams of the specialised path and the optional
 *     profiling events; calls on distinct streams with distinct workspaces
 *     are thread-safe, also across devices of one process.
 */
#ifndef EAGA_H
#define EAGA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define EAGA_API __attribute__((visibility("default")))
#else
#define EAGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EAGA_OK = 0,
    EAGA_ERR_INVALID_ARG = 1,   /* null pointer, non-positive dim, bad dtype */
    EAGA_ERR_UNSUPPORTED = 2,   /* dims outside the supported limits below */
    EAGA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    EAGA_ERR_WORKSPACE = 4,     /* workspace smaller than eaga_workspace_size() */
    EAGA_ERR_CUDA = 5,          /* a CUDA launch or runtime call failed */
    EAGA_ERR_TIMEOUT = 6        /* device-side bounded wait ran out (status word) */
} eaga_status;

typedef enum { EAGA_FP32 = 0, EAGA_BF16 = 1 } eaga_dtype;

/* Problem dims.  Limits: 1 <= n <= 1024; H*dh <= 256 and dh % 8 == 0;
 * de % 8 == 0, de <= 128; dx % 8 == 0, dx <= 1024; dy % 8 == 0, dy <= 1024;
 * 2*H <= 32; H*n <= 8192.  Anything else returns EAGA_ERR_UNSUPPORTED. */
typedef struct {
    int B, n, dx, de, dy, H, dh;
    int dtype;                  /* eaga_dtype */
} eaga_dims;

typedef struct {
    const void *Wq, *bq, *Wk, *bk, *Wv, *bv, *Wfe, *Wfy, *bf, *We, *Wo, *bo;
} eaga_weights;

/* fp32 weight gradients, same shapes as the weights; overwritten, not accumulated. */
typedef struct {
    void *Wq, *bq, *Wk, *bk, *Wv, *bv, *Wfe, *Wfy, *bf, *We, *Wo, *bo;
} eaga_weight_grads;

/* Bytes of workspace eaga_forward (for_backward = 0) or eaga_backward
 * (for_backward = 1) needs.  Both grow with the node count only: O(B*n*H*dh)
 * + O(B*H*n) + fixed-size partial sums, never a per-pair (B*H*n^2) term; no
 * attention coefficient of any pair is stored in memory.
 * Returns 0 for invalid or unsupported dims. */
EAGA_API size_t eaga_workspace_size(const eaga_dims *dims, int for_backward);

/* Bytes of the forward's saved state that eaga_backward consumes:
 * LSE [B,H,n] fp32, then Q, K, V, O [B,n,H*dh] in the storage dtype, each
 * region 256-byte aligned.  Returns 0 for invalid or unsupported dims. */
EAGA_API size_t eaga_saved_size(const eaga_dims *dims);

/* Forward of the layer (the formulas above).  Writes Xout and Eout.  `saved`
 * (nullable; eaga_saved_size bytes) receives the state eaga_backward needs;
 * with saved == NULL that state lives in the workspace and is discarded.
 * `workspace` must hold eaga_workspace_size(dims, 0) bytes.  On the
 * specialised bf16 path the small prologue and row-order kernels run beside
 * the Q/K/V projection on the library's per-device streams, ordered on
 * `stream` like the backward's (below). */
EAGA_API eaga_status eaga_forward(const eaga_dims *dims,
                         const void *X, const void *E, const void *y, const uint8_t *M,
                         const eaga_weights *w,
                         void *Xout, void *Eout, void *saved,
                         void *workspace, size_t ws_bytes, void *stream);

/* Backward of the layer.  Given the forward's inputs, its `saved` state and
 * the upstream gradients dXout, dEout, writes dX, dE, dy and every weight
 * gradient (fp32).  `workspace` must hold eaga_workspace_size(dims, 1) bytes.
 * Gradients of masked nodes / invalid pairs are the residual ones
 * (dX_i = dX'_i, dE_ij = dE'_ij).
 * On the specialised bf16 path some independent kernels run on three streams
 * the library creates once per device; they start after the work already
 * on `stream` and `stream` waits for them before the call's last kernels,
 * so the call is ordered on `stream` as a whole (and a CUDA graph captured
 * around it keeps them as parallel branches).  On that path the key and
 * value gradients are fp32 sums over the graph's row blocks added in the
 * order the blocks run, so dX, dWk, dbk, dWv and dbv may differ in their
 * last bits between calls; every other output is reproducible bit for bit. */
EAGA_API eaga_status eaga_backward(const eaga_dims *dims,
                          const void *X, const void *E, const void *y, const uint8_t *M,
                          const eaga_weights *w, const void *saved,
                          const void *dXout, const void *dEout,
                          void *dX, void *dE, void *dy, const eaga_weight_grads *dW,
                          void *workspace, size_t ws_bytes, void *stream);

/* Ablation variants of the layer (AI-summary page: the method paragraph's
 * ablation of unnormalised coefficients, and the "Light Edge" bullet):
 *   EAGA_VARIANT_LAYER         the layer above (eaga_forward, eaga_backward);
 *   EAGA_VARIANT_LIGHT_EDGE    no per-edge modulation: gamma, beta = y_b Wfy +
 *                              bf.  Wfe is not read (pass any valid pointer)
 *                              and its gradient is written as zero (it is not
 *                              a parameter of that layer); dE = dE'.  On the
 *                              specialised bf16 path the forward reads E only
 *                              once (for the residual) and the backward not
 *                              at all;
 *   EAGA_VARIANT_UNNORMALISED  the edge update from the unnormalised
 *                              coefficients, read as the modulated scores:
 *                              E'_ij = E_ij + sum_h s'^h_ij We[h,:] on valid
 *                              pairs (E_ij elsewhere); the node path is the
 *                              layer's.  Its backward: D_i = sum_j a_ij dO_i.v_j,
 *                              dS'_ij = a_ij (dO_i.v_j - D_i) + u_ij (u_ij =
 *                              We . dE'_ij on valid pairs), dWe = sum s'^T dE'.
 * The pages print neither variant's equations; these are this library's
 * readings.  Arguments, layouts and errors are those of eaga_forward and
 * eaga_backward; an unknown variant returns EAGA_ERR_INVALID_ARG. */
typedef enum {
    EAGA_VARIANT_LAYER = 0,
    EAGA_VARIANT_LIGHT_EDGE = 1,
    EAGA_VARIANT_UNNORMALISED = 2
} eaga_variant;

EAGA_API eaga_status eaga_forward_variant(const eaga_dims *dims, int variant,
                                          const void *X, const void *E, const void *y, const uint8_t *M,
                                          const eaga_weights *w,
                                          void *Xout, void *Eout, void *saved,
                                          void *workspace, size_t ws_bytes, void *stream);
EAGA_API eaga_status eaga_backward_variant(const eaga_dims *dims, int variant,
                                           const void *X, const void *E, const void *y, const uint8_t *M,
                                           const eaga_weights *w, const void *saved,
                                           const void *dXout, const void *dEout,
                                           void *dX, void *dE, void *dy, const eaga_weight_grads *dW,
                                           void *workspace, size_t ws_bytes, void *stream);

/* Row slabs of one graph (rows split over ranks: the AI-summary page's method
 * paragraph notes the edge update stays quadratic, so a large graph's pairs
 * are split by rows i).  The call owns rows row0 .. row0+rows-1 of every
 * graph: E_rows, Eout_rows, dEout_rows and dE_rows are [B, rows, n, de]
 * slabs of the pair tensors; X, y, M, Xout, dXout, dX, dy, the weights and
 * `saved` are whole.  Specialised bf16 path only (EAGA_ERR_UNSUPPORTED
 * otherwise); row0 a multiple of 8, rows even and a multiple of 8 unless the
 * slab ends at n (EAGA_ERR_INVALID_ARG otherwise).  Workspace sizes are those
 * of the whole layer.
 *
 * Forward: Q, K, V of every node (each rank computes them: a node GEMM, no
 * exchange), then the pairs of the slab's rows against all columns.  Writes
 * Eout_rows, and in Xout and `saved` the slab's rows (O of the other rows is
 * zero; their Xout rows are left unspecified).
 *
 * Backward: the gradients of L_r = <dXout, Xout> + <dEout_rows, Eout_rows>
 * with dXout zero outside the slab's rows (the caller passes it so).  dE_rows
 * is final; dX, dy and the weight gradients are this slab's part, and the
 * sum of the parts over slabs covering every row is the layer's gradient
 * (the layer is linear in its upstream gradients), e.g. one all-reduce. */
EAGA_API eaga_status eaga_forward_rows(const eaga_dims *dims, int variant, int row0, int rows,
                                       const void *X, const void *E_rows, const void *y, const uint8_t *M,
                                       const eaga_weights *w, void *Xout, void *Eout_rows, void *saved,
                                       void *workspace, size_t ws_bytes, void *stream);
EAGA_API eaga_status eaga_backward_rows(const eaga_dims *dims, int variant, int row0, int rows,
                                        const void *X, const void *E_rows, const void *y, const uint8_t *M,
                                        const eaga_weights *w, const void *saved,
                                        const void *dXout, const void *dEout_rows,
                                        void *dX, void *dE_rows, void *dy, const eaga_weight_grads *dW,
                                        void *workspace, size_t ws_bytes, void *stream);

/* Forward without a caller-provided workspace.  The paper has no counterpart
 * of this call; it exists for callers that cannot allocate device memory
 * for scratch: plain C clients that link this library but no device
 * allocator, or code under a framework whose memory pool only hands out the
 * tensors it owns.  It computes exactly what eaga_forward computes, with the
 * same arguments minus the workspace; `saved` is required (it is an output
 * as large as the node tensors).
 *
 * Argument checks and error codes are those of eaga_forward (invalid dims
 * give EAGA_ERR_INVALID_ARG, dims outside the limits EAGA_ERR_UNSUPPORTED).
 *
 * The forward's small scratch (status word, global FiLM term g [B,2H] fp32,
 * and on the specialised bf16 path of de = 64, H = 8, dh = 32 also 8 KiB of
 * tensor-core operand images) lives in a 64 KiB array in the library's
 * device memory, held by every GPU that loads the library until the process
 * exits.  Limit: 256 + roundup256(8*H*B) bytes, plus 8192 on the specialised
 * path, must fit in 64 KiB: B <= 892 graphs on the specialised path, B <= 4080
 * at H = 2 on the CUDA-core path; larger B returns EAGA_ERR_UNSUPPORTED
 * without launching.  Where roundup256(4*B*ceil(n/8)) bytes more also fit, the
 * specialised path keeps there the order in which its pair kernel takes the
 * row blocks (longest first, one more kernel launch); otherwise it takes them
 * in index order, with the same results.  No device memory is allocated or
 * freed by this call.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call on a device shares the array and leaves its contents
 * behind: calls that overlap on the GPU (other streams, other host threads)
 * race on it and must be serialised by the caller.  The status word is
 * cleared at the start of each call; eaga_get_device_status(NULL, stream)
 * reads it (EAGA_ERR_TIMEOUT if a bounded device wait of the call ran out). */
EAGA_API eaga_status eaga_forward_noalloc(const eaga_dims *dims,
                                          const void *X, const void *E, const void *y, const uint8_t *M,
                                          const eaga_weights *w, void *Xout, void *Eout, void *saved,
                                          void *stream);

/* Test aid: writes the normalised coefficients A [B,H,n,n] (fp32) that the
 * forward used, recomputed from E, y and the forward's `saved` state.  `A`
 * must hold B*H*n*n + 2*B*H floats (the tail is scratch).  Writes O(B*H*n*n)
 * memory; meant for small graphs only. */
EAGA_API eaga_status eaga_debug_attention_map(const eaga_dims *dims, const void *E, const uint8_t *M,
                                     const eaga_weights *w, const void *y, const void *saved,
                                     float *A, void *stream);

/* Synchronises `stream`, then reads and clears the device status word kept at
 * the start of `workspace`: EAGA_OK, or EAGA_ERR_TIMEOUT if a bounded
 * device-side wait ran out during a call that used this workspace.  With
 * workspace == NULL it reads the status word of eaga_forward_noalloc (the
 * first int of the library's fixed scratch array on the current device). */
EAGA_API eaga_status eaga_get_device_status(void *workspace, void *stream);

/* Profiling aid.  After eaga_set_profile_events(point, before, after) with
 * two cudaEvent_t handles, every later eaga_forward (point 0: the pair
 * kernels of the forward) or eaga_backward (point 1: the pair kernels of the
 * backward; point 2: the backward's row pair kernel alone, specialised bf16
 * path only) records `before` on its stream just before launching those
 * kernels and `after` just after them; points 3 and 4 do the same around the
 * edge kernel of eaga_block_forward and eaga_block_backward.  NULL events
 * clear the point.  This is a process-wide setting: not for concurrent calls. */
typedef enum {
    EAGA_PROF_FWD_PAIR = 0, EAGA_PROF_BWD_PAIR = 1, EAGA_PROF_BWD_ROWS = 2,
    EAGA_PROF_BLOCK_EDGE_FWD = 3, EAGA_PROF_BLOCK_EDGE_BWD = 4
} eaga_prof_point;
EAGA_API eaga_status eaga_set_profile_events(int point, void *before, void *after);

/* Number of kernel launches (this library's kernels) that one eaga_forward
 * (for_backward = 0) or eaga_backward (for_backward = 1) call issues for
 * these dims; -1 for invalid or unsupported dims. */
EAGA_API int eaga_kernel_launches(const eaga_dims *dims, int for_backward);

/* Test aid for the failure path of the bounded device waits.  Launches one
 * small kernel that waits on an mbarrier nothing will ever complete, with the
 * same bounded poll loop the pair kernels use, for `limit` polls
 * (1 <= limit <= 2^24); when the limit runs out the kernel records the
 * timeout in the status word at the start of `workspace` and returns, the
 * way a pair kernel does (no trap, the context stays usable).  A following
 * eaga_get_device_status on that workspace returns EAGA_ERR_TIMEOUT.  With
 * workspace == NULL the probe reports into the status word of
 * eaga_forward_noalloc instead.  The pages have no counterpart. */
EAGA_API eaga_status eaga_debug_wait_probe(void *workspace, unsigned limit, void *stream);

/* Static, human-readable name of a status code. */
/* ---------------------------------------------------------------------
 * The graph-transformer block around the layer.  The pages place the layer
 * inside DeFoG's graph-transformer backbone, which updates node, edge and
 * global features jointly (AI-summary page, method paragraph; paper index
 * page, abstract), but print none of the block's equations; this library's
 * reading is the plain post-norm block (LN over the last axis, biased
 * variance, eps 1e-5; relu; cnt_b = sum_i M_bi; valid as above):
 *
 *   (X', E') = the layer above on (X, E, y, M)
 *   pX_b = sum_i M_bi X'_bi / max(cnt_b, 1)
 *   pE_b = sum_ij valid_bij E'_bij / max(cnt_b^2, 1)
 *   y1_b = y_b + pX_b Wyx + pE_b Wye + by
 *   for Z in (X', E', y1):  Za = LN(Z; ln1_g, ln1_s)
 *                           Zz = Za + relu(Za W1 + b1) W2 + b2
 *                           Zo = LN(Zz; ln2_g, ln2_s)
 *   Xout = M Xo,  Eout = valid Eo,  yout = yo
 *
 * Parameters per sub-block (x: node, e: edge, y: global), [in, out]:
 * ln1_g, ln1_s [w]; W1 [w, 2w]; b1 [2w]; W2 [2w, w]; b2 [w]; ln2_g, ln2_s [w]
 * with w = dx, de, dy; then Wyx [dx, dy], Wye [de, dy], by [dy].  Storage
 * dtype as the layer's weights; gradients fp32.
 *
 * Supported on the specialised bf16 path only (de = 64, H = 8, dh = 32, n
 * even) with dx = 256 or 512 and dy a multiple of 32 up to 128; other dims
 * return EAGA_ERR_UNSUPPORTED.  A stack of blocks calls these once per block
 * with each block's own weights, feeding Xout, Eout, yout on.
 * --------------------------------------------------------------------- */
typedef struct {
    const void *x_ln1_g, *x_ln1_s, *x_W1, *x_b1, *x_W2, *x_b2, *x_ln2_g, *x_ln2_s;
    const void *e_ln1_g, *e_ln1_s, *e_W1, *e_b1, *e_W2, *e_b2, *e_ln2_g, *e_ln2_s;
    const void *y_ln1_g, *y_ln1_s, *y_W1, *y_b1, *y_W2, *y_b2, *y_ln2_g, *y_ln2_s;
    const void *Wyx, *Wye, *by;
} eaga_block_weights;

/* fp32 gradients of the block's parameters, same shapes; overwritten. */
typedef struct {
    void *x_ln1_g, *x_ln1_s, *x_W1, *x_b1, *x_W2, *x_b2, *x_ln2_g, *x_ln2_s;
    void *e_ln1_g, *e_ln1_s, *e_W1, *e_b1, *e_W2, *e_b2, *e_ln2_g, *e_ln2_s;
    void *y_ln1_g, *y_ln1_s, *y_W1, *y_b1, *y_W2, *y_b2, *y_ln2_g, *y_ln2_s;
    void *Wyx, *Wye, *by;
} eaga_block_grads;

/* Bytes of the block's saved state: the layer's (eaga_saved_size, first),
 * then the node sub-block's Za, relu(Za W1 + b1), Zz [B,n,dx|2dx|dx] and y1,
 * pX, pE per graph (fp32).  O(B n dx), no per-pair term.  0 if unsupported. */
EAGA_API size_t eaga_block_saved_size(const eaga_dims *dims);
/* Workspace bytes of eaga_block_forward (0) or eaga_block_backward (1): the
 * layer's workspace, then the block's node-sized buffers and fixed-size
 * partial sums.  No per-pair term.  0 if unsupported. */
EAGA_API size_t eaga_block_workspace_size(const eaga_dims *dims, int for_backward);
/* Kernels one block call launches (the layer's included); -1 if unsupported. */
EAGA_API int eaga_block_kernel_launches(const eaga_dims *dims, int for_backward);

/* Forward of one block.  Writes the layer's outputs Xmid (X') and Emid (E'),
 * the block's outputs Xout, Eout [B,n,n,de], yout [B,dy] and `saved`
 * (eaga_block_saved_size bytes), which eaga_block_backward reads together
 * with Xmid and Emid.  Same conventions as eaga_forward; the outputs and
 * `saved` must not overlap the inputs, Xmid, Emid or the workspace. */
EAGA_API eaga_status eaga_block_forward(const eaga_dims *dims,
                                const void *X, const void *E, const void *y, const uint8_t *M,
                                const eaga_weights *w, const eaga_block_weights *wb,
                                void *Xmid, void *Emid, void *Xout, void *Eout, void *yout, void *saved,
                                void *workspace, size_t ws_bytes, void *stream);

/* Backward of one block: given the forward's inputs, Xmid, Emid, `saved` and
 * the upstream gradients dXout, dEout, dyout, writes dX, dE, dy, the layer's
 * weight gradients dW and the block's dWb.  dEmid [B,n,n,de] (storage dtype)
 * is caller-provided scratch that receives dE' (the gradient at the layer's
 * edge output); it must not overlap anything else.  Sums over rows and pairs
 * run in a fixed order except the layer's key/value gradients and the
 * block's edge pooling sums, whose fp32 additions follow the order the
 * CTAs run (see eaga_backward). */
EAGA_API eaga_status eaga_block_backward(const eaga_dims *dims,
                                 const void *X, const void *E, const void *y, const uint8_t *M,
                                 const eaga_weights *w, const eaga_block_weights *wb,
                                 const void *Xmid, const void *Emid, const void *saved,
                                 const void *dXout, const void *dEout, const void *dyout, void *dEmid,
                                 void *dX, void *dE, void *dy, const eaga_weight_grads *dW,
                                 const eaga_block_grads *dWb, void *workspace, size_t ws_bytes, void *stream);

EAGA_API const char *eaga_strerror(eaga_status s);

#ifdef __cplusplus
}
#endif
#endif /* EAGA_H */
