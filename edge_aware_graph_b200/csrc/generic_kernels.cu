// Plain CUDA-core kernels of the edge-aware attention layer, for every
// supported shape and both storage dtypes (fp32 accumulation).  One CTA per
// row (b,i) for the pair work; row-blocked dot products for the node work.
// These are the fp32-mode path (its results match the fp64 oracle to ~1e-6)
// and the path for shapes the specialised sm_100a kernels do not cover.
//
// Formulas: AI-summary page of "Efficient Edge-aware Attention Network for
// Graph Generation", method paragraph (head-wise FiLM in the score
// modification, masked softmax, identity-concatenated value giving O and the
// normalised map, residual edge update); the exact forms are the ones in
// include/eaga.h.
#include <math.h>
#include "common.cuh"
#include "generic.h"

namespace eaga {
namespace generic {

constexpr int RB = 16;      // rows per CTA in the node kernels
constexpr int NT = 256;     // threads per CTA

// ------------------------------------------------------------------ node work

// Q,K,V = X W + b; rows of masked nodes are written as zero.
template <typename T>
__global__ void __launch_bounds__(NT) k_qkv(const T *X, const T *Wq, const T *bq, const T *Wk,
                                            const T *bk, const T *Wv, const T *bv, const uint8_t *M,
                                            T *Q, T *K, T *V, int rows, int dx, int hd) {
    extern __shared__ float xs[];
    const int r0 = blockIdx.x * RB;
    for (int t = threadIdx.x; t < RB * dx; t += NT) {
        const int r = r0 + t / dx;
        xs[t] = r < rows ? ldf(X + (size_t)r * dx + t % dx) : 0.f;
    }
    __syncthreads();
    for (int o = threadIdx.x; o < 3 * hd; o += NT) {
        const int which = o / hd, col = o % hd;
        const T *W = which == 0 ? Wq : which == 1 ? Wk : Wv;
        const T *bb = which == 0 ? bq : which == 1 ? bk : bv;
        T *out = which == 0 ? Q : which == 1 ? K : V;
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        for (int k = 0; k < dx; ++k) {
            const float w = ldf(W + (size_t)k * hd + col);
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] = fmaf(xs[r * dx + k], w, acc[r]);
        }
        const float bias = ldf(bb + col);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int row = r0 + r;
            if (row < rows) stf(out + (size_t)row * hd + col, M[row] ? acc[r] + bias : 0.f);
        }
    }
}

// g_b = y_b Wfy + bf (fp32).
template <typename T>
__global__ void k_global_film(const T *y, const T *Wfy, const T *bf, float *g, int dy, int F) {
    const int b = blockIdx.x, k = threadIdx.x;
    if (k >= F) return;
    float acc = ldf(bf + k);
    for (int c = 0; c < dy; ++c) acc = fmaf(ldf(y + (size_t)b * dy + c), ldf(Wfy + (size_t)c * F + k), acc);
    g[(size_t)b * F + k] = acc;
}

// X' = X + M (O Wo + bo).
template <typename T>
__global__ void __launch_bounds__(NT) k_out_proj(const T *X, const T *O, const T *Wo, const T *bo,
                                                 const uint8_t *M, T *Xout, int rows, int hd, int dx) {
    extern __shared__ float os[];
    const int r0 = blockIdx.x * RB;
    for (int t = threadIdx.x; t < RB * hd; t += NT) {
        const int r = r0 + t / hd;
        os[t] = r < rows ? ldf(O + (size_t)r * hd + t % hd) : 0.f;
    }
    __syncthreads();
    for (int o = threadIdx.x; o < dx; o += NT) {
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        for (int k = 0; k < hd; ++k) {
            const float w = ldf(Wo + (size_t)k * dx + o);
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] = fmaf(os[r * hd + k], w, acc[r]);
        }
        const float bias = ldf(bo + o);
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int row = r0 + r;
            if (row >= rows) continue;
            const float x = ldf(X + (size_t)row * dx + o);
            stf(Xout + (size_t)row * dx + o, M[row] ? x + (acc[r] + bias) : x);
        }
    }
}

// ------------------------------------------------------------------ pair work

struct RowSmem {
    float *q, *wfe, *we, *gl, *a;
};

template <typename T>
__device__ __forceinline__ void load_row_consts(float *q, const T *Qrow, float *wfe, const T *Wfe,
                                                float *we, const T *We, float *gl, const float *g,
                                                int hd, int de, int H) {
    const int F = 2 * H;
    for (int t = threadIdx.x; t < hd; t += blockDim.x) q[t] = ldf(Qrow + t);
    // Wfe == nullptr: no per-edge FiLM map (the Light Edge variant)
    for (int t = threadIdx.x; t < de * F; t += blockDim.x) wfe[t] = Wfe ? ldf(Wfe + t) : 0.f;
    for (int t = threadIdx.x; t < H * de; t += blockDim.x) we[t] = ldf(We + t);
    for (int t = threadIdx.x; t < F; t += blockDim.x) gl[t] = g[t];
}

// FiLM coefficients of one pair for head h.
template <typename T>
__device__ __forceinline__ void film_h(const T *e, const float *wfe, const float *gl, int de, int H,
                                       int h, float &gam, float &bet) {
    const int F = 2 * H;
    gam = gl[h];
    bet = gl[H + h];
    for (int c = 0; c < de; ++c) {
        const float ev = ldf(e + c);
        gam = fmaf(ev, wfe[c * F + h], gam);
        bet = fmaf(ev, wfe[c * F + H + h], bet);
    }
}

// Forward of one row (b,i): modulated scores, masked softmax, O_i, E'_i*, LSE.
// unnorm: the edge update takes the modulated scores s' (valid pairs) instead of a.
template <typename T>
__global__ void __launch_bounds__(NT) k_attn_fwd_row(const T *E, const uint8_t *M, const T *Q, const T *K,
                                                     const T *V, const T *Wfe, const float *g, const T *We,
                                                     T *O, float *LSE, T *Eout, int n, int de, int H, int dh,
                                                     int unnorm) {
    extern __shared__ float sm[];
    const int F = 2 * H, hd = H * dh;
    float *q = sm, *wfe = q + hd, *we = wfe + de * F, *gl = we + H * de, *a = gl + F, *sps = a + H * n;
    const int b = blockIdx.y, i = blockIdx.x;
    const size_t row = (size_t)b * n + i;
    const uint8_t *mb = M + (size_t)b * n;
    const T *Erow = E + row * n * de;
    T *Eo = Eout + row * n * de;
    if (!mb[i]) {
        for (int t = threadIdx.x; t < hd; t += NT) stf(O + row * hd + t, 0.f);
        for (int h = threadIdx.x; h < H; h += NT) LSE[((size_t)b * H + h) * n + i] = -INFINITY;
        for (int t = threadIdx.x; t < n * de; t += NT) Eo[t] = Erow[t];
        return;
    }
    load_row_consts(q, Q + row * hd, wfe, Wfe, we, We, gl, g + (size_t)b * F, hd, de, H);
    __syncthreads();
    const float rs = 1.0f / sqrtf((float)dh);
    for (int j = threadIdx.x; j < n; j += NT) {
        const bool vj = mb[j];
        const T *e = Erow + (size_t)j * de;
        const T *kj = K + ((size_t)b * n + j) * hd;
        for (int h = 0; h < H; ++h) {
            float sp = -INFINITY;
            if (vj) {
                float gam, bet;
                film_h(e, wfe, gl, de, H, h, gam, bet);
                float s = 0.f;
                for (int t = 0; t < dh; ++t) s = fmaf(q[h * dh + t], ldf(kj + h * dh + t), s);
                s *= rs;
                sp = s * (1.f + gam) + bet;
            }
            a[h * n + j] = sp;
            if (unnorm) sps[h * n + j] = vj ? sp : 0.f;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int h = wid; h < H; h += NT / 32) {
        float m = -INFINITY;
        for (int j = lane; j < n; j += 32) m = fmaxf(m, a[h * n + j]);
        m = warp_max(m);
        float l = 0.f;
        for (int j = lane; j < n; j += 32) {
            const float v = a[h * n + j];
            l += mb[j] ? expf(v - m) : 0.f;
        }
        l = warp_sum(l);
        const float inv = 1.f / l;
        for (int j = lane; j < n; j += 32) {
            const float v = a[h * n + j];
            a[h * n + j] = mb[j] ? expf(v - m) * inv : 0.f;
        }
        if (lane == 0) LSE[((size_t)b * H + h) * n + i] = m + logf(l);
    }
    __syncthreads();
    for (int t = threadIdx.x; t < hd; t += NT) {
        const int h = t / dh;
        float acc = 0.f;
        for (int j = 0; j < n; ++j)
            if (mb[j]) acc = fmaf(a[h * n + j], ldf(V + ((size_t)b * n + j) * hd + t), acc);
        stf(O + row * hd + t, acc);
    }
    for (int t = threadIdx.x; t < n * de; t += NT) {
        const int j = t / de, c = t % de;
        float acc = ldf(Erow + t);
        const float *coef = unnorm ? sps : a;
        if (mb[j])
            for (int h = 0; h < H; ++h) acc = fmaf(coef[h * n + j], we[h * de + c], acc);
        stf(Eo + t, acc);
    }
}

// Normalised coefficients A[b,h,i,j] recomputed from E, Q, K and the LSE (test aid).
template <typename T>
__global__ void __launch_bounds__(NT) k_attn_map(const T *E, const uint8_t *M, const T *Q, const T *K,
                                                 const T *Wfe, const float *g, const float *LSE, float *A,
                                                 int n, int de, int H, int dh) {
    extern __shared__ float sm[];
    const int F = 2 * H, hd = H * dh;
    float *q = sm, *wfe = q + hd, *gl = wfe + de * F;
    const int b = blockIdx.y, i = blockIdx.x;
    const size_t row = (size_t)b * n + i;
    const uint8_t *mb = M + (size_t)b * n;
    for (int t = threadIdx.x; t < hd; t += NT) q[t] = ldf(Q + row * hd + t);
    for (int t = threadIdx.x; t < de * F; t += NT) wfe[t] = ldf(Wfe + t);
    for (int t = threadIdx.x; t < F; t += NT) gl[t] = g[(size_t)b * F + t];
    __syncthreads();
    const float rs = 1.0f / sqrtf((float)dh);
    for (int j = threadIdx.x; j < n; j += NT) {
        const bool v = mb[i] && mb[j];
        const T *e = E + (row * n + j) * de;
        const T *kj = K + ((size_t)b * n + j) * hd;
        for (int h = 0; h < H; ++h) {
            float out = 0.f;
            if (v) {
                float gam, bet;
                film_h(e, wfe, gl, de, H, h, gam, bet);
                float s = 0.f;
                for (int t = 0; t < dh; ++t) s = fmaf(q[h * dh + t], ldf(kj + h * dh + t), s);
                s *= rs;
                out = expf(s * (1.f + gam) + bet - LSE[((size_t)b * H + h) * n + i]);
            }
            A[(((size_t)b * H + h) * n + i) * n + j] = out;
        }
    }
}

// ------------------------------------------------------------------ backward

// dO_i = M_i dX'_i Wo^T (fp32).
template <typename T>
__global__ void __launch_bounds__(NT) k_bwd_dO(const T *dXout, const T *Wo, const uint8_t *M, float *dO,
                                               int rows, int dx, int hd) {
    extern __shared__ float ds[];
    const int r0 = blockIdx.x * RB;
    for (int t = threadIdx.x; t < RB * dx; t += NT) {
        const int r = r0 + t / dx;
        ds[t] = r < rows ? ldf(dXout + (size_t)r * dx + t % dx) : 0.f;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < hd; k += NT) {
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        for (int o = 0; o < dx; ++o) {
            const float w = ldf(Wo + (size_t)k * dx + o);
#pragma unroll
            for (int r = 0; r < RB; ++r) acc[r] = fmaf(ds[r * dx + o], w, acc[r]);
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int row = r0 + r;
            if (row < rows) dO[(size_t)row * hd + k] = M[row] ? acc[r] : 0.f;
        }
    }
}

// Row pass of the backward for row (b,i): a, dA, D_ih, dS', dq_i, dE_i*, and the
// row's parts of dWfe [de,2H], dWe [H,de], dg [2H].  unnorm: the edge path
// reaches s' directly (D from the node term only, u added to dS', dWe from s').
template <typename T>
__global__ void __launch_bounds__(NT) k_attn_bwd_row(const T *E, const uint8_t *M, const T *Q, const T *K,
                                                     const T *V, const float *LSE, const float *dO,
                                                     const T *dEout, const T *Wfe, const float *g, const T *We,
                                                     float *dQ, T *dE, float *Dout, float *parts,
                                                     size_t part_stride, int n, int de, int H, int dh, int unnorm) {
    extern __shared__ float sm[];
    const int F = 2 * H, hd = H * dh;
    float *q = sm, *dOi = q + hd, *wfe = dOi + hd, *we = wfe + de * F, *gl = we + H * de;
    float *A = gl + F, *G = A + H * n, *S = G + H * n, *GM = S + H * n, *D = GM + H * n, *SP = D + H;
    const int b = blockIdx.y, i = blockIdx.x;
    const size_t row = (size_t)b * n + i;
    const uint8_t *mb = M + (size_t)b * n;
    const T *Erow = E + row * n * de;
    const T *dEp = dEout + row * n * de;
    T *dEo = dE + row * n * de;
    float *pWfe = parts + row * part_stride, *pWe = pWfe + de * F, *pg = pWe + H * de;
    if (!mb[i]) {
        for (int t = threadIdx.x; t < hd; t += NT) dQ[row * hd + t] = 0.f;
        for (int t = threadIdx.x; t < n * de; t += NT) dEo[t] = dEp[t];
        for (int t = threadIdx.x; t < (int)part_stride; t += NT) pWfe[t] = 0.f;
        for (int h = threadIdx.x; h < H; h += NT) Dout[((size_t)b * H + h) * n + i] = 0.f;
        return;
    }
    load_row_consts(q, Q + row * hd, wfe, Wfe, we, We, gl, g + (size_t)b * F, hd, de, H);
    for (int t = threadIdx.x; t < hd; t += NT) dOi[t] = dO[row * hd + t];
    __syncthreads();
    const float rs = 1.0f / sqrtf((float)dh);
    for (int j = threadIdx.x; j < n; j += NT) {
        const bool vj = mb[j];
        const T *e = Erow + (size_t)j * de;
        const T *dep = dEp + (size_t)j * de;
        const T *kj = K + ((size_t)b * n + j) * hd;
        const T *vv = V + ((size_t)b * n + j) * hd;
        for (int h = 0; h < H; ++h) {
            float a = 0.f, dA = 0.f, s = 0.f, gam = 0.f, spv = 0.f;
            if (vj) {
                float bet;
                film_h(e, wfe, gl, de, H, h, gam, bet);
                for (int t = 0; t < dh; ++t) s = fmaf(q[h * dh + t], ldf(kj + h * dh + t), s);
                s *= rs;
                spv = s * (1.f + gam) + bet;
                a = expf(spv - LSE[((size_t)b * H + h) * n + i]);
                float u = 0.f, dov = 0.f;
                for (int c = 0; c < de; ++c) u = fmaf(we[h * de + c], ldf(dep + c), u);
                for (int t = 0; t < dh; ++t) dov = fmaf(dOi[h * dh + t], ldf(vv + h * dh + t), dov);
                dA = unnorm ? dov : dov + u;
            }
            if (unnorm) SP[h * n + j] = spv;
            A[h * n + j] = a;
            G[h * n + j] = dA;
            S[h * n + j] = s;
            GM[h * n + j] = gam;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int h = wid; h < H; h += NT / 32) {
        float acc = 0.f;
        for (int j = lane; j < n; j += 32) acc = fmaf(A[h * n + j], G[h * n + j], acc);
        acc = warp_sum(acc);
        if (lane == 0) {
            D[h] = acc;
            Dout[((size_t)b * H + h) * n + i] = acc;
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < H * n; t += NT) {
        const int h = t / n;
        float dsp = A[t] * (G[t] - D[h]);
        if (unnorm && mb[t % n]) {       // + u_ij on valid pairs
            const T *dep = dEp + (size_t)(t % n) * de;
            float u = 0.f;
            for (int c = 0; c < de; ++c) u = fmaf(we[h * de + c], ldf(dep + c), u);
            dsp += u;
        }
        G[t] = dsp;                    // dbeta
        S[t] = dsp * S[t];             // dgamma
        GM[t] = dsp * (1.f + GM[t]);   // ds
    }
    __syncthreads();
    for (int t = threadIdx.x; t < hd; t += NT) {
        const int h = t / dh;
        float acc = 0.f;
        for (int j = 0; j < n; ++j)
            if (mb[j]) acc = fmaf(GM[h * n + j], ldf(K + ((size_t)b * n + j) * hd + t), acc);
        dQ[row * hd + t] = acc * rs;
    }
    for (int t = threadIdx.x; t < n * de; t += NT) {
        const int j = t / de, c = t % de;
        float acc = ldf(dEp + t);
        for (int h = 0; h < H; ++h) {
            acc = fmaf(S[h * n + j], wfe[c * F + h], acc);
            acc = fmaf(G[h * n + j], wfe[c * F + H + h], acc);
        }
        stf(dEo + t, acc);
    }
    for (int t = threadIdx.x; t < de * F; t += NT) {
        const int c = t / F, k = t % F;
        const float *df = k < H ? S + k * n : G + (k - H) * n;
        float acc = 0.f;
        for (int j = 0; j < n; ++j) acc = fmaf(ldf(Erow + (size_t)j * de + c), df[j], acc);
        pWfe[t] = acc;
    }
    for (int t = threadIdx.x; t < H * de; t += NT) {
        const int h = t / de, c = t % de;
        const float *coef = unnorm ? SP : A;
        float acc = 0.f;
        for (int j = 0; j < n; ++j) acc = fmaf(coef[h * n + j], ldf(dEp + (size_t)j * de + c), acc);
        pWe[t] = acc;
    }
    for (int k = threadIdx.x; k < F; k += NT) {
        const float *df = k < H ? S + k * n : G + (k - H) * n;
        float acc = 0.f;
        for (int j = 0; j < n; ++j) acc += df[j];
        pg[k] = acc;
    }
}

// Column pass of the backward for column (b,j): dk_j, dv_j (fp32).
template <typename T>
__global__ void __launch_bounds__(NT) k_attn_bwd_col(const T *E, const uint8_t *M, const T *Q, const T *K,
                                                     const T *V, const float *LSE, const float *dO,
                                                     const T *dEout, const T *Wfe, const float *g, const T *We,
                                                     const float *Dst, float *dK, float *dV,
                                                     int n, int de, int H, int dh, int unnorm) {
    extern __shared__ float sm[];
    const int F = 2 * H, hd = H * dh;
    float *kj = sm, *vj = kj + hd, *wfe = vj + hd, *we = wfe + de * F, *gl = we + H * de;
    float *A = gl + F, *DS = A + H * n;
    const int b = blockIdx.y, j = blockIdx.x;
    const size_t col = (size_t)b * n + j;
    const uint8_t *mb = M + (size_t)b * n;
    if (!mb[j]) {
        for (int t = threadIdx.x; t < hd; t += NT) {
            dK[col * hd + t] = 0.f;
            dV[col * hd + t] = 0.f;
        }
        return;
    }
    load_row_consts(kj, K + col * hd, wfe, Wfe, we, We, gl, g + (size_t)b * F, hd, de, H);
    for (int t = threadIdx.x; t < hd; t += NT) vj[t] = ldf(V + col * hd + t);
    __syncthreads();
    const float rs = 1.0f / sqrtf((float)dh);
    for (int i = threadIdx.x; i < n; i += NT) {
        const size_t ri = (size_t)b * n + i;
        const T *e = E + (ri * n + j) * de;
        const T *dep = dEout + (ri * n + j) * de;
        for (int h = 0; h < H; ++h) {
            float a = 0.f, dsv = 0.f;
            if (mb[i]) {
                float gam, bet;
                film_h(e, wfe, gl, de, H, h, gam, bet);
                float s = 0.f;
                for (int t = 0; t < dh; ++t) s = fmaf(ldf(Q + ri * hd + h * dh + t), kj[h * dh + t], s);
                s *= rs;
                a = expf(s * (1.f + gam) + bet - LSE[((size_t)b * H + h) * n + i]);
                float u = 0.f, dov = 0.f;
                for (int c = 0; c < de; ++c) u = fmaf(we[h * de + c], ldf(dep + c), u);
                for (int t = 0; t < dh; ++t) dov = fmaf(dO[ri * hd + h * dh + t], vj[h * dh + t], dov);
                const float D = Dst[((size_t)b * H + h) * n + i];
                const float dsp = unnorm ? a * (dov - D) + u : a * (dov + u - D);
                dsv = dsp * (1.f + gam);
            }
            A[h * n + i] = a;
            DS[h * n + i] = dsv;
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < hd; t += NT) {
        const int h = t / dh;
        float dk = 0.f, dv = 0.f;
        for (int i = 0; i < n; ++i) {
            if (!mb[i]) continue;
            const size_t ri = (size_t)b * n + i;
            dk = fmaf(DS[h * n + i], ldf(Q + ri * hd + t), dk);
            dv = fmaf(A[h * n + i], dO[ri * hd + t], dv);
        }
        dK[col * hd + t] = dk * rs;
        dV[col * hd + t] = dv;
    }
}

// dX = dX' + dQ Wq^T + dK Wk^T + dV Wv^T.
template <typename T>
__global__ void __launch_bounds__(NT) k_bwd_dX(const T *dXout, const float *dQ, const float *dK,
                                               const float *dV, const T *Wq, const T *Wk, const T *Wv,
                                               T *dX, int rows, int dx, int hd) {
    extern __shared__ float gs[];   // 3 * RB * hd
    const int r0 = blockIdx.x * RB;
    for (int t = threadIdx.x; t < RB * hd; t += NT) {
        const int r = r0 + t / hd;
        const size_t idx = (size_t)r * hd + t % hd;
        gs[t] = r < rows ? dQ[idx] : 0.f;
        gs[RB * hd + t] = r < rows ? dK[idx] : 0.f;
        gs[2 * RB * hd + t] = r < rows ? dV[idx] : 0.f;
    }
    __syncthreads();
    for (int c = threadIdx.x; c < dx; c += NT) {
        float acc[RB];
#pragma unroll
        for (int r = 0; r < RB; ++r) acc[r] = 0.f;
        for (int p = 0; p < 3; ++p) {
            const T *W = p == 0 ? Wq : p == 1 ? Wk : Wv;
            const float *gp = gs + p * RB * hd;
            for (int k = 0; k < hd; ++k) {
                const float w = ldf(W + (size_t)c * hd + k);
#pragma unroll
                for (int r = 0; r < RB; ++r) acc[r] = fmaf(gp[r * hd + k], w, acc[r]);
            }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r) {
            const int row = r0 + r;
            if (row < rows) stf(dX + (size_t)row * dx + c, ldf(dXout + (size_t)row * dx + c) + acc[r]);
        }
    }
}

// out[c,k] = sum_r A[r,c] Bm[r,k]  (weight gradient X^T dY), and, when bias is
// given, bias[k] = sum_r w_r Bm[r,k] with w_r = M_r if M given else 1.
constexpr int CB = 16;
template <typename TA, typename TB>
__global__ void __launch_bounds__(NT) k_xty(const TA *A, const TB *Bm, float *out, float *bias,
                                            const uint8_t *M, int rows, int C, int Kd) {
    const int c0 = blockIdx.x * CB;
    const int k = blockIdx.y * NT + threadIdx.x;
    __shared__ float as[CB][64];
    float acc[CB];
#pragma unroll
    for (int t = 0; t < CB; ++t) acc[t] = 0.f;
    float bacc = 0.f;
    for (int r0 = 0; r0 < rows; r0 += 64) {
        __syncthreads();
        for (int t = threadIdx.x; t < CB * 64; t += NT) {
            const int cc = t / 64, rr = t % 64;
            const int r = r0 + rr, c = c0 + cc;
            as[cc][rr] = (r < rows && c < C) ? ldf(A + (size_t)r * C + c) : 0.f;
        }
        __syncthreads();
        if (k < Kd) {
            const int rn = min(64, rows - r0);
            for (int rr = 0; rr < rn; ++rr) {
                const float bv = ldf(Bm + (size_t)(r0 + rr) * Kd + k);
#pragma unroll
                for (int t = 0; t < CB; ++t) acc[t] = fmaf(as[t][rr], bv, acc[t]);
                if (bias && blockIdx.x == 0) bacc += (M ? (M[r0 + rr] ? bv : 0.f) : bv);
            }
        }
    }
    if (k >= Kd) return;
#pragma unroll
    for (int t = 0; t < CB; ++t)
        if (c0 + t < C) out[(size_t)(c0 + t) * Kd + k] = acc[t];
    if (bias && blockIdx.x == 0) bias[k] = bacc;
}

// dWfe, dWe = sums of the per-row parts (row order); dg[b,:] = sum over the graph's rows.
__global__ void k_reduce_parts(const float *parts, size_t part_stride, int B, int n, int nWfe, int nWe, int F,
                               float *dWfe, float *dWe, float *dg, int zero_wfe) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int rows = B * n;
    if (t < nWfe) {
        float acc = 0.f;
        for (int r = 0; r < rows; ++r) acc += parts[(size_t)r * part_stride + t];
        dWfe[t] = zero_wfe ? 0.f : acc;     // Light Edge: Wfe is not a parameter
    } else if (t < nWfe + nWe) {
        float acc = 0.f;
        for (int r = 0; r < rows; ++r) acc += parts[(size_t)r * part_stride + t];
        dWe[t - nWfe] = acc;
    } else if (t < nWfe + nWe + B * F) {
        const int u = t - nWfe - nWe, b = u / F, k = u % F;
        float acc = 0.f;
        for (int i = 0; i < n; ++i) acc += parts[((size_t)b * n + i) * part_stride + nWfe + nWe + k];
        dg[(size_t)b * F + k] = acc;
    }
}

// dWfy = sum_b y_b^T dg_b, dbf = sum_b dg_b, dy_b = dg_b Wfy^T.
template <typename T>
__global__ void k_film_grads(const T *y, const T *Wfy, const float *dg, float *dWfy, float *dbf, T *dy,
                             int B, int dy_, int F) {
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < dy_ * F) {
        const int c = t / F, k = t % F;
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc = fmaf(ldf(y + (size_t)b * dy_ + c), dg[(size_t)b * F + k], acc);
        dWfy[t] = acc;
    } else if (t < dy_ * F + F) {
        const int k = t - dy_ * F;
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc += dg[(size_t)b * F + k];
        dbf[k] = acc;
    } else if (t < dy_ * F + F + B * dy_) {
        const int u = t - dy_ * F - F, b = u / dy_, c = u % dy_;
        float acc = 0.f;
        for (int k = 0; k < F; ++k) acc = fmaf(dg[(size_t)b * F + k], ldf(Wfy + (size_t)c * F + k), acc);
        stf(dy + (size_t)b * dy_ + c, acc);
    }
}

// ------------------------------------------------------------------ host side

// (the unnormalised variant keeps the modulated scores of the row too: H*n more floats)
static inline size_t row_smem_fwd(const eaga_dims &d, int unnorm = 1) {
    return sizeof(float) * (size_t(d.H) * d.dh + size_t(d.de) * 2 * d.H + size_t(d.H) * d.de + 2 * d.H +
                            size_t(1 + (unnorm ? 1 : 0)) * d.H * d.n);
}
static inline size_t row_smem_bwd(const eaga_dims &d, int unnorm = 1) {
    return sizeof(float) * (2 * size_t(d.H) * d.dh + size_t(d.de) * 2 * d.H + size_t(d.H) * d.de + 2 * d.H +
                            size_t(4 + (unnorm ? 1 : 0)) * d.H * d.n + d.H);
}
static inline size_t col_smem_bwd(const eaga_dims &d) {
    return sizeof(float) * (2 * size_t(d.H) * d.dh + size_t(d.de) * 2 * d.H + size_t(d.H) * d.de + 2 * d.H +
                            2 * size_t(d.H) * d.n);
}

size_t max_dynamic_smem(const eaga_dims &d) {
    size_t m = row_smem_fwd(d);
    m = m > row_smem_bwd(d) ? m : row_smem_bwd(d);
    m = m > col_smem_bwd(d) ? m : col_smem_bwd(d);
    const size_t node = sizeof(float) * RB * size_t(d.dx > d.H * d.dh ? d.dx : d.H * d.dh) * 3;
    return m > node ? m : node;
}

template <typename K>
static cudaError_t set_smem(K kernel, size_t bytes) {
    if (bytes <= 48 * 1024) return cudaSuccess;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

#define EAGA_TRY(x)                                   \
    do {                                              \
        cudaError_t e_ = (x);                         \
        if (e_ != cudaSuccess) return e_;             \
    } while (0)

template <typename T>
static cudaError_t forward_t(const eaga_dims &d, const FwdArgs &a, cudaStream_t st) {
    const int rows = d.B * d.n, hd = d.H * d.dh, F = 2 * d.H;
    const T *W[12];
    for (int t = 0; t < 12; ++t) W[t] = static_cast<const T *>(a.w[t]);
    T *Q = static_cast<T *>(a.Q), *K = static_cast<T *>(a.K), *V = static_cast<T *>(a.V), *O = static_cast<T *>(a.O);
    const size_t sq = sizeof(float) * RB * d.dx;
    EAGA_TRY(set_smem(k_qkv<T>, sq));
    k_qkv<T><<<(rows + RB - 1) / RB, NT, sq, st>>>(static_cast<const T *>(a.X), W[0], W[1], W[2], W[3], W[4], W[5],
                                                    a.M, Q, K, V, rows, d.dx, hd);
    k_global_film<T><<<d.B, 32, 0, st>>>(static_cast<const T *>(a.y), W[7], W[8], a.g, d.dy, F);
    const int unnorm = a.variant == EAGA_VARIANT_UNNORMALISED;
    const T *Wfe = a.variant == EAGA_VARIANT_LIGHT_EDGE ? nullptr : W[6];
    const size_t sr = row_smem_fwd(d, unnorm);
    EAGA_TRY(set_smem(k_attn_fwd_row<T>, row_smem_fwd(d)));
    prof_mark(0, 0, st);
    k_attn_fwd_row<T><<<dim3(d.n, d.B), NT, sr, st>>>(static_cast<const T *>(a.E), a.M, Q, K, V, Wfe, a.g, W[9], O,
                                                       a.LSE, static_cast<T *>(a.Eout), d.n, d.de, d.H, d.dh, unnorm);
    prof_mark(0, 1, st);
    const size_t so = sizeof(float) * RB * hd;
    EAGA_TRY(set_smem(k_out_proj<T>, so));
    k_out_proj<T><<<(rows + RB - 1) / RB, NT, so, st>>>(static_cast<const T *>(a.X), O, W[10], W[11], a.M,
                                                         static_cast<T *>(a.Xout), rows, hd, d.dx);
    return cudaGetLastError();
}

template <typename T>
static cudaError_t backward_t(const eaga_dims &d, const BwdArgs &a, cudaStream_t st) {
    const int rows = d.B * d.n, hd = d.H * d.dh, F = 2 * d.H;
    const T *W[12];
    for (int t = 0; t < 12; ++t) W[t] = static_cast<const T *>(a.w[t]);
    const T *X = static_cast<const T *>(a.X), *E = static_cast<const T *>(a.E);
    const T *Q = static_cast<const T *>(a.Q), *K = static_cast<const T *>(a.K);
    const T *V = static_cast<const T *>(a.V), *O = static_cast<const T *>(a.O);
    const T *dXo = static_cast<const T *>(a.dXout), *dEo = static_cast<const T *>(a.dEout);
    k_global_film<T><<<d.B, 32, 0, st>>>(static_cast<const T *>(a.y), W[7], W[8], a.g, d.dy, F);
    const size_t sd = sizeof(float) * RB * d.dx;
    EAGA_TRY(set_smem(k_bwd_dO<T>, sd));
    k_bwd_dO<T><<<(rows + RB - 1) / RB, NT, sd, st>>>(dXo, W[10], a.M, a.dO, rows, d.dx, hd);
    const int unnorm = a.variant == EAGA_VARIANT_UNNORMALISED, light = a.variant == EAGA_VARIANT_LIGHT_EDGE;
    const T *Wfe = light ? nullptr : W[6];
    const size_t sr = row_smem_bwd(d, unnorm);
    EAGA_TRY(set_smem(k_attn_bwd_row<T>, row_smem_bwd(d)));
    const size_t sc = col_smem_bwd(d);
    EAGA_TRY(set_smem(k_attn_bwd_col<T>, sc));
    prof_mark(1, 0, st);
    k_attn_bwd_row<T><<<dim3(d.n, d.B), NT, sr, st>>>(E, a.M, Q, K, V, a.LSE, a.dO, dEo, Wfe, a.g, W[9], a.dQ,
                                                       static_cast<T *>(a.dE), a.D, a.parts, a.part_stride, d.n,
                                                       d.de, d.H, d.dh, unnorm);
    k_attn_bwd_col<T><<<dim3(d.n, d.B), NT, sc, st>>>(E, a.M, Q, K, V, a.LSE, a.dO, dEo, Wfe, a.g, W[9], a.D,
                                                       a.dK, a.dV, d.n, d.de, d.H, d.dh, unnorm);
    prof_mark(1, 1, st);
    const int nWfe = d.de * F, nWe = d.H * d.de, tot = nWfe + nWe + d.B * F;
    k_reduce_parts<<<(tot + 255) / 256, 256, 0, st>>>(a.parts, a.part_stride, d.B, d.n, nWfe, nWe, F, a.dW[6],
                                                      a.dW[9], a.dg, light);
    const int tf = d.dy * F + F + d.B * d.dy;
    k_film_grads<T><<<(tf + 255) / 256, 256, 0, st>>>(static_cast<const T *>(a.y), W[7], a.dg, a.dW[7], a.dW[8],
                                                      static_cast<T *>(a.dy), d.B, d.dy, F);
    const size_t sx = sizeof(float) * 3 * RB * hd;
    EAGA_TRY(set_smem(k_bwd_dX<T>, sx));
    k_bwd_dX<T><<<(rows + RB - 1) / RB, NT, sx, st>>>(dXo, a.dQ, a.dK, a.dV, W[0], W[2], W[4],
                                                       static_cast<T *>(a.dX), rows, d.dx, hd);
    const dim3 gq((d.dx + CB - 1) / CB, (hd + NT - 1) / NT);
    k_xty<T, float><<<gq, NT, 0, st>>>(X, a.dQ, a.dW[0], a.dW[1], nullptr, rows, d.dx, hd);
    k_xty<T, float><<<gq, NT, 0, st>>>(X, a.dK, a.dW[2], a.dW[3], nullptr, rows, d.dx, hd);
    k_xty<T, float><<<gq, NT, 0, st>>>(X, a.dV, a.dW[4], a.dW[5], nullptr, rows, d.dx, hd);
    const dim3 go((hd + CB - 1) / CB, (d.dx + NT - 1) / NT);
    k_xty<T, T><<<go, NT, 0, st>>>(O, dXo, a.dW[10], a.dW[11], a.M, rows, hd, d.dx);
    return cudaGetLastError();
}

int kernel_launches(const eaga_dims &, int for_backward) { return for_backward ? 10 : 4; }

cudaError_t forward(const eaga_dims &d, const FwdArgs &a, cudaStream_t st) {
    return d.dtype == EAGA_BF16 ? forward_t<__nv_bfloat16>(d, a, st) : forward_t<float>(d, a, st);
}
cudaError_t backward(const eaga_dims &d, const BwdArgs &a, cudaStream_t st) {
    return d.dtype == EAGA_BF16 ? backward_t<__nv_bfloat16>(d, a, st) : backward_t<float>(d, a, st);
}

template <typename T>
static cudaError_t attn_map_t(const eaga_dims &d, const MapArgs &a, cudaStream_t st) {
    const int F = 2 * d.H;
    k_global_film<T><<<d.B, 32, 0, st>>>(static_cast<const T *>(a.y), static_cast<const T *>(a.Wfy),
                                         static_cast<const T *>(a.bf), a.g, d.dy, F);
    const size_t s = sizeof(float) * (size_t(d.H) * d.dh + size_t(d.de) * F + F);
    EAGA_TRY(set_smem(k_attn_map<T>, s));
    k_attn_map<T><<<dim3(d.n, d.B), NT, s, st>>>(static_cast<const T *>(a.E), a.M, static_cast<const T *>(a.Q),
                                                 static_cast<const T *>(a.K), static_cast<const T *>(a.Wfe), a.g,
                                                 a.LSE, a.A, d.n, d.de, d.H, d.dh);
    return cudaGetLastError();
}

cudaError_t attention_map(const eaga_dims &d, const MapArgs &a, cudaStream_t st) {
    return d.dtype == EAGA_BF16 ? attn_map_t<__nv_bfloat16>(d, a, st) : attn_map_t<float>(d, a, st);
}

}  // namespace generic
}  // namespace eaga
