// Shared constants, workspace layout and device helpers of the specialised
// sm_100a path (de = 64, H = 8, dh = 32, bf16 storage).
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "sm100.cuh"

namespace eaga {
namespace fast {

constexpr int DE = 64, NH = 8, DH = 32, HD = 256, NF = 16;
constexpr int TB = 8;            // pair tile: 8 "own" rows x 32*NR "cluster" rows
// NR = 1: 32 cluster rows per CTA (n <= 512; two CTAs fit on an SM);
// NR = 2: 64 cluster rows per CTA (n <= 1024).
__host__ __device__ constexpr int tile_cols(int NR) { return 32 * NR; }
inline int pick_nr(int n) { return n <= 512 ? 1 : 2; }
// Streaming multiprocessors of the current device (cached per process).
inline int sm_count() {
    static int cached = 0;
    if (!cached) {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess)
            cached = v;
        else
            cached = 148;
    }
    return cached;
}

// Operand images prepared once per call by the prologue kernel (bf16, in the
// exact shared-memory layout the tensor-core descriptors expect).
//   IMG_WFE_T_SW : B[N=16 k][K=64 c] = Wfe^T, 128B-swizzled     (FiLM)
//   IMG_WE_T_NS  : B[N=64 c][K=16 h] = We^T, h>=8 zero, no swizzle (edge update)
//   IMG_WE_SW    : B[N=16 h][K=64 c] = We, h>=8 zero, 128B-swizzled (u = We . dE')
//   IMG_WFE_NS   : B[N=64 c][K=16 k] = Wfe, no swizzle            (dE = df Wfe^T)
constexpr uint32_t IMG_WFE_T_SW = 0, IMG_WE_T_NS = 2048, IMG_WE_SW = 4096, IMG_WFE_NS = 6144, IMG_BYTES = 8192;

// byte offset of 16-byte chunk `ch` of row `row` in a 128B-swizzled region
__host__ __device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t ch) {
    return row * 128u + ((ch ^ (row & 7u)) << 4);
}
// byte offset of element (row, k) in a no-swizzle K-major [rows][16] bf16 tile
// byte offset of 16-byte chunk `ch` of row `row` in a 64B-swizzled region of 64-byte rows
__host__ __device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t ch) {
    return row * 64u + ((ch ^ ((row >> 1) & 3u)) << 4);
}
__host__ __device__ __forceinline__ uint32_t ns16(uint32_t row, uint32_t k) {
    return (row >> 3) * 256u + (k >> 3) * 128u + (row & 7u) * 16u + (k & 7u) * 2u;
}

// Workspace of the fast path (after the common status word and g).
struct FastWs {
    size_t img, dO, dQ, dK, dV, D, Pa, Pds, rparts, wparts, bparts, r2, dg, total;
    int n_rparts, wsplits, bsplits, rsplits, npad;
};

inline int row_blocks(const eaga_dims &d) { return ((d.n + TB - 1) / TB) * d.B; }
constexpr int RPART = DE * NF + NH * DE + NF;            // dWfe, dWe, dg per (graph, row block)
inline int wgrad_splits(const eaga_dims &d) {
    const int rows = d.B * d.n;
    int s = rows / 512;
    return s < 1 ? 1 : (s > 32 ? 32 : s);
}

inline FastWs fast_ws(const eaga_dims &d, size_t base) {
    FastWs W;
    const size_t rows = size_t(d.B) * d.n;
    size_t off = base;
    W.img = off; off = align256(off + IMG_BYTES);
    W.dO = off; off = align256(off + rows * HD * 2);
    W.dQ = off; off = align256(off + rows * HD * 2);
    W.dK = off; off = align256(off + rows * HD * 2);
    W.dV = off; off = align256(off + rows * HD * 2);
    W.D = off; off = align256(off + size_t(d.B) * NH * d.n * 4);
    // a and ds of every pair, [B][H][n][npad] bf16, for the dk / dv pass
    W.npad = (d.n + 7) / 8 * 8;
    W.Pa = off; off = align256(off + size_t(d.B) * NH * d.n * W.npad * 2);
    W.Pds = off; off = align256(off + size_t(d.B) * NH * d.n * W.npad * 2);
    W.n_rparts = row_blocks(d);
    W.rparts = off; off = align256(off + size_t(W.n_rparts) * RPART * 4);
    W.wsplits = wgrad_splits(d);
    // split-K partials of dWq, dWk, dWv [dx, 256] and dWo [256, dx]
    W.wparts = off; off = align256(off + size_t(W.wsplits) * 4 * d.dx * HD * 4);
    W.bsplits = 64;
    W.bparts = off; off = align256(off + size_t(W.bsplits) * (3 * HD + d.dx) * 4);
    W.rsplits = 32;
    W.r2 = off; off = align256(off + size_t(W.rsplits) * (DE * NF + NH * DE) * 4);
    W.dg = off; off = align256(off + size_t(d.B) * NF * 4);
    W.total = off;
    return W;
}

bool encode_pair_map(CUtensorMap *m, const void *base, int B, int n, bool transposed, int box_rows, int box_s = 2);
bool encode_node_map(CUtensorMap *m, const void *base, int B, int n, int box_rows);
bool encode_p_map(CUtensorMap *m, const void *base, int B, int n, int npad);


// ------------------------------------------------------------------ device pieces
// The pair kernels run 16 warps.  Warp W owns TMEM lane quadrant q = W % 4
// (the pairs of chunk rows 8q+t/4 (+32 when NR = 2)) and the two heads
// 2hq, 2hq+1 with hq = W / 4.  Tile (r,s) of an [s][32NR][4][64] pair tile
// holds 128 pairs: chunk rows 32r..32r+31 with own-row parity s.
namespace dev {
using namespace sm100;
constexpr int NWARP = 16, NTHR = 512;
constexpr float LOG2E = 1.4426950408889634f;

template <int NR>
__device__ __forceinline__ uint32_t tile_off(int e) {   // byte offset of pair group e = 2r + s
    return (e & 1) * NR * 16384 + (e >> 1) * 16384;
}

// One thread issues D[e] (+)= tile(e) x B for the 2NR pair groups of a pair
// tile (FiLM with B = Wfe^T, u with B = We), K = 64 in four steps.
template <int NR>
__device__ __forceinline__ void issue_pair_products(uint32_t tile, uint32_t bimg, uint32_t tm_col) {
    const uint32_t idesc = idesc_bf16_f32(128, NF);
#pragma unroll
    for (int e = 0; e < 2 * NR; ++e) {
        const uint32_t a0 = tile + tile_off<NR>(e);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tm_col + 16 * e, smem_desc(a0 + kk * 32, 16, 1024, LAYOUT_SW128),
                        smem_desc(bimg + kk * 32, 16, 1024, LAYOUT_SW128), idesc, kk > 0);
    }
}

// B-operand fragments of 8 node rows base+g8 for heads 2hq, 2hq+1 (zero past n).
__device__ __forceinline__ void load_frags2(const __nv_bfloat16 *X, int b, int n, int base, int hq, int g8, int c4,
                                            uint32_t (&f)[2][2][2]) {
    const int r = base + g8;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int d = (2 * hq + hh) * DH + kk * 16 + 2 * c4;
            uint32_t lo = 0, hi = 0;
            if (r < n) {
                const __nv_bfloat16 *row = X + ((size_t)b * n + r) * HD;
                lo = *reinterpret_cast<const uint32_t *>(row + d);
                hi = *reinterpret_cast<const uint32_t *>(row + d + 8);
            }
            f[hh][kk][0] = lo;
            f[hh][kk][1] = hi;
        }
}

// Chunk row of ldmatrix lane t for the m16 tile of quadrant q: rows 8q.. for
// the first 8 and 32+8q.. for the second 8 (NR = 2); with NR = 1 the second 8
// repeat the first (their products are never used).
template <int NR>
__device__ __forceinline__ int frag_row(int q, int t, int second) {
    return (NR == 2 && second ? 32 : 0) + 8 * q + (t & 7);
}

// acc[hh][e] = X_rows . Y_cols over dh for heads 2hq+hh: X from a [32NR][256]
// swizzled chunk (4 boxes of 64 features), Y from fragments.
template <int NR>
__device__ __forceinline__ void warp_scores2(uint32_t chunk, int q, int t, int hq, const uint32_t (&yf)[2][2][2],
                                             float (&acc)[2][4]) {
    const int mrow = frag_row<NR>(q, t, (t >> 3) & 1);
    const int mch = t >> 4;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        acc[hh][0] = acc[hh][1] = acc[hh][2] = acc[hh][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const int h = 2 * hq + hh;
            const int ch = ((h & 1) * 32 + kk * 16) / 8 + mch;
            uint32_t a[4];
            ldsm_x4(chunk + (h >> 1) * (NR * 4096) + sw128(mrow, ch), a);
            mma16816(acc[hh], a, yf[hh][kk][0], yf[hh][kk][1]);
        }
    }
}

// acc[hh][mt] (+)= Z^T[d, chunk rows] P[chunk rows, 8 cols] for heads 2hq+hh: Z
// from the warp's rows of a [32NR][256] swizzled chunk, P the warp's m16n8
// fragment (entries 2,3 are ignored when NR = 1).
template <int NR, bool ACC = false>
__device__ __forceinline__ void warp_contract2(uint32_t chunk, int q, int t, int hq, const float (&pv)[2][4],
                                               float (&acc)[2][2][4]) {
    const int vrow = frag_row<NR>(q, t, (t >> 4) & 1);
    const int vch = (t >> 3) & 1;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const uint32_t b0 = movmatrix_t(pack_bf16(pv[hh][0], pv[hh][1]));
        const uint32_t b1 = NR == 2 ? movmatrix_t(pack_bf16(pv[hh][2], pv[hh][3])) : 0u;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            if (!ACC) acc[hh][mt][0] = acc[hh][mt][1] = acc[hh][mt][2] = acc[hh][mt][3] = 0.f;
            const int d0 = (2 * hq + hh) * DH + mt * 16;
            uint32_t a[4];
            ldsm_x4_t(chunk + (d0 >> 6) * (NR * 4096) + sw128(vrow, (d0 & 63) / 8 + vch), a);
            mma16816(acc[hh][mt], a, b0, b1);
        }
    }
}

// Store this warp's [8 i][256 d] contribution (2 heads) into quadrant slot q
// of a [4][8][256] fp32 buffer (32 KB).
__device__ __forceinline__ void store_quadrant_part(uint8_t *sp, uint32_t s_part, const float (&acc)[2][2][4], int q,
                                                    int hq, int t) {
    const int c4 = t & 3, g8 = t >> 2;
    float *dst = reinterpret_cast<float *>(sp + s_part) + q * TB * HD;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int d = (2 * hq + hh) * DH + mt * 16 + g8 + 8 * (e >> 1), il = 2 * c4 + (e & 1);
                dst[il * HD + d] = acc[hh][mt][e];
            }
}

// Cluster-wide sum of NB quadrant buffers (each [4][8][256] fp32, written by
// store_quadrant_part on every CTA of the cluster): this CTA reduces its
// 1/nclu slice, one quadrant per lane, all peer loads in flight, quadrants
// combined by shuffles in a fixed order.  Writes rows base+il < n of out[k]
// ([B,n,256] bf16) times scale[k].  Starts with a cluster barrier; ends with
// cluster_arrive(): the caller executes cluster_wait() before its shared
// memory can be reused or the CTA exits.
template <int NB>
__device__ __forceinline__ void cluster_reduce_rows(uint32_t sbase, const uint32_t (&s_part)[NB], int tid,
                                                    uint32_t rank, uint32_t nclu, __nv_bfloat16 *const (&out)[NB],
                                                    int b, int n, int base, const float (&scale)[NB]) {
    cluster_sync();
    constexpr int G = TB * HD / 4;                       // float4 groups per buffer
    const int per = (NB * G + nclu - 1) / nclu;
    const int lo = rank * per, hi = min((int)(rank + 1) * per, NB * G);
    const int q = tid & 3;
    for (int x0 = lo; x0 < hi; x0 += NTHR / 4) {
        const int x = x0 + (tid >> 2);
        const bool act = x < hi;
        const int k = act ? x / G : 0, gq = act ? x % G : 0;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        if (act) {
            const uint32_t off = s_part[k] + (q * G + gq) * 16;
            for (uint32_t p0 = 0; p0 < nclu; p0 += 4) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    v[u] = (p0 + u < nclu) ? ld_peer_f32x4(map_peer(sbase + off, p0 + u)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    a.x += v[u].x; a.y += v[u].y; a.z += v[u].z; a.w += v[u].w;
                }
            }
        }
#pragma unroll
        for (int o = 1; o < 4; o <<= 1) {
            a.x += __shfl_xor_sync(0xffffffffu, a.x, o);
            a.y += __shfl_xor_sync(0xffffffffu, a.y, o);
            a.z += __shfl_xor_sync(0xffffffffu, a.z, o);
            a.w += __shfl_xor_sync(0xffffffffu, a.w, o);
        }
        if (act && q == 0) {
            const int il = (gq * 4) / HD, d = (gq * 4) % HD;
            if (base + il < n) {
                const float sc = scale[k];
                __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(out[k] + ((size_t)b * n + base + il) * HD + d);
                o2[0] = __floats2bfloat162_rn(a.x * sc, a.y * sc);
                o2[1] = __floats2bfloat162_rn(a.z * sc, a.w * sc);
            }
        }
    }
    cluster_arrive();
}

// Cluster-wide combine of per-CTA (row, head) values: 64 entries, this CTA
// reads entry x from every peer (thread = (x, peer group of 8)) and combines
// in a fixed order.  Mode 0: softmax (max, sum) pairs at s_in (8 bytes per
// entry) -> (max, 1/sum) at s_out; mode 1: sums of one float at s_in -> s_out.
template <int MODE>
__device__ __forceinline__ void cluster_combine64(uint8_t *sp, uint32_t sbase, uint32_t s_in, uint32_t s_out,
                                                  int tid, uint32_t nclu) {
    const int x = tid >> 3, p = tid & 7;      // 64 entries x 8 lanes
    constexpr uint32_t STRIDE = MODE == 0 ? 8 : 4;
    float m0 = -INFINITY, l0 = 0.f, m1 = -INFINITY, l1 = 0.f;
    if ((uint32_t)p < nclu) {
        const uint32_t a = map_peer(sbase + s_in + x * STRIDE, p);
        if (MODE == 0) { m0 = ld_peer_f32(a); l0 = ld_peer_f32(a + 4); } else { l0 = ld_peer_f32(a); }
    }
    if ((uint32_t)(p + 8) < nclu) {
        const uint32_t a = map_peer(sbase + s_in + x * STRIDE, p + 8);
        if (MODE == 0) { m1 = ld_peer_f32(a); l1 = ld_peer_f32(a + 4); } else { l1 = ld_peer_f32(a); }
    }
    if (MODE == 0) {
        float m = fmaxf(m0, m1);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        if (m != -INFINITY) {
            if (m0 != -INFINITY) l += l0 * exp2f((m0 - m) * LOG2E);
            if (m1 != -INFINITY) l += l1 * exp2f((m1 - m) * LOG2E);
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (p == 0) {
            float *fo = reinterpret_cast<float *>(sp + s_out);
            fo[x * 2] = m;
            fo[x * 2 + 1] = l;   // sum (the caller turns it into 1/sum)
        }
    } else {
        float l = l0 + l1;
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (p == 0) reinterpret_cast<float *>(sp + s_out)[x] = l;
    }
}

// ---- push-based cluster exchanges (no cluster barrier on the critical path)
// Every CTA initialises its receive mbarriers, arms them with the bytes its
// peers will send (expect_tx), then cluster_arrive(); the matching
// cluster_wait() precedes its first push.  Each receiver waits only on its
// own mbarrier, so no CTA ever reads a peer's shared memory.

constexpr uint32_t RECV_ROWVALS_BYTES = 16 * 64 * 8;             // [16 peers][64 entries][8 bytes]
__host__ __device__ constexpr uint32_t recv_rows_bytes(int NB) {  // [nclu][per] float4, per = ceil(NB*512/nclu)
    return (uint32_t)(NB * 512 + 16) * 16;
}
__host__ __device__ inline uint32_t rows_per(int NB, uint32_t nclu) { return (NB * 512 + nclu - 1) / nclu; }
__host__ __device__ inline uint32_t rows_slice(int NB, uint32_t nclu, uint32_t r) {
    const int per = (int)rows_per(NB, nclu), lo = (int)r * per, hi = min(NB * 512, lo + per);
    return hi > lo ? (uint32_t)(hi - lo) : 0u;
}

// Push this CTA's 64 (row, head) values (v0, v1) from s_src ([64][2] f32) to
// slot `rank` of every CTA's receive buffer s_recv.
__device__ __forceinline__ void push_rowvals(uint8_t *sp, uint32_t sbase, uint32_t s_src, uint32_t s_recv,
                                             uint32_t bar, int tid, uint32_t rank, uint32_t nclu) {
    const int x = tid >> 3, p0 = tid & 7;
    const float *src = reinterpret_cast<const float *>(sp + s_src);
    const float v0 = src[x * 2], v1 = src[x * 2 + 1];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const uint32_t p = p0 + 8 * u;
        if (p < nclu)
            st_async_v2(map_peer(sbase + s_recv + (rank * 64 + x) * 8, p), v0, v1, map_peer(bar, p));
    }
}

// Combine the nclu received copies of the 64 entries in a fixed order.
// MODE 0: softmax (max, sum) pairs -> (max, sum) at s_out; MODE 1: sums of v0.
template <int MODE>
__device__ __forceinline__ void combine_rowvals(uint8_t *sp, uint32_t s_recv, uint32_t s_out, int tid,
                                                uint32_t nclu) {
    const int x = tid >> 3, p = tid & 7;
    const float *rv = reinterpret_cast<const float *>(sp + s_recv);
    float m0 = -INFINITY, l0 = 0.f, m1 = -INFINITY, l1 = 0.f;
    if ((uint32_t)p < nclu) { m0 = rv[(p * 64 + x) * 2]; l0 = rv[(p * 64 + x) * 2 + 1]; }
    if ((uint32_t)(p + 8) < nclu) { m1 = rv[((p + 8) * 64 + x) * 2]; l1 = rv[((p + 8) * 64 + x) * 2 + 1]; }
    float *fo = reinterpret_cast<float *>(sp + s_out);
    if (MODE == 0) {
        float m = fmaxf(m0, m1);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        float l = 0.f;
        if (m != -INFINITY) {
            if (m0 != -INFINITY) l += l0 * exp2f((m0 - m) * LOG2E);
            if (m1 != -INFINITY) l += l1 * exp2f((m1 - m) * LOG2E);
        }
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (p == 0) { fo[x * 2] = m; fo[x * 2 + 1] = l; }
    } else {
        float l = ((uint32_t)p < nclu ? m0 : 0.f) + ((uint32_t)(p + 8) < nclu ? m1 : 0.f);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        if (p == 0) fo[x] = l;
    }
}

// Sum the NSLOT slot partials of NB [NSLOT][8][256] fp32 buffers and push
// float4 group gg (over the NB buffers) to its owner rank gg / per, slot
// rank * per + (gg - owner * per) of the owner's receive buffer.
template <int NB, int NSLOT = 4>
__device__ __forceinline__ void push_rows_partials(uint8_t *sp, uint32_t sbase, const uint32_t (&s_part)[NB],
                                                   uint32_t s_recv, uint32_t bar, int tid, uint32_t rank,
                                                   uint32_t nclu) {
    constexpr int G = TB * HD / 4;
    const uint32_t per = rows_per(NB, nclu);
    for (int gg = tid; gg < NB * G; gg += NTHR) {
        const int k = gg / G, g = gg % G;
        const float4 *pt = reinterpret_cast<const float4 *>(sp + s_part[k]);
        float4 v = pt[g];
#pragma unroll
        for (int qq = 1; qq < NSLOT; ++qq) {
            const float4 w = pt[qq * G + g];
            v.x += w.x; v.y += w.y; v.z += w.z; v.w += w.w;
        }
        const uint32_t owner = gg / per, slot = rank * per + (gg - owner * per);
        st_async_v4(map_peer(sbase + s_recv + slot * 16, owner), v, map_peer(bar, owner));
    }
}

// The warps' [8 i][256 d] contributions summed over the 4 quadrants in two
// fixed-order phases into a [2][8][256] fp32 buffer (16 KB): quadrants 0,1
// write slots 0,1, then quadrants 2,3 add into them.  All threads call it.
__device__ __forceinline__ void store_quadrant_part_2ph(uint8_t *sp, uint32_t s_part, const float (&acc)[2][2][4],
                                                        int q, int hq, int t) {
    const int c4 = t & 3, g8 = t >> 2;
    float *dst = reinterpret_cast<float *>(sp + s_part) + (q & 1) * TB * HD;
    for (int phase = 0; phase < 2; ++phase) {
        if ((q >> 1) == phase) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int d = (2 * hq + hh) * DH + mt * 16 + g8 + 8 * (e >> 1), il = 2 * c4 + (e & 1);
                        float *x = dst + il * HD + d;
                        *x = (phase ? *x : 0.f) + acc[hh][mt][e];
                    }
        }
        __syncthreads();
    }
}

// Push 64 per-(row, head) floats src[x] to slot `rank` of every CTA's
// receive buffer s_recv ([16][64] f32).
__device__ __forceinline__ void push_rowvals_f32(uint8_t *sp, uint32_t sbase, uint32_t s_src, uint32_t s_recv,
                                                 uint32_t bar, int tid, uint32_t rank, uint32_t nclu) {
    const int x = tid >> 3, p0 = tid & 7;
    const float v = reinterpret_cast<const float *>(sp + s_src)[x];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const uint32_t pp = p0 + 8 * u;
        if (pp < nclu) st_async_f32(map_peer(sbase + s_recv + (rank * 64 + x) * 4, pp), v, map_peer(bar, pp));
    }
}

// Sum of the nclu received copies of 64 floats ([16][64] f32), fixed order.
__device__ __forceinline__ void combine_rowvals_f32(uint8_t *sp, uint32_t s_recv, uint32_t s_out, int tid,
                                                    uint32_t nclu) {
    const int x = tid >> 3, pp = tid & 7;
    const float *rv = reinterpret_cast<const float *>(sp + s_recv);
    float l = ((uint32_t)pp < nclu ? rv[pp * 64 + x] : 0.f) + ((uint32_t)(pp + 8) < nclu ? rv[(pp + 8) * 64 + x] : 0.f);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (pp == 0) reinterpret_cast<float *>(sp + s_out)[x] = l;
}

// Push a flat fp32 array of `count` floats (count % 4 == 0) to its owners:
// float4 group g goes to rank g / per4 (per4 = ceil(count/4 / nclu)), slot
// rank * per4 + (g - owner * per4) of the owner's receive buffer.
__device__ __forceinline__ void push_flat(uint8_t *sp, uint32_t sbase, uint32_t s_src, int count, uint32_t s_recv,
                                          uint32_t bar, int tid, uint32_t rank, uint32_t nclu) {
    const int g4 = count / 4;
    const uint32_t per = (g4 + nclu - 1) / nclu;
    const float4 *src = reinterpret_cast<const float4 *>(sp + s_src);
    for (int g = tid; g < g4; g += NTHR) {
        const uint32_t owner = g / per, slot = rank * per + (g - owner * per);
        st_async_v4(map_peer(sbase + s_recv + slot * 16, owner), src[g], map_peer(bar, owner));
    }
}
__host__ __device__ inline uint32_t flat_slice(int count, uint32_t nclu, uint32_t r) {
    const int g4 = count / 4, per = (g4 + (int)nclu - 1) / (int)nclu, lo = (int)r * per, hi = min(g4, lo + per);
    return hi > lo ? (uint32_t)(hi - lo) : 0u;
}

// Owner side: after its receive mbarrier completed, sum the nclu pushed
// copies of its groups (fixed order) and write rows base+il < n of out[k].
template <int NB>
__device__ __forceinline__ void finish_rows_partials(uint8_t *sp, uint32_t s_recv, int tid, uint32_t rank,
                                                     uint32_t nclu, __nv_bfloat16 *const (&out)[NB], int b, int n,
                                                     int base, const float (&scale)[NB]) {
    constexpr int G = TB * HD / 4;
    const uint32_t per = rows_per(NB, nclu), slice = rows_slice(NB, nclu, rank);
    const float4 *rv = reinterpret_cast<const float4 *>(sp + s_recv);
    for (uint32_t k0 = tid; k0 < slice; k0 += NTHR) {
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (uint32_t p = 0; p < nclu; ++p) {
            const float4 v = rv[p * per + k0];
            a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
        }
        const int gg = rank * per + k0, k = gg / G, g = gg % G;
        const int il = (g * 4) / HD, d = (g * 4) % HD;
        if (base + il < n) {
            const float sc = scale[k];
            __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(out[k] + ((size_t)b * n + base + il) * HD + d);
            o2[0] = __floats2bfloat162_rn(a.x * sc, a.y * sc);
            o2[1] = __floats2bfloat162_rn(a.z * sc, a.w * sc);
        }
    }
}

// In-place residual on a 128-byte swizzled pair row: row[c] += dv[c - 16hq]
// for the 16 channels c in [16hq, 16hq + 16), rounded to bf16.
__device__ __forceinline__ void add_residual16(uint8_t *row, uint32_t L, int hq, const float (&dv)[16]) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const uint32_t ch = 2 * hq + hh;
        uint4 *ptr = reinterpret_cast<uint4 *>(row + ((ch ^ (L & 7u)) << 4));
        uint4 ev = *ptr;
        __nv_bfloat162 *e2 = reinterpret_cast<__nv_bfloat162 *>(&ev);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float2 x = __bfloat1622float2(e2[u]);
            e2[u] = __floats2bfloat162_rn(x.x + dv[8 * hh + 2 * u], x.y + dv[8 * hh + 2 * u + 1]);
        }
        *ptr = ev;
    }
}

__device__ __forceinline__ void flag_timeout(int *status) { atomicExch(status, DEV_TIMEOUT); }
}  // namespace dev
}  // namespace fast
}  // namespace eaga
