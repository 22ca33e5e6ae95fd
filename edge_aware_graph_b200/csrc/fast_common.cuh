// Shared constants, workspace layout and device helpers of the specialised
// sm_100a path (de = 64, H = 8, dh = 32, bf16 storage).
#pragma once
#include <cuda.h>
#include <utility>
#include "common.cuh"
#include "sm100.cuh"

namespace eaga {
namespace fast {

constexpr int DE = 64, NH = 8, DH = 32, HD = 256, NF = 16;
constexpr int TB = 8;            // query rows per pair-kernel CTA (one row block)
// Streaming multiprocessors of the current device.
inline int sm_count() {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        v > 0)
        return v;
    return 148;
}

// Launch of a kernel that may start behind the previous kernel of its stream
// (programmatic stream serialisation): its CTAs become resident while that
// kernel's last CTAs finish and wait in griddep_wait before touching global
// memory.  cluster > 1 adds a cluster dimension.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
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

// Workspace of the fast path (after the common status word and g).  Every
// region grows with the node count B*n (or is fixed): no per-pair buffer.
struct FastWs {
    size_t img, dO, dQ, dK, dV, dK32, dV32, rparts, wparts, bparts, r2, dg, order, total;
    int n_rparts, wsplits, bsplits, rsplits;
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
    // fp32 accumulators of dk (unscaled) and dv [B*n, 256], summed over row blocks in L2
    W.dK32 = off; off = align256(off + rows * HD * 4);
    W.dV32 = off; off = align256(off + rows * HD * 4);
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
    // the order in which the backward pair kernel's CTAs take the row blocks
    W.order = off; off = align256(off + size_t(row_blocks(d)) * 4);
    W.total = off;
    return W;
}

bool encode_pair_map(CUtensorMap *m, const void *base, int B, int rows, int n, int box_rows, int box_s = 2);
bool encode_node_map(CUtensorMap *m, const void *base, int B, int n, int box_rows);


// ------------------------------------------------------------------ device pieces
// The pair kernels run 16 compute warps.  Warp W owns TMEM lane quadrant
// q = W % 4 (the pairs of chunk columns 8q + t/4) and the two heads 2hq,
// 2hq+1 with hq = W / 4.  A chunk is 32 columns j of the CTA's 8 rows i, held
// as two [32 j][4 ic][64 c] tiles (i = 2ic + s, one per parity s): 256 pairs.
// The helpers keep an NR parameter: NR = 1 is the 32-column chunk.
namespace dev {
using namespace sm100;
constexpr int NWARP = 16, NTHR = 512;
constexpr float LOG2E = 1.4426950408889634f;

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

// Residual of a 128-byte swizzled pair row written to global memory: dst[c] =
// row[c] (+ dv[c - 16hq] when `add`) for the 16 channels c in [16hq, 16hq + 16),
// rounded to bf16, two 16-byte streaming stores (the row itself is unchanged).
__device__ __forceinline__ void residual16_to_global(const uint8_t *row, uint32_t L, int hq, const float (&dv)[16],
                                                     bool add, __nv_bfloat16 *dst) {
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const uint32_t ch = 2 * hq + hh;
        uint4 ev = *reinterpret_cast<const uint4 *>(row + ((ch ^ (L & 7u)) << 4));
        if (add) {
            __nv_bfloat162 *e2 = reinterpret_cast<__nv_bfloat162 *>(&ev);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 x = __bfloat1622float2(e2[u]);
                e2[u] = __floats2bfloat162_rn(x.x + dv[8 * hh + 2 * u], x.y + dv[8 * hh + 2 * u + 1]);
            }
        }
        __stcs(reinterpret_cast<uint4 *>(dst) + hh, ev);
    }
}

__device__ __forceinline__ void flag_timeout(int *status) { atomicExch(status, DEV_TIMEOUT); }

// Block sparsity of a row block (the rows i0 .. i0+TB-1 of graph b): bit c is
// set when chunk c (columns 32c .. 32c+31) holds at least one valid pair, i.e.
// some row of the block and some column of the chunk are nodes of the graph.
// Every other pair of the chunk has a = 0, so its outputs are its inputs (E' =
// E, dE = dE') and it adds nothing to any sum.  One warp; every lane returns
// the mask.  n is even, so the mask row is 2-byte aligned.
__device__ __forceinline__ uint32_t live_chunk_mask(const uint8_t *M, int b, int n, int i0, int t) {
    const uint8_t *mb = M + (size_t)b * n;
    const bool row = t < TB && i0 + t < n && mb[i0 + t] != 0;
    if (!__any_sync(0xffffffffu, row)) return 0u;
    const uint16_t *m2 = reinterpret_cast<const uint16_t *>(mb);
    uint32_t any = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int j = 32 * t + 2 * k;
        if (j < n) any |= m2[j >> 1];
    }
    return __ballot_sync(0xffffffffu, any != 0);
}

// Largest number of row blocks that k_row_block_order sorts (its keys live
// in 48 KB of shared memory); beyond it the CTAs take the row blocks in order.
constexpr int ORDER_MAX_ITEMS = 12288;

// Position of the k-th (from 0) set bit of m; m has more than k bits set.
__device__ __forceinline__ int nth_set_bit(uint32_t m, int k) {
    for (int x = 0; x < k; ++x) m &= m - 1u;
    return __ffs(m) - 1;
}

// Bounded wait on phase `parity` of mbarrier `bar` that gives up for the
// whole CTA.  `fail` is a flag in shared memory, zero at the start.  The
// first wait of the CTA that runs out of polls sets it and records
// DEV_TIMEOUT in the status word; from then on every wait returns false at
// once (a thread already waiting notices within 256 polls), the issuing
// threads stop issuing TMA copies and MMAs, and the CTA runs its remaining
// control flow (the same named barriers, in-bounds addresses) to the end,
// where it waits, again with a bound, for what it already issued and frees
// its tensor memory.  A stalled CTA therefore costs about one bound, not one
// bound per wait.  (Polls without a suspend-time hint: sleeping between
// polls was measured slower, the wake-up sits on the critical path.)
__device__ __forceinline__ bool cta_wait(uint32_t bar, uint32_t parity, volatile int *fail, int *status,
                                         uint32_t limit = (1u << 24)) {
    if (*fail) return false;
    for (uint32_t it = 0; it < limit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && *fail) return false;
    }
    *fail = 1;
    flag_timeout(status);
    return false;
}
}  // namespace dev
}  // namespace fast
}  // namespace eaga
