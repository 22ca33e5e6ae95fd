// Edge sub-block of the graph-transformer block around the layer, fused per
// tile of 128 pairs (sm_100a, de = 64, FFN width 128, bf16 storage).
//
// The layer sits in DeFoG's graph-transformer backbone, which updates node,
// edge and global features jointly (AI-summary page, method paragraph; paper
// index page, abstract).  The pages print no equations for the block; the
// edge part taken here is the plain post-norm one:
//   Ea   = LN(E'; g1, s1)
//   Ez   = Ea + relu(Ea W1 + b1) W2 + b2
//   Eout = valid_ij * LN(Ez; g2, s2)
// with LN over the 64 channels of a pair (biased variance, eps 1e-5).
//
// k_eblk_fwd streams tiles of 4 rows i x 32 columns j (128 pairs, 16 KB) of
// E' through shared memory: the LayerNorms run per pair in registers (thread
// r owns pair r, TMEM lane r), the two FFN products run on the tensor cores
// (tcgen05, M = 128, fp32 in TMEM: Ea W1 is 128 x 128 over K = 64, H W2 is
// 128 x 64 over K = 128), and the result is written in place into the tile and
// stored with TMA: E' is read once and Eout written once.  A tile without a
// valid pair is not read; it is stored as zeros.  The same pass adds the valid
// pairs' E' into per-graph sums for the global update's edge pooling.
//
// k_eblk_bwd recomputes the forward of a tile from E' and runs its chain rule:
//   dEz = LN^T(valid * dEout; g2)      dg2 += dEout x2, ds2 += dEout
//   dh  = dEz W2^T [Ea W1 + b1 > 0]    dW2 += h^T dEz,   db2 += dEz
//   dEa = dEz + dh W1^T                dW1 += Ea^T dh,   db1 += dh
//   dE' = valid * (LN^T(dEa; g1) + dpE_b)               dg1 += dEa x1, ds1 += dEa
// (dpE_b: the global update's gradient of the edge pooling, already divided
// by the pair count).  The four products and the two weight-gradient products
// (M = 128 over the tile's 128 pairs, accumulated in TMEM over the CTA's
// tiles) run on the tensor cores; the per-channel sums are column sums on
// the warps' tensor cores (a ones matrix times the warp's rows staged as bf16
// in a tile already held); each CTA writes its partial sums once.
//
// Four warps, one pair row per thread; thread 0 also issues the MMAs (after
// a named barrier of the CTA) and the TMA loads and stores, and warp 0 loads
// the node-mask bytes of a tile one tile before its validity masks are
// needed.  The forward double-buffers its tiles (the next tile's load is
// issued with the current tile's first product) and keeps h in tensor memory
// as the A operand of h W2, so three CTAs fit an SM; the backward holds one
// tile pair, prefetches the next into L2 and runs two CTAs per SM (8 warps:
// 255 registers a thread).  Persistent grids, tiles taken in a stride of the
// grid size.
#include "fast.h"
#include "fast_common.cuh"
#include "fast_block.h"

namespace eaga {
namespace fast {
namespace blk {

using namespace sm100;
using dev::cta_wait;

constexpr int EB_THR = 128;                   // four warps, one pair row per thread
constexpr int EF = 128;                       // FFN width of the edge sub-block (2 de)
constexpr uint32_t EB_TILE = 16384;           // 128 pairs x 64 channels bf16
constexpr float LN_EPS = 1e-5f;

// Forward shared memory (bytes from a 1024-aligned base).
struct EfSmem {
    static constexpr uint32_t SLOT = 0;                  // 2 x 16 KB: E' tile -> Ea -> output
    static constexpr uint32_t W1 = 2 * EB_TILE;          // W1 [64][128] as two 64 x 64 boxes (8 KB each)
    static constexpr uint32_t W2 = W1 + EB_TILE;         // W2 [128][64] as one box
    static constexpr uint32_t PAR = W2 + EB_TILE;        // fp32: g1, s1 [64], b1 [128], b2, g2, s2 [64]
    static constexpr uint32_t INFO = PAR + 448 * 4;      // per slot: column mask, row mask | live << 8
    static constexpr uint32_t BAR = INFO + 16;           // full[2], mma, wts
    static constexpr uint32_t TM = BAR + 4 * 8;
    static constexpr uint32_t FAIL = TM + 8;
    static constexpr uint32_t BYTES = FAIL + 8 + 1024;
};
static_assert(EfSmem::BYTES <= 74 * 1024, "three CTAs per SM");
// TMEM columns of the forward: Ea W1 (fp32) 0..127; then h (bf16 pairs) 0..63
// as the A operand of h W2, whose result lands in 64..127
constexpr uint32_t EF_TM_COLS = 128, EF_TM_Z = 64;
constexpr int PAR_G1 = 0, PAR_S1 = 64, PAR_B1 = 128, PAR_B2 = 256, PAR_G2 = 320, PAR_S2 = 384;

// Backward shared memory: one E' tile (-> Ea), one dEout tile (-> dEz -> dE'),
// H (h -> dh), the weights and the parameters.
struct EbSmem {
    static constexpr uint32_t SA = 0;
    static constexpr uint32_t SB = EB_TILE;
    static constexpr uint32_t H = 2 * EB_TILE;
    static constexpr uint32_t W1 = H + 2 * EB_TILE;
    static constexpr uint32_t W2 = W1 + EB_TILE;
    static constexpr uint32_t PAR = W2 + EB_TILE;
    static constexpr uint32_t INFO = PAR + 448 * 4;
    static constexpr uint32_t BAR = INFO + 16;           // full, mma, wts
    static constexpr uint32_t TM = BAR + 3 * 8;
    static constexpr uint32_t FAIL = TM + 8;
    static constexpr uint32_t BYTES = FAIL + 8 + 1024;
};
static_assert(EbSmem::BYTES <= 113 * 1024, "two CTAs per SM");
// TMEM columns of the backward: the tile's products 0..127, dW2 128..191, dW1^T 192..255
constexpr uint32_t EB_TM_COLS = 256, EB_TM_DW2 = 128, EB_TM_DW1 = 192;

// Column sums over the warp's 32 rows (32 w .. 32 w + 31) of a 128B-swizzled
// [128][64] bf16 tile, on the warp's tensor cores: D = ones(16 x 16) B with B
// the tile's rows (pairs, K) by channels (N), 8 channel groups of 8, the two
// 16-row halves accumulated; every row of D is the column sum.  Lane l
// returns channels 2l, 2l + 1 (the D row's columns 2(l%4), 2(l%4)+1 of
// channel group l/4).
__device__ __forceinline__ float2 warp_tile_colsum(uint32_t tile, int w, int lane) {
    const uint32_t ones[4] = {0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u};
    const int j = lane >> 2;
    float v0 = 0.f, v1 = 0.f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        float da[4] = {0.f, 0.f, 0.f, 0.f}, db[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
            const uint32_t row = 32 * w + 16 * kb + (lane & 7) + 8 * ((lane >> 3) & 1);
            const uint32_t chunk = 2 * g + (lane >> 4);
            uint32_t q[4];
            ldsm_x4_t(tile + sw128(row, chunk), q);
            mma16816(da, ones, q[0], q[1]);
            mma16816(db, ones, q[2], q[3]);
        }
        if (j == 2 * g) {
            v0 = da[0];
            v1 = da[1];
        }
        if (j == 2 * g + 1) {
            v0 = db[0];
            v1 = db[1];
        }
    }
    return make_float2(v0, v1);
}

// Row r of a 128B-swizzled [128][64] bf16 tile from f(c), c = 0..63.
template <class F>
__device__ __forceinline__ void row_store_fn(uint8_t *tile, int r, F f) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(f(8 * c), f(8 * c + 1));
        u.y = pack_bf16(f(8 * c + 2), f(8 * c + 3));
        u.z = pack_bf16(f(8 * c + 4), f(8 * c + 5));
        u.w = pack_bf16(f(8 * c + 6), f(8 * c + 7));
        *reinterpret_cast<uint4 *>(tile + sw128(r, c)) = u;
    }
}

// Tile t of the grid of (graph, 4-row block, 32-column block).
struct TileAt {
    int b, i0, j0;
};
__device__ __forceinline__ TileAt tile_at(int t, int ti, int tj) {
    TileAt r;
    const int per = ti * tj;
    r.b = t / per;
    const int rem = t - r.b * per;
    r.i0 = (rem / tj) * 4;
    r.j0 = (rem % tj) * 32;
    return r;
}

// Validity masks of a tile (one warp; every lane returns both): bit jj of
// the column mask is set when column j0 + jj is a node, bit ii of the row mask
// when row i0 + ii is.
__device__ __forceinline__ void tile_masks(const uint8_t *M, int n, const TileAt &T, int lane, uint32_t &cm,
                                           uint32_t &rm) {
    const uint8_t *mb = M + (size_t)T.b * n;
    const bool c = T.j0 + lane < n && mb[T.j0 + lane] != 0;
    const bool r = lane < 4 && T.i0 + lane < n && mb[T.i0 + lane] != 0;
    cm = __ballot_sync(0xffffffffu, c);
    rm = __ballot_sync(0xffffffffu, r) & 0xFu;
}

// The lane's node-mask bytes of tile t (column j0 + lane; row i0 + lane for
// lanes < 4; 0 outside the graph or past the last tile), loaded one tile
// before the ballot that turns them into the tile's masks, so the load's
// latency is hidden behind a tile of work.
__device__ __forceinline__ void mask_bytes(const uint8_t *M, int n, int t, int ti, int tj, int ntile, int lane,
                                           uint32_t &c, uint32_t &r) {
    c = 0;
    r = 0;
    if (t >= ntile) return;
    const TileAt T = tile_at(t, ti, tj);
    const uint8_t *mb = M + (size_t)T.b * n;
    if (T.j0 + lane < n) c = mb[T.j0 + lane];
    if (lane < 4 && T.i0 + lane < n) r = mb[T.i0 + lane];
}

// Row r of a 128B-swizzled [128][64] bf16 tile <-> 64 fp32 values.
__device__ __forceinline__ void row_load64(const uint8_t *tile, int r, float (&x)[64]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 u = *reinterpret_cast<const uint4 *>(tile + sw128(r, c));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(h[k]);
            x[8 * c + 2 * k] = f.x;
            x[8 * c + 2 * k + 1] = f.y;
        }
    }
}
__device__ __forceinline__ void row_store64(uint8_t *tile, int r, const float (&x)[64]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 u;
        u.x = pack_bf16(x[8 * c], x[8 * c + 1]);
        u.y = pack_bf16(x[8 * c + 2], x[8 * c + 3]);
        u.z = pack_bf16(x[8 * c + 4], x[8 * c + 5]);
        u.w = pack_bf16(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128(r, c)) = u;
    }
}
__device__ __forceinline__ void row_zero(uint8_t *tile, int r) {
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4 *>(tile + sw128(r, c)) = make_uint4(0, 0, 0, 0);
}

// x <- (x - mean) / sqrt(var + eps) over 64 values; returns 1/sqrt(var + eps).
__device__ __forceinline__ float normalise64(float (&x)[64]) {
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) s += x[c];
    const float mean = s * (1.f / 64.f);
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        x[c] -= mean;
        q = fmaf(x[c], x[c], q);
    }
    const float r = rsqrtf(q * (1.f / 64.f) + LN_EPS);
#pragma unroll
    for (int c = 0; c < 64; ++c) x[c] *= r;
    return r;
}

// Parameters from shared memory four at a time (the arrays are 16-byte aligned).
__device__ __forceinline__ float4 par4(const float *par, int i) { return *reinterpret_cast<const float4 *>(par + i); }
// x = x g + s over 64 channels (g, s at par offsets), or 0 where !keep.
__device__ __forceinline__ void affine64(float (&x)[64], const float *par, int g, int s, bool keep = true) {
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
        const float4 a = par4(par, g + c), b = par4(par, s + c);
        x[c] = keep ? fmaf(x[c], a.x, b.x) : 0.f;
        x[c + 1] = keep ? fmaf(x[c + 1], a.y, b.y) : 0.f;
        x[c + 2] = keep ? fmaf(x[c + 2], a.z, b.z) : 0.f;
        x[c + 3] = keep ? fmaf(x[c + 3], a.w, b.w) : 0.f;
    }
}
// Four 16-column TMEM loads of the thread's lane into v[64], one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
    tmem_ld16(taddr, *reinterpret_cast<float(*)[16]>(v));
    tmem_ld16(taddr + 16, *reinterpret_cast<float(*)[16]>(v + 16));
    tmem_ld16(taddr + 32, *reinterpret_cast<float(*)[16]>(v + 32));
    tmem_ld16(taddr + 48, *reinterpret_cast<float(*)[16]>(v + 48));
    tmem_ld_wait();
}
// x += v + b over 64 channels (b at a par offset).
__device__ __forceinline__ void add_bias64(float (&x)[64], const float (&v)[64], const float *par, int b) {
#pragma unroll
    for (int c = 0; c < 64; c += 4) {
        const float4 q = par4(par, b + c);
        x[c] += v[c] + q.x;
        x[c + 1] += v[c + 1] + q.y;
        x[c + 2] += v[c + 2] + q.z;
        x[c + 3] += v[c + 3] + q.w;
    }
}

__device__ __forceinline__ void load_params(float *par, const EbParams &p, int tid, int nthr) {
    for (int c = tid; c < 448; c += nthr) {
        float v;
        if (c < 64) v = __bfloat162float(p.g1[c]);
        else if (c < 128) v = __bfloat162float(p.s1[c - 64]);
        else if (c < 256) v = __bfloat162float(p.b1[c - 128]);
        else if (c < 320) v = __bfloat162float(p.b2[c - 256]);
        else if (c < 384) v = __bfloat162float(p.g2[c - 320]);
        else v = __bfloat162float(p.s2[c - 384]);
        par[c] = v;
    }
}

// Issue A[128 x K] * B -> TMEM with A K-major 128B-swizzled tiles of 64
// columns (16 KB apart) and B as the weights' boxes (MN-major: k-steps of 16
// rows; K-major: 64-column boxes `bstep` apart).
__device__ __forceinline__ void mma_tile(uint32_t d, uint32_t a, int ksteps, uint32_t b, bool b_mn, uint32_t bstep,
                                         uint32_t idesc) {
#pragma unroll 1
    for (int kk = 0; kk < ksteps; ++kk) {
        const uint64_t ad = smem_desc(a + (kk >> 2) * EB_TILE + (kk & 3) * 32, 16, 1024, LAYOUT_SW128);
        const uint64_t bd = b_mn ? smem_desc(b + kk * 2048, 8192, 1024, LAYOUT_SW128)
                                 : smem_desc(b + (kk >> 2) * bstep + (kk & 3) * 32, 16, 1024, LAYOUT_SW128);
        mma_bf16_ss(d, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
}
// D[M = 128 channels][N = 64] (+)= A^T B over the tile's 128 pairs: A the two
// 64-channel halves of a [128 pairs][128] tile (16 KB apart), B a [128 pairs][64]
// tile, both read MN-major.
__device__ __forceinline__ void mma_wgrad(uint32_t d, uint32_t a, uint32_t b, bool accumulate) {
    const uint32_t idesc = idesc_bf16_f32_mn(128, 64);
#pragma unroll 1
    for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(d, smem_desc(a + kk * 2048, EB_TILE, 1024, LAYOUT_SW128),
                    smem_desc(b + kk * 2048, 8192, 1024, LAYOUT_SW128), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// The H epilogue of one pair row: h = relu(T + b1) for the 128 columns,
// written as bf16 into the two 64-channel halves of the H tile.
__device__ __forceinline__ void h_epilogue(uint8_t *Ht, int r, uint32_t tl, const float *b1) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float v[64];
        tmem_ld64(tl + 64 * hf, v);
        uint8_t *half = Ht + hf * EB_TILE;
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
#pragma unroll
            for (int u = 0; u < 16; u += 4) {
                const float4 q = par4(b1, 64 * hf + c0 + u);
                v[c0 + u] = fmaxf(v[c0 + u] + q.x, 0.f);
                v[c0 + u + 1] = fmaxf(v[c0 + u + 1] + q.y, 0.f);
                v[c0 + u + 2] = fmaxf(v[c0 + u + 2] + q.z, 0.f);
                v[c0 + u + 3] = fmaxf(v[c0 + u + 3] + q.w, 0.f);
            }
            const int ch = c0 >> 3;
            const float *w = v + c0;
            uint4 u0, u1;
            u0.x = pack_bf16(w[0], w[1]); u0.y = pack_bf16(w[2], w[3]);
            u0.z = pack_bf16(w[4], w[5]); u0.w = pack_bf16(w[6], w[7]);
            u1.x = pack_bf16(w[8], w[9]); u1.y = pack_bf16(w[10], w[11]);
            u1.z = pack_bf16(w[12], w[13]); u1.w = pack_bf16(w[14], w[15]);
            *reinterpret_cast<uint4 *>(half + sw128(r, ch)) = u0;
            *reinterpret_cast<uint4 *>(half + sw128(r, ch + 1)) = u1;
        }
    }
}

// The forward's H epilogue in tensor memory: h = relu(T + b1) for the 128
// columns of the thread's lane, stored back as bf16 pairs into columns
// 0..63 (the A operand of h W2: row = lane, K along the columns).  Columns
// are read 32 at a time in increasing order, so each store lands on columns
// already read.
__device__ __forceinline__ void h_epilogue_tmem(uint32_t tl, const float *b1) {
#pragma unroll
    for (int c0 = 0; c0 < EF; c0 += 32) {
        float v[32];
        tmem_ld16(tl + c0, *reinterpret_cast<float(*)[16]>(v));
        tmem_ld16(tl + c0 + 16, *reinterpret_cast<float(*)[16]>(v + 16));
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int u = 0; u < 16; u += 2) {
            const float4 q = par4(b1, c0 + 2 * u);
            pk[u] = pack_bf16(fmaxf(v[2 * u] + q.x, 0.f), fmaxf(v[2 * u + 1] + q.y, 0.f));
            pk[u + 1] = pack_bf16(fmaxf(v[2 * u + 2] + q.z, 0.f), fmaxf(v[2 * u + 3] + q.w, 0.f));
        }
        tmem_st16(tl + c0 / 2, pk);
    }
    tmem_st_wait();
}

// dh = dh' where the stored h > 0 (relu(x) > 0 exactly when x > 0), for 8
// channels held as one 16-byte chunk of the H tile.
__device__ __forceinline__ void relu_gate8(const uint4 hq, float *v) {
    const uint32_t w[4] = {hq.x, hq.y, hq.z, hq.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = (int16_t)(w[k] & 0xFFFFu) > 0 ? v[2 * k] : 0.f;        // a positive bf16, as int16
        v[2 * k + 1] = (int16_t)(w[k] >> 16) > 0 ? v[2 * k + 1] : 0.f;
    }
}

// Packed bf16 pairs <-> floats of a 64-channel row kept in 32 registers.
__device__ __forceinline__ float pk_get(const uint32_t (&p)[32], int c) {
    return __uint_as_float((c & 1) ? (p[c >> 1] & 0xFFFF0000u) : (p[c >> 1] << 16));
}

// ------------------------------------------------------------------ forward

// Thread 0: load tile t into slot `sl` (or mark it empty when the tile has no
// valid pair), after the bulk stores issued so far have read their tiles.
__device__ __forceinline__ void issue_tile(int t, int ntile, uint32_t slot_addr, uint32_t full, uint32_t *info,
                                           uint32_t cm, uint32_t rm, const CUtensorMap *map, const EbParams &p,
                                           volatile int *fail, uint32_t &issued) {
    if (t >= ntile) return;
    ++issued;                                    // one phase of `full` per call
    tma_store_wait_read0();
    const bool live = cm != 0 && rm != 0;
    info[0] = cm;
    info[1] = rm | (live ? 0x100u : 0u);
    if (live && !*fail) {
        const TileAt T = tile_at(t, p.ti, p.tj);
        mbar_expect_tx(full, EB_TILE);
        tma_load_4d(slot_addr, map, full, 0, T.j0, T.i0, T.b);
    } else {
        mbar_arrive(full);
    }
}

__global__ void __launch_bounds__(EB_THR, 3)
k_eblk_fwd(const __grid_constant__ CUtensorMap tmIn, const __grid_constant__ CUtensorMap tmOut,
           const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2, EbParams p) {
    using S = EfSmem;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);
    const uint32_t bar0 = sbase + S::BAR;
    auto full = [&](int s) { return bar0 + 8 * s; };
    const uint32_t mmab = bar0 + 16, wtsb = bar0 + 24;
    uint32_t *info = reinterpret_cast<uint32_t *>(sp + S::INFO);
    float *par = reinterpret_cast<float *>(sp + S::PAR);

    if (tid == 0) {
        mbar_init(full(0), 1);
        mbar_init(full(1), 1);
        mbar_init(mmab, 1);
        mbar_init(wtsb, 1);
        fence_mbar_init();
        *fail = 0;
    }
    if (w == 0) {
        tmem_alloc(sbase + S::TM, EF_TM_COLS);
        tmem_relinquish();
    }
    load_params(par, p, tid, EB_THR);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const int ntile = p.B * p.ti * p.tj, G = gridDim.x;
    const int r = tid;                           // pair row of the tile, TMEM lane
    const uint32_t tl = tmem + ((uint32_t)(32 * w) << 16);
    const uint32_t idesc1 = idesc_bf16_f32(128, EF) | (1u << 16);
    const uint32_t idesc2 = idesc_bf16_f32(128, 64) | (1u << 16);

    // thread 0's count of the phases it started on each slot's load barrier and
    // of its MMA commits: on a failed wait, what it issued completes before exit
    uint32_t nfull[2] = {0u, 0u}, ncommit = 0;
    if (w == 0 && (int)blockIdx.x < ntile) {
        uint32_t cm, rm;
        tile_masks(p.M, p.n, tile_at(blockIdx.x, p.ti, p.tj), lane, cm, rm);
        if (lane == 0) {
            mbar_expect_tx(wtsb, 2 * EB_TILE);
            tma_load_2d(sbase + S::W1, &tmW1, wtsb, 0, 0);
            tma_load_2d(sbase + S::W1 + 8192, &tmW1, wtsb, 64, 0);
            tma_load_2d(sbase + S::W2, &tmW2, wtsb, 0, 0);
            issue_tile(blockIdx.x, ntile, sbase + S::SLOT, full(0), info, cm, rm, &tmIn, p, fail, nfull[0]);
        }
        __syncwarp();
    }
    uint32_t mc = 0, mr = 0;                     // warp 0: mask bytes of the tile after the next
    if (w == 0) mask_bytes(p.M, p.n, blockIdx.x + G, p.ti, p.tj, ntile, lane, mc, mr);
    uint32_t mph = 0;
    bool wts_ready = false;
    float pool[2] = {0.f, 0.f};                  // lane's channels 2 lane, 2 lane + 1 of the current graph
    int pool_b = -1;
    auto flush_pool = [&]() {
        if (pool_b >= 0) {
            atomicAdd(p.pool + (size_t)pool_b * 64 + 2 * lane, pool[0]);
            atomicAdd(p.pool + (size_t)pool_b * 64 + 2 * lane + 1, pool[1]);
        }
        pool[0] = pool[1] = 0.f;
    };
    int k = 0;
    for (int t = blockIdx.x; t < ntile; t += G, ++k) {
        const int s = k & 1, tn = t + G;
        const uint32_t slot_a = sbase + S::SLOT + s * EB_TILE, next_a = sbase + S::SLOT + (s ^ 1) * EB_TILE;
        uint8_t *slot = sp + S::SLOT + s * EB_TILE;
        uint32_t cmn = 0, rmn = 0;
        if (w == 0) {
            cmn = __ballot_sync(0xffffffffu, mc != 0);
            rmn = __ballot_sync(0xffffffffu, mr != 0) & 0xFu;
            mask_bytes(p.M, p.n, tn + G, p.ti, p.tj, ntile, lane, mc, mr);
        }
        cta_wait(full(s), (k >> 1) & 1, fail, p.status);
        const uint32_t cm = info[2 * s], rmw = info[2 * s + 1];
        const TileAt T = tile_at(t, p.ti, p.tj);
        const bool live = (rmw & 0x100u) != 0 && !*fail;
        const bool valid = ((rmw >> (r >> 5)) & 1u) && ((cm >> (r & 31)) & 1u);
        if (T.b != pool_b) {                     // warp-uniform
            flush_pool();
            pool_b = T.b;
        }
        if (!live) {
            row_zero(slot, r);
            fence_proxy_async_smem();
            named_bar_sync(1, EB_THR);
            if (r == 0) {
                if (!*fail) {
                    tma_store_4d(&tmOut, slot_a, 0, T.j0, T.i0, T.b);
                    tma_store_commit();
                }
                issue_tile(tn, ntile, next_a, full(s ^ 1), info + 2 * (s ^ 1), cmn, rmn, &tmIn, p, fail, nfull[s ^ 1]);
            }
            continue;
        }
        if (!wts_ready) {
            cta_wait(wtsb, 0, fail, p.status);
            wts_ready = true;
        }
        float x[64];
        row_load64(slot, r, x);
        {   // the warp's valid E' rows summed on the tensor cores (invalid rows zeroed first)
            if (!valid) row_zero(slot, r);
            __syncwarp();
            const float2 ps = warp_tile_colsum(slot_a, w, lane);
            pool[0] += ps.x;
            pool[1] += ps.y;
            __syncwarp();
        }
        normalise64(x);
#pragma unroll
        affine64(x, par, PAR_G1, PAR_S1);
        row_store64(slot, r, x);
        fence_proxy_async_smem();
        named_bar_sync(1, EB_THR);
        if (r == 0) {
            if (!*fail) {
                tc_fence_after();
                mma_tile(tmem, slot_a, 4, sbase + S::W1, true, 0, idesc1);
                mma_commit(mmab);
                ++ncommit;
            }
            issue_tile(tn, ntile, next_a, full(s ^ 1), info + 2 * (s ^ 1), cmn, rmn, &tmIn, p, fail, nfull[s ^ 1]);
        }
        cta_wait(mmab, mph, fail, p.status);
        mph ^= 1u;
        tc_fence_after();
        h_epilogue_tmem(tl, par + PAR_B1);
        tc_fence_before();
        named_bar_sync(1, EB_THR);
        if (r == 0 && !*fail) {
            tc_fence_after();
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk)      // h (TMEM, 8 columns a k-step) x W2 (MN-major)
                mma_bf16_ts(tmem + EF_TM_Z, tmem + kk * 8, smem_desc(sbase + S::W2 + kk * 2048, 8192, 1024, LAYOUT_SW128),
                            idesc2, kk > 0 ? 1u : 0u);
            mma_commit(mmab);
                ++ncommit;
        }
        cta_wait(mmab, mph, fail, p.status);
        mph ^= 1u;
        tc_fence_after();
        {
            float v[64];
            tmem_ld64(tl + EF_TM_Z, v);
            add_bias64(x, v, par, PAR_B2);
        }
        normalise64(x);
        affine64(x, par, PAR_G2, PAR_S2, valid);
        row_store64(slot, r, x);
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(1, EB_THR);
        if (r == 0 && !*fail) {
            tma_store_4d(&tmOut, slot_a, 0, T.j0, T.i0, T.b);
            tma_store_commit();
        }
    }
    flush_pool();
    if (r == 0) {
        if (*fail) {   // (bounded) the products and loads already issued land before the memory is released
            mma_commit(mmab);
            mbar_wait(mmab, ncommit & 1u);
            for (int s = 0; s < 2; ++s)
                if (nfull[s]) mbar_wait(full(s), (nfull[s] - 1u) & 1u);
        }
        tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, EF_TM_COLS);
}

// ------------------------------------------------------------------ backward

__global__ void __launch_bounds__(EB_THR, 2)
k_eblk_bwd(const __grid_constant__ CUtensorMap tmIn, const __grid_constant__ CUtensorMap tmDOut,
           const __grid_constant__ CUtensorMap tmDIn, const __grid_constant__ CUtensorMap tmW1,
           const __grid_constant__ CUtensorMap tmW2, EbParams p) {
    using S = EbSmem;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    volatile int *fail = reinterpret_cast<volatile int *>(sp + S::FAIL);
    const uint32_t bar0 = sbase + S::BAR;
    const uint32_t fullb = bar0, mmab = bar0 + 8, wtsb = bar0 + 16;
    uint32_t *info = reinterpret_cast<uint32_t *>(sp + S::INFO);
    float *par = reinterpret_cast<float *>(sp + S::PAR);

    if (tid == 0) {
        mbar_init(fullb, 1);
        mbar_init(mmab, 1);
        mbar_init(wtsb, 1);
        fence_mbar_init();
        *fail = 0;
    }
    if (w == 0) {
        tmem_alloc(sbase + S::TM, EB_TM_COLS);
        tmem_relinquish();
    }
    load_params(par, p, tid, EB_THR);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const int ntile = p.B * p.ti * p.tj, G = gridDim.x;
    const int r = tid;
    const uint32_t tl = tmem + ((uint32_t)(32 * w) << 16);
    const uint32_t idesc_h = idesc_bf16_f32(128, EF) | (1u << 16);    // Ea W1: B MN-major
    const uint32_t idesc_z = idesc_bf16_f32(128, 64) | (1u << 16);    // h W2: B MN-major
    const uint32_t idesc_dh = idesc_bf16_f32(128, EF);                // dEz W2^T: B K-major
    const uint32_t idesc_da = idesc_bf16_f32(128, 64);                // dh W1^T: B K-major

    // thread 0's count of the phases it started on the load barrier and of its
    // MMA commits: on a failed wait, what it issued completes before exit
    uint32_t nfull = 0, ncommit = 0;
    // thread 0: the loads of tile t (E' and dEout) and an L2 prefetch of the CTA's next tile
    auto issue = [&](int t, uint32_t cm, uint32_t rm) {
        if (t >= ntile) return;
        ++nfull;
        tma_store_wait_read0();
        const bool live = cm != 0 && rm != 0;
        info[0] = cm;
        info[1] = rm | (live ? 0x100u : 0u);
        if (live && !*fail) {
            const TileAt T = tile_at(t, p.ti, p.tj);
            mbar_expect_tx(fullb, 2 * EB_TILE);
            tma_load_4d(sbase + S::SA, &tmIn, fullb, 0, T.j0, T.i0, T.b);
            tma_load_4d(sbase + S::SB, &tmDOut, fullb, 0, T.j0, T.i0, T.b);
            if (t + G < ntile) {
                const TileAt N = tile_at(t + G, p.ti, p.tj);
                tma_prefetch_4d(&tmIn, 0, N.j0, N.i0, N.b);
                tma_prefetch_4d(&tmDOut, 0, N.j0, N.i0, N.b);
            }
        } else {
            mbar_arrive(fullb);
        }
    };
    if (w == 0 && (int)blockIdx.x < ntile) {
        uint32_t cm, rm;
        tile_masks(p.M, p.n, tile_at(blockIdx.x, p.ti, p.tj), lane, cm, rm);
        if (lane == 0) {
            mbar_expect_tx(wtsb, 2 * EB_TILE);
            tma_load_2d(sbase + S::W1, &tmW1, wtsb, 0, 0);
            tma_load_2d(sbase + S::W1 + 8192, &tmW1, wtsb, 64, 0);
            tma_load_2d(sbase + S::W2, &tmW2, wtsb, 0, 0);
            issue(blockIdx.x, cm, rm);
        }
        __syncwarp();
    }
    uint32_t mph = 0;
    bool wts_ready = false, any = false;
    // per-lane channel sums: channels 2l, 2l+1 of dg2, ds2, db2, dg1, ds1 and of both halves of db1
    float acc[14];
#pragma unroll
    for (int u = 0; u < 14; ++u) acc[u] = 0.f;
    uint8_t *sa = sp + S::SA, *sb = sp + S::SB;
    int k = 0;
    for (int t = blockIdx.x; t < ntile; t += G, ++k) {
        const int tn = t + G;
        uint32_t mc = 0, mr = 0;                 // warp 0: mask bytes of the next tile, used at the end
        if (w == 0) mask_bytes(p.M, p.n, tn, p.ti, p.tj, ntile, lane, mc, mr);
        cta_wait(fullb, k & 1, fail, p.status);
        const uint32_t cm = info[0], rmw = info[1];
        const TileAt T = tile_at(t, p.ti, p.tj);
        const bool live = (rmw & 0x100u) != 0 && !*fail;
        const bool valid = ((rmw >> (r >> 5)) & 1u) && ((cm >> (r & 31)) & 1u);
        if (live) {
            if (!wts_ready) {
                cta_wait(wtsb, 0, fail, p.status);
                wts_ready = true;
            }
            // LN1 recomputed: x1 = normalised E', Ea = x1 g1 + s1
            float z[64], d[64];
            uint32_t x1[32];                 // normalised E' (LN1's x), bf16 pairs
            row_load64(sa, r, z);
            const float r1 = normalise64(z);
#pragma unroll
            for (int c = 0; c < 32; ++c) x1[c] = pack_bf16(z[2 * c], z[2 * c + 1]);
            affine64(z, par, PAR_G1, PAR_S1);
            row_store64(sa, r, z);
            fence_proxy_async_smem();
            named_bar_sync(1, EB_THR);
            if (r == 0 && !*fail) {
                tc_fence_after();
                mma_tile(tmem, sbase + S::SA, 4, sbase + S::W1, true, 0, idesc_h);
                mma_commit(mmab);
                ++ncommit;
            }
            cta_wait(mmab, mph, fail, p.status);
            mph ^= 1u;
            tc_fence_after();
            h_epilogue(sp + S::H, r, tl, par + PAR_B1);
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, EB_THR);
            if (r == 0 && !*fail) {
                tc_fence_after();
                mma_tile(tmem, sbase + S::H, 8, sbase + S::W2, true, 0, idesc_z);
                mma_commit(mmab);
                ++ncommit;
            }
            cta_wait(mmab, mph, fail, p.status);
            mph ^= 1u;
            tc_fence_after();
            // Ez = Ea + h W2 + b2 (z holds Ea), normalised in place (x2)
            {
                float v[64];
                tmem_ld64(tl, v);
                add_bias64(z, v, par, PAR_B2);
            }
            const float r2 = normalise64(z);
            // upstream gradient, masked: dg2, ds2; LN2's input gradient dEz
            row_load64(sb, r, d);
#pragma unroll
            for (int c = 0; c < 64; ++c) d[c] = valid ? d[c] : 0.f;
            {   // dg2 = sum dEout x2, ds2 = sum dEout: rows staged in the dEout tile (read already)
                row_store_fn(sb, r, [&](int c) { return d[c] * z[c]; });
                __syncwarp();
                float2 o = warp_tile_colsum(sbase + S::SB, w, lane);
                acc[0] += o.x;
                acc[1] += o.y;
                __syncwarp();
                row_store_fn(sb, r, [&](int c) { return d[c]; });
                __syncwarp();
                o = warp_tile_colsum(sbase + S::SB, w, lane);
                acc[2] += o.x;
                acc[3] += o.y;
                __syncwarp();
            }
            float m1 = 0.f, m2 = 0.f;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float4 g = par4(par, PAR_G2 + c);
                d[c] *= g.x; d[c + 1] *= g.y; d[c + 2] *= g.z; d[c + 3] *= g.w;
            }
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                m1 += d[c];
                m2 = fmaf(d[c], z[c], m2);
            }
            m1 *= (1.f / 64.f);
            m2 *= (1.f / 64.f);
#pragma unroll
            for (int c = 0; c < 64; ++c) d[c] = r2 * (d[c] - m1 - z[c] * m2);     // dEz
            row_store64(sb, r, d);
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, EB_THR);
            if (r == 0 && !*fail) {
                tc_fence_after();
                // dh' = dEz W2^T (B = W2 read K-major: [N = 128][K = 64]); dW2 += h^T dEz
                mma_tile(tmem, sbase + S::SB, 4, sbase + S::W2, false, 0, idesc_dh);
                mma_wgrad(tmem + EB_TM_DW2, sbase + S::H, sbase + S::SB, any);
                mma_commit(mmab);
                ++ncommit;
            }
            {   // db2 = sum dEz, from the dEz tile the products read
                const float2 o = warp_tile_colsum(sbase + S::SB, w, lane);
                acc[4] += o.x;
                acc[5] += o.y;
            }
            cta_wait(mmab, mph, fail, p.status);
            mph ^= 1u;
            tc_fence_after();
            // dh = dh' [h > 0] into the H tile (h is no longer read); db1 from that tile
            {
#pragma unroll
                for (int c0 = 0; c0 < 64; c0 += 16) {
                    float va[16], vb[16];
                    tmem_ld16(tl + c0, va);
                    tmem_ld16(tl + c0 + 64, vb);
                    tmem_ld_wait();
                    const int ch = c0 >> 3;
                    relu_gate8(*reinterpret_cast<const uint4 *>(sp + S::H + sw128(r, ch)), va);
                    relu_gate8(*reinterpret_cast<const uint4 *>(sp + S::H + sw128(r, ch + 1)), va + 8);
                    relu_gate8(*reinterpret_cast<const uint4 *>(sp + S::H + EB_TILE + sw128(r, ch)), vb);
                    relu_gate8(*reinterpret_cast<const uint4 *>(sp + S::H + EB_TILE + sw128(r, ch + 1)), vb + 8);
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        const float *v = hf ? vb : va;
                        uint8_t *half = sp + S::H + hf * EB_TILE;
                        uint4 u0, u1;
                        u0.x = pack_bf16(v[0], v[1]); u0.y = pack_bf16(v[2], v[3]);
                        u0.z = pack_bf16(v[4], v[5]); u0.w = pack_bf16(v[6], v[7]);
                        u1.x = pack_bf16(v[8], v[9]); u1.y = pack_bf16(v[10], v[11]);
                        u1.z = pack_bf16(v[12], v[13]); u1.w = pack_bf16(v[14], v[15]);
                        *reinterpret_cast<uint4 *>(half + sw128(r, ch)) = u0;
                        *reinterpret_cast<uint4 *>(half + sw128(r, ch + 1)) = u1;
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(1, EB_THR);
                if (r == 0 && !*fail) {
                    tc_fence_after();
                    // dEa' = dh W1^T (B = W1 read K-major: [N = 64][K = 128], two 64-column boxes);
                    // dW1^T += dh^T Ea
                    mma_tile(tmem, sbase + S::H, 8, sbase + S::W1, false, 8192, idesc_da);
                    mma_wgrad(tmem + EB_TM_DW1, sbase + S::H, sbase + S::SA, any);
                    mma_commit(mmab);
                ++ncommit;
                }
                const float2 o0 = warp_tile_colsum(sbase + S::H, w, lane);
                const float2 o1 = warp_tile_colsum(sbase + S::H + EB_TILE, w, lane);
                acc[10] += o0.x;
                acc[11] += o0.y;
                acc[12] += o1.x;
                acc[13] += o1.y;
            }
            any = true;
            cta_wait(mmab, mph, fail, p.status);
            mph ^= 1u;
            tc_fence_after();
            // dEa = dEz + dh W1^T (d holds dEz); dg1, ds1; dE' = valid (LN1^T(dEa) + dpE_b)
            {
                float v[64];
                tmem_ld64(tl, v);
#pragma unroll
                for (int c = 0; c < 64; ++c) d[c] += v[c];
            }
            {   // dg1 = sum dEa x1, ds1 = sum dEa: rows staged in the dEz tile (its products are done)
                row_store_fn(sb, r, [&](int c) { return d[c] * pk_get(x1, c); });
                __syncwarp();
                float2 o = warp_tile_colsum(sbase + S::SB, w, lane);
                acc[6] += o.x;
                acc[7] += o.y;
                __syncwarp();
                row_store_fn(sb, r, [&](int c) { return d[c]; });
                __syncwarp();
                o = warp_tile_colsum(sbase + S::SB, w, lane);
                acc[8] += o.x;
                acc[9] += o.y;
                __syncwarp();
            }
            float n1 = 0.f, n2 = 0.f;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
                const float4 g = par4(par, PAR_G1 + c);
                d[c] *= g.x; d[c + 1] *= g.y; d[c + 2] *= g.z; d[c + 3] *= g.w;
            }
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                n1 += d[c];
                n2 = fmaf(d[c], pk_get(x1, c), n2);
            }
            n1 *= (1.f / 64.f);
            n2 *= (1.f / 64.f);
            const float4 *dp = reinterpret_cast<const float4 *>(p.dpool + (size_t)T.b * 64);
#pragma unroll
            for (int c4 = 0; c4 < 16; ++c4) {
                const float4 q = __ldg(dp + c4);
                const float qa[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int c = 4 * c4 + u;
                    d[c] = valid ? r1 * (d[c] - n1 - pk_get(x1, c) * n2) + qa[u] : 0.f;
                }
            }
            row_store64(sb, r, d);
        } else {
            row_zero(sb, r);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(1, EB_THR);
        if (w == 0) {
            const uint32_t cmn = __ballot_sync(0xffffffffu, mc != 0);
            const uint32_t rmn = __ballot_sync(0xffffffffu, mr != 0) & 0xFu;
            if (lane == 0) {
                if (!*fail) {
                    tma_store_4d(&tmDIn, sbase + S::SB, 0, T.j0, T.i0, T.b);
                    tma_store_commit();
                }
                issue(tn, cmn, rmn);
            }
            __syncwarp();
        }
    }
    // the CTA's partial sums [CTA][448] in the order dg2, ds2, db2, dg1, ds1, db1:
    // the four warps' sums added in warp order through shared memory (the H tile)
    {
        float *red = reinterpret_cast<float *>(sp + S::H);
        tc_fence_before();
        __syncthreads();
        float *pw = red + w * EB_PART;
#pragma unroll
        for (int q = 0; q < 5; ++q) {
            pw[64 * q + 2 * lane] = acc[2 * q];
            pw[64 * q + 2 * lane + 1] = acc[2 * q + 1];
        }
        pw[320 + 2 * lane] = acc[10];
        pw[320 + 2 * lane + 1] = acc[11];
        pw[384 + 2 * lane] = acc[12];
        pw[384 + 2 * lane + 1] = acc[13];
        __syncthreads();
        for (int c = tid; c < EB_PART; c += EB_THR)
            p.parts[(size_t)blockIdx.x * EB_PART + c] = red[c] + red[EB_PART + c] + red[2 * EB_PART + c] +
                                                        red[3 * EB_PART + c];
    }
    // the CTA's dW2 [128][64] and dW1^T [128][64] from TMEM (zero without a live
    // tile); every product was waited for in the loop
    tc_fence_after();
    float *pwt = p.wparts + (size_t)blockIdx.x * 2 * EF * 64;
#pragma unroll 1
    for (int m = 0; m < 2; ++m) {
        float *dst = pwt + (size_t)m * EF * 64 + (size_t)r * 64;
#pragma unroll
        for (int c0 = 0; c0 < 64; c0 += 16) {
            float v[16];
            tmem_ld16(tl + (m == 0 ? EB_TM_DW2 : EB_TM_DW1) + c0, v);
            tmem_ld_wait();
            float4 *d4 = reinterpret_cast<float4 *>(dst + c0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                d4[u] = any ? make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3])
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (r == 0) {
        if (*fail) {   // (bounded) the products and loads already issued land before the memory is released
            mma_commit(mmab);
            mbar_wait(mmab, ncommit & 1u);
            if (nfull) mbar_wait(fullb, (nfull - 1u) & 1u);
        }
        tma_store_wait_all();
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) tmem_dealloc(tmem, EB_TM_COLS);
}

// ------------------------------------------------------------------ host

static int grid_ctas(int ntile, int per_sm) {
    const int g = per_sm * sm_count();
    return ntile < g ? ntile : g;
}

cudaError_t edge_forward(const EdgeArgs &a, cudaStream_t st) {
    CUtensorMap tIn, tOut, tW1, tW2;
    if (!encode_tile_map(&tIn, a.Ein, a.B, a.n) || !encode_tile_map(&tOut, a.Eout, a.B, a.n) ||
        !encode_2d(&tW1, a.W1, 64, EF, 64) || !encode_2d(&tW2, a.W2, EF, 64, EF))
        return cudaErrorInvalidValue;
    EbParams p = a.par;
    p.ti = (a.n + 3) / 4;
    p.tj = (a.n + 31) / 32;
    const int ntile = a.B * p.ti * p.tj;
    static std::atomic<uint32_t> attr{0};
    if (cudaError_t e = ensure_smem_attr(k_eblk_fwd, EfSmem::BYTES, attr); e != cudaSuccess) return e;
    k_eblk_fwd<<<grid_ctas(ntile, 3), EB_THR, EfSmem::BYTES, st>>>(tIn, tOut, tW1, tW2, p);
    return cudaGetLastError();
}

int edge_backward_ctas(int B, int n) {
    return grid_ctas(B * ((n + 3) / 4) * ((n + 31) / 32), 2);
}

cudaError_t edge_backward(const EdgeArgs &a, cudaStream_t st) {
    CUtensorMap tIn, tDOut, tDIn, tW1, tW2;
    if (!encode_tile_map(&tIn, a.Ein, a.B, a.n) || !encode_tile_map(&tDOut, a.dEout, a.B, a.n) ||
        !encode_tile_map(&tDIn, a.dEin, a.B, a.n) || !encode_2d(&tW1, a.W1, 64, EF, 64) ||
        !encode_2d(&tW2, a.W2, EF, 64, EF))
        return cudaErrorInvalidValue;
    EbParams p = a.par;
    p.ti = (a.n + 3) / 4;
    p.tj = (a.n + 31) / 32;
    const int ntile = a.B * p.ti * p.tj;
    static std::atomic<uint32_t> attr{0};
    if (cudaError_t e = ensure_smem_attr(k_eblk_bwd, EbSmem::BYTES, attr); e != cudaSuccess) return e;
    k_eblk_bwd<<<grid_ctas(ntile, 2), EB_THR, EbSmem::BYTES, st>>>(tIn, tDOut, tDIn, tW1, tW2, p);
    return cudaGetLastError();
}

}  // namespace blk
}  // namespace fast
}  // namespace eaga
