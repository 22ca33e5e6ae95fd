// Backward pair kernels for de = 64, H = 8, dh = 32, bf16 storage (sm_100a).
//
// Chain rule of the layer (same formulas as the forward's, differentiated):
//   u_ij^h = We[h,:] . dE'_ij          dA^h_ij = dO_ih . v_jh + u_ij^h
//   D_ih   = sum_j a_ij dA_ij          dS'_ij  = a_ij (dA_ij - D_ih)
//   dgamma = dS' s,  dbeta = dS',  ds = dS' (1 + gamma)
//   dq_i = sum_j ds_ij k_j / sqrt(dh),  dk_j = sum_i ds_ij q_i / sqrt(dh),  dv_j = sum_i a_ij dO_i
//   dE = dE' + [dgamma|dbeta] Wfe^T,  dWfe = sum E^T [dgamma|dbeta],  dWe = sum a^T dE',  dg = sum [dgamma|dbeta]
// D needs a whole row of pairs before any dS' exists, so the work is split in
//   k_bwd_rows: clusters along j (like the forward): a, u, dA, cluster-wide D,
//               dS', dq (cluster-reduced), dE (tensor cores, written in place,
//               TMA store), dWfe / dWe / dg partials reduced over the cluster,
//               and a, ds of every pair stored in bf16 (32 bytes per pair);
//   k_bwd_kv:   dk, dv as sums over rows i of those a, ds times Q, dO (warp
//               MMAs fed by a TMA pipeline), so E and dE' are read only once.
// The row kernel loads both pair tiles once with TMA and keeps them in shared memory; the FiLM and
// u = dE' We^T products run on tcgen05 with the same pair <-> TMEM lane map as
// the forward.  16 warps: warp W reads TMEM quadrant W%4, heads 2(W/4)+{0,1}.
// NR selects 32NR cluster rows per CTA (NR = 1: two CTAs share an SM).
#include <math.h>
#include "fast.h"
#include "fast_common.cuh"

namespace eaga {
namespace fast {

using namespace sm100;
using namespace dev;

struct BwdRowParams {
    const __nv_bfloat16 *Q, *dO;
    const float *LSE, *g;
    const uint8_t *img, *M;
    float *D;                // [B,H,n] out
    __nv_bfloat16 *dQ;       // [B,n,256] out (scaled)
    float *rparts;           // [graph * row block][RPART] out
    __nv_bfloat16 *Pa, *Pds; // [B,H,n,npad] out: a and ds (unscaled) of every pair
    int *status;
    int n, npad;
};

struct BwdKvParams {
    __nv_bfloat16 *dK, *dV;  // [B,n,256] out (dK scaled)
    int *status;
    int n;
};

// ---------------------------------------------------------------- row kernel

template <int NR>
struct RowSmem {
    static constexpr uint32_t E = 0, DEP = NR * 32768, K = NR * 65536, V = K + NR * 16384;
    static constexpr uint32_t DF = V, AT = V + NR * 8192;          // reuse of the V chunk after dP
    static constexpr uint32_t IMG = V + NR * 16384;                // Wfe^T sw, We sw, Wfe ns (2 KB each)
    static constexpr uint32_t WD = IMG + 6144;                     // per-quadrant D partials [4][8][8]
    static constexpr uint32_t CD = WD + 1024;                      // CTA D [64] (read by peers)
    static constexpr uint32_t FD = CD + 256;                       // final D [64]
    static constexpr uint32_t WDG = FD + 256;                      // per-warp dg [16][4]
    static constexpr uint32_t G = WDG + 256;
    static constexpr uint32_t LSE = G + 64;                        // [8 i][8 h]
    static constexpr uint32_t MI = LSE + 256, MJ = MI + 16;
    static constexpr uint32_t BAR = MJ + 64;                       // 9 mbarriers
    static constexpr uint32_t TM = BAR + 72;
    static constexpr uint32_t RD = TM + 24;                        // received D partials [16][64] f32
    static constexpr uint32_t BYTES = RD + 4096 + 1024;
    // in the E tile once it is dead: the CTA weight-grad partial, the pushed
    // weight-grad slices and the pushed dq slices of the cluster
    static constexpr uint32_t WP = E, RWP = E + 6400, RQ = E + 13056;
    static constexpr uint32_t QPART = K;                           // 16 KB two-slot dq sums (K, V dead)
};

template <int NR>
__global__ void __launch_bounds__(NTHR, NR == 1 ? 2 : 1)
k_bwd_rows(const __grid_constant__ CUtensorMap tmE, const __grid_constant__ CUtensorMap tmDEp,
           const __grid_constant__ CUtensorMap tmDE, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, BwdRowParams p) {
    using S = RowSmem<NR>;
    constexpr int TCN = tile_cols(NR), NE = 2 * NR;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    uint8_t *sp = smem_raw + (sbase - smem_u32(smem_raw));
    const int tid = threadIdx.x, W = tid >> 5, q = W & 3, hq = W >> 2, t = tid & 31, c4 = t & 3, g8 = t >> 2;
    const uint32_t rank = cluster_rank(), nclu = gridDim.x;
    const int n = p.n;
    const int j0 = blockIdx.x * TCN, i0 = blockIdx.y * TB, b = blockIdx.z;
    const uint32_t bar_e = sbase + S::BAR, bar_dep = bar_e + 8, bar_kv = bar_e + 16, bar_film = bar_e + 24,
                   bar_u = bar_e + 32, bar_de = bar_e + 40, bar_d = bar_e + 48, bar_wp = bar_e + 56,
                   bar_q = bar_e + 64;
    float *g = reinterpret_cast<float *>(sp + S::G);
    float *lse = reinterpret_cast<float *>(sp + S::LSE);
    uint8_t *mi = sp + S::MI, *mj = sp + S::MJ;
    constexpr uint32_t TM_FILM = 0, TM_U = 64, TM_DE = 128, TM_COLS = 256;

    if (tid == 0) {
        mbar_init(bar_e, 1); mbar_init(bar_dep, 1); mbar_init(bar_kv, 1);
        mbar_init(bar_film, 1); mbar_init(bar_u, 1); mbar_init(bar_de, 1);
        mbar_init(bar_d, 1); mbar_init(bar_wp, 1); mbar_init(bar_q, 1);
        fence_mbar_init();
        mbar_expect_tx(bar_d, nclu * 64 * 4);
        mbar_expect_tx(bar_wp, nclu * flat_slice(RPART, nclu, rank) * 16);
        mbar_expect_tx(bar_q, nclu * rows_slice(1, nclu, rank) * 16);
        mbar_expect_tx(bar_e, NR * 32768);
        tma_load_5d(sbase + S::E, &tmE, bar_e, 0, i0 / 2, j0, 0, b);
        mbar_expect_tx(bar_dep, NR * 32768);
        tma_load_5d(sbase + S::DEP, &tmDEp, bar_dep, 0, i0 / 2, j0, 0, b);
        mbar_expect_tx(bar_kv, NR * 32768);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            tma_load_3d(sbase + S::K + k * NR * 4096, &tmK, bar_kv, 64 * k, j0, b);
            tma_load_3d(sbase + S::V + k * NR * 4096, &tmV, bar_kv, 64 * k, j0, b);
        }
    }
    if (W == 0) {
        tmem_alloc(sbase + S::TM, TM_COLS);
        tmem_relinquish();
    }
    if (tid < 384) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.img);
        const uint32_t img_off = (tid >> 7) == 0 ? IMG_WFE_T_SW : (tid >> 7) == 1 ? IMG_WE_SW : IMG_WFE_NS;
        reinterpret_cast<uint4 *>(sp + S::IMG)[tid] = src[(img_off >> 4) + (tid & 127)];
    }
    if (tid < NF) g[tid] = p.g[(size_t)b * NF + tid];
    if (tid >= 32 && tid < 32 + TB) mi[tid - 32] = (i0 + tid - 32 < n) ? p.M[(size_t)b * n + i0 + tid - 32] : 0;
    if (tid >= 64 && tid < 64 + TCN) mj[tid - 64] = (j0 + tid - 64 < n) ? p.M[(size_t)b * n + j0 + tid - 64] : 0;
    if (tid >= 128 && tid < 192) {
        const int x = tid - 128, il = x >> 3, h = x & 7;
        lse[x] = (i0 + il < n) ? p.LSE[((size_t)b * NH + h) * n + i0 + il] : 0.f;
    }
    uint32_t qf[2][2][2], of[2][2][2];
    load_frags2(p.Q, b, n, i0, hq, g8, c4, qf);
    load_frags2(p.dO, b, n, i0, hq, g8, c4, of);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sp + S::TM);
    const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
    cluster_arrive();   // receive barriers of this CTA are armed

    if (tid == 0) {
        if (!mbar_wait(bar_e, 0)) flag_timeout(p.status);
        tc_fence_after();
        issue_pair_products<NR>(sbase + S::E, sbase + S::IMG, tmem + TM_FILM);
        mma_commit(bar_film);
        if (!mbar_wait(bar_dep, 0)) flag_timeout(p.status);
        tc_fence_after();
        issue_pair_products<NR>(sbase + S::DEP, sbase + S::IMG + 2048, tmem + TM_U);
        mma_commit(bar_u);
    }
    __syncwarp();
    if (!mbar_wait(bar_kv, 0)) flag_timeout(p.status);
    float sv[2][4], da[2][4], av[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    warp_scores2<NR>(sbase + S::K, q, t, hq, qf, sv);
    warp_scores2<NR>(sbase + S::V, q, t, hq, of, da);

    if (!mbar_wait(bar_film, 0)) flag_timeout(p.status);
    if (!mbar_wait(bar_u, 0)) flag_timeout(p.status);
    tc_fence_after();
    const float rs = rsqrtf((float)DH);
    float gm[2][4];
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        const int jl = 32 * (e >> 1) + 8 * q + g8, il = 2 * c4 + (e & 1);
        const bool valid = mi[il] && mj[jl];
        float f0, f1, b0, b1, u0, u1;
        tmem_ld2(tl + TM_FILM + 16 * e + 2 * hq, f0, f1);
        tmem_ld2(tl + TM_FILM + 16 * e + NH + 2 * hq, b0, b1);
        tmem_ld2(tl + TM_U + 16 * e + 2 * hq, u0, u1);
        tmem_ld_wait();
        const float fg[2] = {f0, f1}, fb[2] = {b0, b1}, fu[2] = {u0, u1};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int h = 2 * hq + hh;
            const float s = sv[hh][e] * rs;
            const float gam = fg[hh] + g[h], bet = fb[hh] + g[NH + h];
            av[hh][e] = valid ? exp2f((s * (1.f + gam) + bet - lse[il * 8 + h]) * LOG2E) : 0.f;
            sv[hh][e] = s;
            gm[hh][e] = gam;
            da[hh][e] += fu[hh];
        }
    }
    // D_ih = sum_j a dA: warp, CTA, cluster
    float *wd = reinterpret_cast<float *>(sp + S::WD);
    float *cd = reinterpret_cast<float *>(sp + S::CD);
    float *fd = reinterpret_cast<float *>(sp + S::FD);
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            float x = av[hh][s] * da[hh][s];
            if (NR == 2) x += av[hh][2 + s] * da[hh][2 + s];
            x += __shfl_xor_sync(0xffffffffu, x, 4);
            x += __shfl_xor_sync(0xffffffffu, x, 8);
            x += __shfl_xor_sync(0xffffffffu, x, 16);
            if (g8 == 0) wd[(q * 8 + 2 * c4 + s) * 8 + 2 * hq + hh] = x;
        }
    __syncthreads();
    if (tid < 64) cd[tid] = wd[tid] + wd[64 + tid] + wd[128 + tid] + wd[192 + tid];
    __syncthreads();
    cluster_wait();     // every peer's receive barriers are armed
    push_rowvals_f32(sp, sbase, S::CD, S::RD, bar_d, tid, rank, nclu);
    if (!mbar_wait(bar_d, 0)) flag_timeout(p.status);
    combine_rowvals_f32(sp, S::RD, S::FD, tid, nclu);
    __syncthreads();
    if (tid < 64) {
        const int il = tid >> 3, h = tid & 7;
        if (rank == 0 && i0 + il < n) p.D[((size_t)b * NH + h) * n + i0 + il] = fd[tid];
    }

    // dS', df = [dgamma | dbeta], ds = dS'(1+gamma); df and a tiles for the tensor cores
    float dgp[4] = {0.f, 0.f, 0.f, 0.f};   // dgamma h0, h1, dbeta h0, h1
    const uint32_t L = 32 * q + t;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        if (e >= NE) {
            da[0][e] = da[1][e] = 0.f;
            continue;
        }
        const int il = 2 * c4 + (e & 1);
        float dgam[2], dbet[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const float dsp = av[hh][e] * (da[hh][e] - fd[il * 8 + 2 * hq + hh]);
            dgam[hh] = dsp * sv[hh][e];
            dbet[hh] = dsp;
            da[hh][e] = dsp * (1.f + gm[hh][e]);     // ds (unscaled)
            dgp[hh] += dgam[hh];
            dgp[2 + hh] += dbet[hh];
        }
        *reinterpret_cast<uint32_t *>(sp + S::DF + e * 4096 + ns16(L, 2 * hq)) = pack_bf16(dgam[0], dgam[1]);
        *reinterpret_cast<uint32_t *>(sp + S::DF + e * 4096 + ns16(L, NH + 2 * hq)) = pack_bf16(dbet[0], dbet[1]);
        *reinterpret_cast<uint32_t *>(sp + S::AT + e * 4096 + ns16(L, 2 * hq)) = pack_bf16(av[0][e], av[1][e]);
        if (hq == 0) *reinterpret_cast<uint4 *>(sp + S::AT + e * 4096 + ns16(L, 8)) = make_uint4(0, 0, 0, 0);
    }
    // a and ds of the tile's pairs for the dk / dv pass: [b][h][i][j] bf16.
    // Lanes t and t^4 hold neighbouring columns j; they swap one head so that
    // each stores two columns of one head in a 4-byte word.
    {
        const bool odd = g8 & 1;
#pragma unroll
        for (int e = 0; e < NE; ++e) {
            const float xa = __shfl_xor_sync(0xffffffffu, odd ? av[0][e] : av[1][e], 4);
            const float xd = __shfl_xor_sync(0xffffffffu, odd ? da[0][e] : da[1][e], 4);
            const int i = i0 + 2 * c4 + (e & 1), j = j0 + 32 * (e >> 1) + 8 * q + (g8 & ~1);
            if (i < n && j < n) {
                const size_t o = (((size_t)b * NH + 2 * hq + (odd ? 1 : 0)) * n + i) * p.npad + j;
                *reinterpret_cast<uint32_t *>(p.Pa + o) = odd ? pack_bf16(xa, av[1][e]) : pack_bf16(av[0][e], xa);
                *reinterpret_cast<uint32_t *>(p.Pds + o) = odd ? pack_bf16(xd, da[1][e]) : pack_bf16(da[0][e], xd);
            }
        }
    }
    float *wdg = reinterpret_cast<float *>(sp + S::WDG);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float x = dgp[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (t == 0) wdg[W * 4 + k] = x;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    const uint32_t idesc_de = idesc_bf16_f32(128, DE);
    if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ee = 0; ee < 2; ++ee)
            mma_bf16_ss(tmem + TM_DE + 64 * ee, smem_desc(sbase + S::DF + ee * 4096, 128, 256, LAYOUT_NONE),
                        smem_desc(sbase + S::IMG + 4096, 128, 256, LAYOUT_NONE), idesc_de, 0);
        mma_commit(bar_de);
    }
    __syncwarp();

    // dq partial = K^T ds^T (warp MMAs)
    float qacc[2][2][4];
    warp_contract2<NR>(sbase + S::K, q, t, hq, da, qacc);

    // dWfe [64 c][16 k] and dWe^T [64 c][8 h] partials: warp W owns c in
    // [16ct, 16ct+16) (ct = W%4) over k-range kr = W/4 of the CTA's pairs; the
    // four k-ranges are added in a fixed order.
    {
        const int ct = W & 3, kr = W >> 2;
        float wf[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        float we4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 2
        for (int kk = 4 * NR * kr; kk < 4 * NR * (kr + 1); ++kk) {
            const int e = kk >> 3, L0 = 16 * (kk & 7);
            const uint32_t row0 = tile_off<NR>(e) / 128 + L0;
            const uint32_t arow = row0 + (t & 7) + ((t >> 4) & 1) * 8;
            const uint32_t ach = 2 * ct + ((t >> 3) & 1);
            uint32_t aE[4], aD[4], bF[4], bA0, bA1;
            ldsm_x4_t(sbase + S::E + sw128(arow, ach), aE);
            ldsm_x4_t(sbase + S::DEP + sw128(arow, ach), aD);
            const uint32_t Lr = L0 + (t & 7) + ((t >> 3) & 1) * 8;
            ldsm_x4_t(sbase + S::DF + e * 4096 + ns16(Lr, 8 * (t >> 4)), bF);
            ldsm_x2_t(sbase + S::AT + e * 4096 + ns16(Lr, 0), bA0, bA1);
            mma16816(wf[0], aE, bF[0], bF[1]);
            mma16816(wf[1], aE, bF[2], bF[3]);
            mma16816(we4, aD, bA0, bA1);
        }
        __syncthreads();   // the E tile is dead from here on
        cluster_arrive();  // peers may now push into this CTA's E tile space
        float *rp = reinterpret_cast<float *>(sp + S::WP);
        for (int phase = 0; phase < 4; ++phase) {
            if (kr == phase) {
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int c = 16 * ct + g8 + 8 * (e >> 1), k = nt * 8 + 2 * c4 + (e & 1);
                        rp[c * NF + k] = (phase ? rp[c * NF + k] : 0.f) + wf[nt][e];
                    }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 16 * ct + g8 + 8 * (e >> 1), h = 2 * c4 + (e & 1);
                    float *dst = rp + DE * NF + h * DE + c;
                    *dst = (phase ? *dst : 0.f) + we4[e];
                }
            }
            __syncthreads();
        }
        if (tid < NF) {
            const int which = tid >> 3, h = tid & 7, hq2 = h >> 1, hh = h & 1;
            float x = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) x += wdg[(4 * hq2 + k) * 4 + which * 2 + hh];
            rp[DE * NF + NH * DE + tid] = x;
        }
    }
    // sum the CTA partials over the cluster: one partial per (graph, row block)
    __syncthreads();
    cluster_wait();
    push_flat(sp, sbase, S::WP, RPART, S::RWP, bar_wp, tid, rank, nclu);

    // dE = dE' + df Wfe^T, written in place over the dE' tile, NR rounds of two MMAs
    for (int round = 0; round < NR; ++round) {
        if (!mbar_wait(bar_de, round)) flag_timeout(p.status);
        tc_fence_after();
#pragma unroll
        for (int ee = 0; ee < 2; ++ee) {
            const int e = 2 * round + ee;
            float dv[16];
            tmem_ld16(tl + TM_DE + 64 * ee + 16 * hq, dv);
            tmem_ld_wait();
            add_residual16(sp + S::DEP + tile_off<NR>(e) + L * 128, L, hq, dv);
        }
        if (round + 1 < NR) {
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ee = 0; ee < 2; ++ee)
                    mma_bf16_ss(tmem + TM_DE + 64 * ee,
                                smem_desc(sbase + S::DF + (2 * (round + 1) + ee) * 4096, 128, 256, LAYOUT_NONE),
                                smem_desc(sbase + S::IMG + 4096, 128, 256, LAYOUT_NONE), idesc_de, 0);
                mma_commit(bar_de);
            }
            __syncwarp();
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tma_store_5d(&tmDE, sbase + S::DEP, 0, i0 / 2, j0, 0, b);
        tma_store_commit();
    }
    // weight-grad partial of the cluster: this CTA's slice of the sum over peers
    if (!mbar_wait(bar_wp, 0)) flag_timeout(p.status);
    {
        float *rp = p.rparts + (size_t)(blockIdx.z * gridDim.y + blockIdx.y) * RPART;
        const uint32_t per4 = (RPART / 4 + nclu - 1) / nclu, slice = flat_slice(RPART, nclu, rank);
        const float4 *rv = reinterpret_cast<const float4 *>(sp + S::RWP);
        for (uint32_t k0 = tid; k0 < slice; k0 += NTHR) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            for (uint32_t pp = 0; pp < nclu; ++pp) {
                const float4 v = rv[pp * per4 + k0];
                a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
            }
            reinterpret_cast<float4 *>(rp)[rank * per4 + k0] = a;
        }
    }
    // dq: reduce over the quadrant warps and the cluster
    store_quadrant_part_2ph(sp, S::QPART, qacc, q, hq, t);
    {
        const uint32_t parts[1] = {S::QPART};
        push_rows_partials<1, 2>(sp, sbase, parts, S::RQ, bar_q, tid, rank, nclu);
        if (!mbar_wait(bar_q, 0)) flag_timeout(p.status);
        __nv_bfloat16 *const outs[1] = {p.dQ};
        const float sc[1] = {rs};
        finish_rows_partials<1>(sp, S::RQ, tid, rank, nclu, outs, b, n, i0, sc);
    }
    if (tid == 0) tma_store_wait_read0();
    tc_fence_before();
    __syncthreads();
    if (W == 0) tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------- dk, dv pass
// dk_j = sum_i ds_ij q_i / sqrt(dh) and dv_j = sum_i a_ij dO_i from the a and
// ds the row kernel stored.  CTA = (32 columns j, graph), warp = head; each
// pipeline stage brings 16 rows i of a, ds (all heads), Q and dO with TMA and
// every warp adds their products on warp MMAs (M = j, N = d, K = i).
constexpr int KV_J = 32, KV_I = 16, KV_STAGES = 3, KV_THR = 256;
struct KvSmem {
    static constexpr uint32_t PDS = 0, PA = 8192, QT = 16384, DOT = 24576, STAGE = 32768;
    static constexpr uint32_t BAR = KV_STAGES * STAGE;            // full[S], empty[S]
    static constexpr uint32_t BYTES = BAR + 2 * KV_STAGES * 8 + 1024;
};

__global__ void __launch_bounds__(KV_THR, 2)
k_bwd_kv(const __grid_constant__ CUtensorMap tmPds, const __grid_constant__ CUtensorMap tmPa,
         const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO, BwdKvParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
    const int tid = threadIdx.x, h = tid >> 5, t = tid & 31, g8 = t >> 2, c4 = t & 3;
    const int n = p.n, j0 = blockIdx.x * KV_J, b = blockIdx.y;
    const int nsteps = (n + KV_I - 1) / KV_I;
    const uint32_t bar0 = sbase + KvSmem::BAR;
    auto full = [&](int s) { return bar0 + 8 * s; };
    auto empty = [&](int s) { return bar0 + 8 * (KV_STAGES + s); };
    auto issue = [&](int k) {
        const int s = k % KV_STAGES, i0 = k * KV_I;
        const uint32_t st = sbase + s * KvSmem::STAGE;
        mbar_expect_tx(full(s), KvSmem::STAGE);
        tma_load_4d(st + KvSmem::PDS, &tmPds, full(s), j0, i0, 0, b);
        tma_load_4d(st + KvSmem::PA, &tmPa, full(s), j0, i0, 0, b);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            tma_load_3d(st + KvSmem::QT + c * 2048, &tmQ, full(s), 64 * c, i0, b);
            tma_load_3d(st + KvSmem::DOT + c * 2048, &tmDO, full(s), 64 * c, i0, b);
        }
    };
    if (tid == 0) {
        for (int s = 0; s < KV_STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), KV_THR / 32);
        }
        fence_mbar_init();
        for (int k = 0; k < KV_STAGES && k < nsteps; ++k) issue(k);
    }
    __syncthreads();

    float kacc[2][4][4], vacc[2][4][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int x = 0; x < 4; ++x) kacc[mt][nt][x] = vacc[mt][nt][x] = 0.f;
    // ldmatrix lanes: A = P^T (stored [i][j]) and B = Q, dO (stored [i][d]), both transposed loads
    const int arow = (t & 7) + ((t >> 4) & 1) * 8, ach = (t >> 3) & 1;
    const int brow = (t & 7) + ((t >> 3) & 1) * 8, bch = t >> 4;
    for (int k = 0; k < nsteps; ++k) {
        const int s = k % KV_STAGES;
        const uint32_t ph = (k / KV_STAGES) & 1;
        if (!mbar_wait(full(s), ph)) flag_timeout(p.status);
        const uint32_t st = sbase + s * KvSmem::STAGE;
        uint32_t bq[2][4], bo[2][4];
#pragma unroll
        for (int np = 0; np < 2; ++np) {
            const uint32_t off = (h >> 1) * 2048 + sw128(brow, (h & 1) * 4 + 2 * np + bch);
            ldsm_x4_t(st + KvSmem::QT + off, bq[np]);
            ldsm_x4_t(st + KvSmem::DOT + off, bo[np]);
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const uint32_t off = h * 1024 + sw64(arow, 2 * mt + ach);
            uint32_t ad[4], aa[4];
            ldsm_x4_t(st + KvSmem::PDS + off, ad);
            ldsm_x4_t(st + KvSmem::PA + off, aa);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                mma16816(kacc[mt][nt], ad, bq[nt >> 1][2 * (nt & 1)], bq[nt >> 1][2 * (nt & 1) + 1]);
                mma16816(vacc[mt][nt], aa, bo[nt >> 1][2 * (nt & 1)], bo[nt >> 1][2 * (nt & 1) + 1]);
            }
        }
        __syncwarp();
        if (t == 0) mbar_arrive(empty(s));
        if (tid == 0 && k + KV_STAGES < nsteps) {
            if (!mbar_wait(empty(s), ph)) flag_timeout(p.status);
            issue(k + KV_STAGES);
        }
        __syncwarp();
    }
    const float rs = rsqrtf((float)DH);
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int j = j0 + 16 * mt + 8 * hf + g8;
            if (j >= n) continue;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const size_t o = ((size_t)b * n + j) * HD + h * DH + nt * 8 + 2 * c4;
                *reinterpret_cast<uint32_t *>(p.dK + o) =
                    pack_bf16(kacc[mt][nt][2 * hf] * rs, kacc[mt][nt][2 * hf + 1] * rs);
                *reinterpret_cast<uint32_t *>(p.dV + o) = pack_bf16(vacc[mt][nt][2 * hf], vacc[mt][nt][2 * hf + 1]);
            }
        }
}

// ---------------------------------------------------------------- reductions
// All sums run in a fixed order (deterministic): first over segments of rows
// (or CTAs) in parallel blocks, then over the segments.

// Column sums of segment z of the rows: out[z][col].  Sources by column:
// [0,256) dQ, [256,512) dK, [512,768) dV, [768,768+dx) M-masked dX'.  Block
// (256-column strip, row segment): lane = 8 columns (one 16-byte load per
// row), warp = every 8th row of the segment, warps added in a fixed order.
__global__ void __launch_bounds__(256) k_bias_partial(const __nv_bfloat16 *dQ, const __nv_bfloat16 *dK,
                                                      const __nv_bfloat16 *dV, const __nv_bfloat16 *dXo,
                                                      const uint8_t *M, int rows, int dx, int seg_rows, float *out) {
    __shared__ float red[8][256];
    const int w = threadIdx.x >> 5, t = threadIdx.x & 31;
    const int strip = blockIdx.x, ncol = 3 * HD + dx;
    const bool masked = strip >= 3;
    const __nv_bfloat16 *src = strip == 0 ? dQ : strip == 1 ? dK : strip == 2 ? dV : dXo;
    const int ld = masked ? dx : HD, c0 = (masked ? (strip - 3) * 256 : 0) + 8 * t;
    const bool active = c0 < ld;
    const int r0 = blockIdx.y * seg_rows, r1 = min(rows, r0 + seg_rows);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
#pragma unroll 4
        for (int r = r0 + w; r < r1; r += 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(src + (size_t)r * ld + c0);
            const bool keep = !masked || M[r];
            const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 f = __bfloat1622float2(v2[u]);
                acc[2 * u] += keep ? f.x : 0.f;
                acc[2 * u + 1] += keep ? f.y : 0.f;
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) red[w][8 * t + u] = acc[u];
    __syncthreads();
    const int col = threadIdx.x, gcol = strip * 256 + col;
    if (gcol < ncol && (!masked || (strip - 3) * 256 + col < dx)) {
        float x = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) x += red[k][col];
        out[(size_t)blockIdx.y * ncol + gcol] = x;
    }
}

// Row-kernel partials: out[z][e] = sum over CTAs of segment z of rparts[cta][e], e < dWfe+dWe.
__global__ void k_rparts_partial(const float *rparts, int ctas, int seg, float *out) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    constexpr int NE = DE * NF + NH * DE;
    if (e >= NE) return;
    const int c0 = blockIdx.y * seg, c1 = min(ctas, c0 + seg);
    float acc = 0.f;
    for (int c = c0; c < c1; ++c) acc += rparts[(size_t)c * RPART + e];
    out[(size_t)blockIdx.y * NE + e] = acc;
}

struct DWPtrs {
    float *p[12];
};

// Final sums: weight gradients of the four node projections (split-K
// partials), bias gradients, dWfe / dWe, and the global FiLM term's dg_b,
// dWfy, dbf, dy.
__global__ void k_bwd_finish(const float *wparts, int wsplits, const float *bparts, int bsplits,
                             const float *r2, int rsplits, const float *rparts, int ctas_per_graph, int B, int dx,
                             int dy, const __nv_bfloat16 *y, const __nv_bfloat16 *Wfy, DWPtrs dW,
                             __nv_bfloat16 *dyo, float *dg) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const int msz = dx * HD;
    const int ncol = 3 * HD + dx;
    constexpr int NE = DE * NF + NH * DE;
    if (e < 4 * msz) {
        const int q = e / msz, o = e % msz;
        const float *src = wparts + (size_t)q * wsplits * msz + o;
        float acc = 0.f;
        for (int z = 0; z < wsplits; ++z) acc += src[(size_t)z * msz];
        dW.p[q == 0 ? 0 : q == 1 ? 2 : q == 2 ? 4 : 10][o] = acc;
        return;
    }
    int x = e - 4 * msz;
    if (x < ncol) {
        float acc = 0.f;
        for (int z = 0; z < bsplits; ++z) acc += bparts[(size_t)z * ncol + x];
        if (x < 3 * HD) dW.p[1 + 2 * (x / HD)][x % HD] = acc;
        else dW.p[11][x - 3 * HD] = acc;
        return;
    }
    x -= ncol;
    if (x < NE) {
        float acc = 0.f;
        for (int z = 0; z < rsplits; ++z) acc += r2[(size_t)z * NE + x];
        if (x < DE * NF) dW.p[6][x] = acc; else dW.p[9][x - DE * NF] = acc;
        return;
    }
    x -= NE;
    if (x < B * NF) {
        const int b = x / NF, k = x % NF;
        float acc = 0.f;
        for (int c = 0; c < ctas_per_graph; ++c) acc += rparts[((size_t)b * ctas_per_graph + c) * RPART + NE + k];
        dg[x] = acc;
    }
}

// dbf, dWfy, dy from dg (after k_bwd_finish).
__global__ void k_film_grads(const float *dg, int B, int dy, const __nv_bfloat16 *y, const __nv_bfloat16 *Wfy,
                             float *dbf, float *dWfy, __nv_bfloat16 *dyo) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < NF) {
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc += dg[b * NF + e];
        dbf[e] = acc;
    } else if (e < NF + dy * NF) {
        const int x = e - NF, c = x / NF, k = x % NF;
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc = fmaf(__bfloat162float(y[(size_t)b * dy + c]), dg[b * NF + k], acc);
        dWfy[x] = acc;
    } else if (e < NF + dy * NF + B * dy) {
        const int x = e - NF - dy * NF, b = x / dy, c = x % dy;
        float acc = 0.f;
        for (int k = 0; k < NF; ++k) acc = fmaf(dg[b * NF + k], __bfloat162float(Wfy[c * NF + k]), acc);
        dyo[x] = __float2bfloat16_rn(acc);
    }
}

// ---------------------------------------------------------------- host side

cudaError_t launch_bwd_stream(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                              cudaStream_t st);

template <int NR>
static cudaError_t launch_bwd_nr(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                                 cudaStream_t st) {
    constexpr int TCN = tile_cols(NR);
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e;
        if ((e = cudaFuncSetAttribute(k_bwd_rows<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      RowSmem<NR>::BYTES)) != cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(k_bwd_rows<NR>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1)) !=
            cudaSuccess)
            return e;
        if ((e = cudaFuncSetAttribute(k_bwd_kv, cudaFuncAttributeMaxDynamicSharedMemorySize, KvSmem::BYTES)) !=
            cudaSuccess)
            return e;
        attr_done = true;
    }
    __nv_bfloat16 *dO = reinterpret_cast<__nv_bfloat16 *>(ws + W.dO);
    __nv_bfloat16 *dQ = reinterpret_cast<__nv_bfloat16 *>(ws + W.dQ);
    __nv_bfloat16 *dK = reinterpret_cast<__nv_bfloat16 *>(ws + W.dK);
    __nv_bfloat16 *dV = reinterpret_cast<__nv_bfloat16 *>(ws + W.dV);
    float *D = reinterpret_cast<float *>(ws + W.D);
    const int nc = (d.n + TCN - 1) / TCN;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = nc;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(NTHR);
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    prof_mark(2, 0, st);
    {
        cudaError_t e = launch_bwd_stream(d, a, W, ws, g, st);
        if (e != cudaSuccess) return e;
    }
    prof_mark(2, 1, st);
    {
        CUtensorMap mPds, mPa, mQ, mDO;
        if (!encode_p_map(&mPds, ws + W.Pds, d.B, d.n, W.npad) || !encode_p_map(&mPa, ws + W.Pa, d.B, d.n, W.npad) ||
            !encode_node_map(&mQ, a.Q, d.B, d.n, KV_I) || !encode_node_map(&mDO, dO, d.B, d.n, KV_I))
            return cudaErrorInvalidValue;
        BwdKvParams p;
        p.dK = dK;
        p.dV = dV;
        p.status = a.status;
        p.n = d.n;
        k_bwd_kv<<<dim3((d.n + KV_J - 1) / KV_J, d.B), KV_THR, KvSmem::BYTES, st>>>(mPds, mPa, mQ, mDO, p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

cudaError_t launch_bwd_pairs(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, const float *g,
                             cudaStream_t st) {
    return pick_nr(d.n) == 1 ? launch_bwd_nr<1>(d, a, W, ws, g, st) : launch_bwd_nr<2>(d, a, W, ws, g, st);
}

cudaError_t launch_bwd_finish(const eaga_dims &d, const BwdArgs &a, const FastWs &W, char *ws, float *dg,
                              cudaStream_t st) {
    const __nv_bfloat16 *dQ = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dQ);
    const __nv_bfloat16 *dK = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dK);
    const __nv_bfloat16 *dV = reinterpret_cast<const __nv_bfloat16 *>(ws + W.dV);
    const int rows = d.B * d.n, ncol = 3 * HD + d.dx;
    float *bparts = reinterpret_cast<float *>(ws + W.bparts);
    const int seg_rows = (rows + W.bsplits - 1) / W.bsplits;
    k_bias_partial<<<dim3(3 + (d.dx + 255) / 256, W.bsplits), 256, 0, st>>>(
        dQ, dK, dV, static_cast<const __nv_bfloat16 *>(a.dXout), a.M, rows, d.dx, seg_rows, bparts);
    float *r2 = reinterpret_cast<float *>(ws + W.r2);
    const int ctas = W.n_rparts, seg = (ctas + W.rsplits - 1) / W.rsplits;
    constexpr int NE = DE * NF + NH * DE;
    const float *rparts = reinterpret_cast<const float *>(ws + W.rparts);
    k_rparts_partial<<<dim3((NE + 255) / 256, W.rsplits), 256, 0, st>>>(rparts, ctas, seg, r2);
    DWPtrs dWdev;
    for (int q = 0; q < 12; ++q) dWdev.p[q] = a.dW[q];
    const int total = 4 * d.dx * HD + ncol + NE + d.B * NF;
    const int cpg = (d.n + TB - 1) / TB;
    k_bwd_finish<<<(total + 255) / 256, 256, 0, st>>>(reinterpret_cast<const float *>(ws + W.wparts), W.wsplits,
                                                      bparts, W.bsplits, r2, W.rsplits, rparts, cpg, d.B, d.dx,
                                                      d.dy, static_cast<const __nv_bfloat16 *>(a.y),
                                                      static_cast<const __nv_bfloat16 *>(a.w[7]), dWdev,
                                                      static_cast<__nv_bfloat16 *>(a.dy), dg);
    const int tf = NF + d.dy * NF + d.B * d.dy;
    k_film_grads<<<(tf + 255) / 256, 256, 0, st>>>(dg, d.B, d.dy, static_cast<const __nv_bfloat16 *>(a.y),
                                                   static_cast<const __nv_bfloat16 *>(a.w[7]), a.dW[8], a.dW[7],
                                                   static_cast<__nv_bfloat16 *>(a.dy));
    return cudaGetLastError();
}

}  // namespace fast
}  // namespace eaga
