// fa_bwd64.cuh -- main backward kernel of exact tiled attention at head dimension 64 on
// sm_100a (the preprocess and dQ conversion kernels are those of fa_bwd.cuh).
//
// The method is the one of fa_bwd.cuh (anthology note "NOTE-005: FlashAttention", sections
// "Method" and "Key components"): each probability block is recomputed on chip from Q, K
// and the stored LSE instead of being read from a saved N x N matrix, and the textbook
// chain rule gives dV = P^T dO, dP = dO V^T, dS = P o (dP - D), dK = scale dS^T Q and
// dQ = scale dS K.
//
// What shapes this kernel: one thread issues tcgen05.mma at most about once every 120
// cycles, whatever the product's N up to 128 (measured), while an iteration here (a
// 128-key tile against a 128-query tile) has 32 MMAs: S^T and dP^T (N = 128, four steps
// each) and dV, dK, dQ (N = 64, eight steps each).  From one thread that is ~3900 cycles of
// issue for ~1300 cycles of tensor work.  So the products are issued by four threads in
// four warps, each with its own chain and barriers, and the tensor core interleaves them:
//   warp 9      S^T_i = K Q_i^T and dP^T_i = V dO_i^T
//   warp 10     dV += P^T_i dO_i      (P^T from TMEM)
//   warp 11     dK += dS^T_i Q_i      (dS^T from shared memory)
//   warp 12     dQ_i = dS_i K         (dS from shared memory; lane 0, before its share of
//               the dQ drain below)
// and the other roles are those of fa_bwd_kernel:
//   warps 0..7  P and dS: one key row per thread (TMEM lane), query half w / 4
//   warp 8      TMA producer: K, V once per item; Q_i, dO_i (+ LSE_i, D_i) into a 2-stage ring
//   warps 12..15 dQ drain: TMEM -> swizzled shared-memory staging -> TMA reduce-add into
//               the fp32 accumulator
// TMEM: S^T [0,128), dP^T [128,256), dV [256,320), dK [320,384), dQ [384,448), P^T
// [448,512).  dS is written once, to shared memory (two buffers), in the 128-byte-swizzled
// layout [query half][key row][64 queries]: read one way it is the K-major A operand dS^T of
// dK, read the other way the MN-major A operand dS of dQ.  No product then waits for
// another to free TMEM columns: S^T_{i+1} and dP^T_{i+1} follow the loads of S^T_i and
// dP^T_i, P_{i+1} waits only for dV_i, dS_{i+1} only for the products of dS_{i-1}.
//
// Item boundaries (a CTA walks about five key tiles at GPT-2 size, so they matter): K has
// two buffers, so the next tile's K is loaded while the last dQ of this one still reads K;
// V is reloaded as soon as the last dP^T has read it.  The next item's first S^T is then
// ready when the P/dS warps get to it.  Those warps write the finished dK, dV of an item
// only after they have formed the next item's first P block (the deferred epilogue), so the
// last dK / dV products run while they work, and they store dK, dV straight from registers
// (no staging, no barrier across warps).
#pragma once

#include <cuda.h>

#include "fa_bwd.cuh"
#include "sm100.cuh"

namespace fa {

// Of every 8 groups of four probabilities in an unmasked tile, this many are computed on
// the FMA pipe (exp2_poly2) instead of the MUFU (3 measured best for this kernel on long
// sequences; the general kernel keeps every exponential on the MUFU).
constexpr int kBwd64EmuOf8 = 3;

struct Bwd64Cfg {
    static constexpr int D = 64;
    static constexpr int TILE = 128 * D * 2;  // one 128-row tile of Q / K / V / dO
    static constexpr int HALF = 128 * 128;    // one 128-byte column block
    static constexpr int QS = 2;              // Q_i / dO_i ring stages
    static constexpr int OFF_K = 0;                    // two K buffers (item parity)
    static constexpr int OFF_V = OFF_K + 2 * TILE;
    static constexpr int OFF_Q = OFF_V + TILE;
    static constexpr int OFF_DO = OFF_Q + QS * TILE;
    static constexpr int OFF_DS = OFF_DO + QS * TILE;  // two 32 KB dS buffers
    static constexpr int OFF_DQ = OFF_DS + 2 * 32768;  // fp32 dQ staging
    static constexpr int OFF_LSE = OFF_DQ + 128 * D * 4;
    static constexpr int OFF_DV = OFF_LSE + QS * 512;
    static constexpr int OFF_BAR = OFF_DV + QS * 512;
    static constexpr int USED = OFF_BAR + 256;
    static constexpr int SLACK = 1024;
    static constexpr int SMEM = USED + SLACK;
    static constexpr int THREADS = 512;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 320, COL_DQ = 384;
    static constexpr uint32_t COL_P = 448;
    static constexpr uint32_t P_HALF_STRIDE = 32;  // P^T pairs of queries 64h.. start 32h columns in
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct Bwd64Bars {
    uint64_t k_full[2], k_empty[2];  // K buffer of item parity; empty: S^T and dQ are done with it
    uint64_t v_full, v_empty;        // V; empty: the item's last dP^T has read it
    uint64_t q_full[Bwd64Cfg::QS];
    uint64_t do_full[Bwd64Cfg::QS];
    uint64_t stage_empty[Bwd64Cfg::QS];  // the S^T/dP^T, dV and dK issuers are done with a stage
    uint64_t s_full, s_free, dp_full, dp_read, p_full, p_free;
    uint64_t ds_full[2];   // dS_i is in buffer i & 1
    uint64_t dk_done[2];   // dK has read buffer b
    uint64_t ds_empty[2];  // dQ has read buffer b
    uint64_t dq_full, dq_empty;
    uint64_t dkv_full;   // the item's last dV and dK products are done
    uint64_t dkv_empty;  // the P/dS warps have read dK, dV out of TMEM
    uint32_t tmem_base;
};

// (tmdK and tmdV are the output maps the common launcher builds for the general kernel;
// this kernel writes dK and dV from registers and does not read them.)
template <bool BF16>
__global__ void __launch_bounds__(512, 1)
fa_bwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
                const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
    using C = Bwd64Cfg;
    constexpr int D = 64;
    constexpr int W_TMA = 8, W_SDP = 9, W_DV = 10, W_DK = 11, W_DQ0 = 12;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > (uint32_t)C::SLACK) {  // cannot happen with a 1024-aligned dynamic base
        if (threadIdx.x == 0) atomicExch(&g_status, 5);
        return;
    }
    uint8_t *smem = smem_raw + pad;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sdO = smem + C::OFF_DO;
    uint8_t *sdS = smem + C::OFF_DS;
    uint8_t *sDQ = smem + C::OFF_DQ;
    float *sLSE = reinterpret_cast<float *>(smem + C::OFF_LSE);
    float *sDv = reinterpret_cast<float *>(smem + C::OFF_DV);
    Bwd64Bars *bars = reinterpret_cast<Bwd64Bars *>(smem + C::OFF_BAR);
    static_assert(sizeof(Bwd64Bars) <= 256, "barrier area");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == W_TMA && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmdQacc);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->k_full[b], 1);
            mbar_init(&bars->k_empty[b], 2);
        }
        mbar_init(&bars->v_full, 1);
        mbar_init(&bars->v_empty, 1);
        for (int i = 0; i < C::QS; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->do_full[i], 1);
            mbar_init(&bars->stage_empty[i], 3);
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 256);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->dp_read, 256);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->p_free, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->ds_full[b], 256);
            mbar_init(&bars->dk_done[b], 1);
            mbar_init(&bars->ds_empty[b], 1);
        }
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 128);
        mbar_init(&bars->dkv_full, 2);
        mbar_init(&bars->dkv_empty, 256);
        fence_mbar_init();
    }
    if (warp == W_SDP) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_wait();  // the preprocess kernel's outputs are visible from here on

    // Persistent CTA: work items are (key tile kt, head bh), u = kt * BH + bh, so that the
    // heavier causal tiles (small kt) come first; round r of CTA c takes item r * G + c on
    // even rounds and r * G + (G - 1 - c) on odd ones.  Every role walks the same list.
    struct Item {
        int kt, bh, L;        // key tile, head, valid keys of the sequence
        int q_first, n;       // first visited query tile, number of visited query tiles
        const uint8_t *mcol;  // block-mask column of kt (nullptr: dense)
    };
    auto next_q = [&](const Item &it, int qi) -> int {
        if (it.mcol)
            while (qi < p.num_tiles && it.mcol[(size_t)qi * p.num_tiles] == 0) ++qi;
        return qi;
    };
    auto item_at = [&](int r, Item &it) -> bool {
        const int G = (int)gridDim.x;
        const int u = r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        if (u >= p.num_tiles * p.BH) return false;
        it.kt = u / p.BH;
        it.bh = u - it.kt * p.BH;
        int L = p.N;
        if (p.kv_len != nullptr) {
            L = p.kv_len[it.bh / p.H];
            L = L < 0 ? 0 : (L > p.N ? p.N : L);
        }
        it.L = L;
        it.mcol = p.bmask ? p.bmask + (size_t)it.bh * p.bmask_bh_stride + it.kt : nullptr;
        it.q_first = next_q(it, p.causal ? it.kt : 0);
        it.n = 0;
        if (it.kt * 128 < L)
            for (int qi = it.q_first; qi < p.num_tiles; qi = next_q(it, qi + 1)) ++it.n;
        return true;
    };
    auto stage_off = [](int st) { return (uint64_t)((st * C::TILE) >> 4); };
    constexpr uint32_t kIdescSq = idesc_f16(BF16, false, false, 128, 128);  // S^T, dP^T
    constexpr uint32_t kIdescTs = idesc_f16(BF16, false, true, 128, D);     // dV, dK
    constexpr uint32_t kIdescDq = idesc_f16(BF16, true, true, 128, D);      // dQ

    if (warp == W_TMA) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            auto load_q = [&](int g, int qi, int bh) -> bool {
                const int s = g % C::QS;
                if (g >= C::QS && !mbar_wait(&bars->stage_empty[s], ((g / C::QS) - 1) & 1))
                    return false;
                const size_t vec_off = (size_t)bh * p.Npad + (size_t)qi * 128;
                mbar_arrive_expect_tx(&bars->q_full[s], C::TILE + 512);
                tma_load_3d(sQ + s * C::TILE, &tmQ, &bars->q_full[s], 0, qi * 128, bh);
                bulk_load(sLSE + s * 128, p.nlse2 + vec_off, 512, &bars->q_full[s]);
                mbar_arrive_expect_tx(&bars->do_full[s], C::TILE + 512);
                tma_load_3d(sdO + s * C::TILE, &tmdO, &bars->do_full[s], 0, qi * 128, bh);
                bulk_load(sDv + s * 128, p.ndvec + vec_off, 512, &bars->do_full[s]);
                return true;
            };
            bool ok = true;
            int gi = 0, tn = 0;
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.n == 0) continue;
                // the item's first Q/dO tiles go in while the previous item still runs; K
                // into the buffer of the item two back once its S^T and dQ products are done,
                // V once the previous item's last dP^T has read it
                const int pre = min(it.n, C::QS - 1);
                const int kb = tn & 1;
                int qi = it.q_first;
                for (int i = 0; ok && i < pre; ++i, qi = next_q(it, qi + 1)) ok = load_q(gi + i, qi, it.bh);
                if (ok && tn >= 2) ok = mbar_wait(&bars->k_empty[kb], ((tn >> 1) - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars->k_full[kb], C::TILE);
                tma_load_3d(sK + kb * C::TILE, &tmK, &bars->k_full[kb], 0, it.kt * 128, it.bh);
                if (tn >= 1 && !mbar_wait(&bars->v_empty, (tn - 1) & 1)) break;
                mbar_arrive_expect_tx(&bars->v_full, C::TILE);
                tma_load_3d(sV, &tmV, &bars->v_full, 0, it.kt * 128, it.bh);
                for (int i = pre; ok && i < it.n; ++i, qi = next_q(it, qi + 1)) ok = load_q(gi + i, qi, it.bh);
                gi += it.n;
                ++tn;
            }
        }
    } else if (warp == W_SDP) {
        // ------------------------------ S^T and dP^T ------------------------------
        if (lane == 0) {
            const uint64_t k_kmaj = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t v_kmaj = smem_desc_sw128(smem_u32(sV), 16, 1024);
            const uint64_t q_kmaj = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t do_kmaj = smem_desc_sw128(smem_u32(sdO), 16, 1024);
            bool ok = true;
            int gi = 0, tn = 0;
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.n == 0) continue;
                const int kb = tn & 1;
                if (!mbar_wait(&bars->k_full[kb], (tn >> 1) & 1)) break;
                const uint64_t kd = k_kmaj + stage_off(kb);
                for (int i = 0; i < it.n; ++i) {
                    const int g = gi + i, s = g % C::QS;
                    // S^T_g over S^T_{g-1} once every P/dS warp has read it
                    if ((g > 0 && !mbar_wait(&bars->s_free, (g - 1) & 1)) ||
                        !mbar_wait(&bars->q_full[s], (g / C::QS) & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + C::COL_S, kd + (uint64_t)(kk * 2),
                               q_kmaj + stage_off(s) + (uint64_t)(kk * 2), kIdescSq, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->s_full);
                    // dP^T_g over dP^T_{g-1} once every P/dS warp has loaded it
                    if ((i == 0 && !mbar_wait(&bars->v_full, tn & 1)) ||
                        (g > 0 && !mbar_wait(&bars->dp_read, (g - 1) & 1)) ||
                        !mbar_wait(&bars->do_full[s], (g / C::QS) & 1)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + C::COL_DP, v_kmaj + (uint64_t)(kk * 2),
                               do_kmaj + stage_off(s) + (uint64_t)(kk * 2), kIdescSq, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->dp_full);
                    mma_commit(&bars->stage_empty[s]);
                }
                if (!ok) break;
                mma_commit(&bars->k_empty[kb]);  // (with the item's dQ products)
                mma_commit(&bars->v_empty);
                gi += it.n;
                ++tn;
            }
        }
    } else if (warp == W_DV || warp == W_DK) {
        // ------------------------------ dV / dK ------------------------------------
        // dV += P^T_g dO_g (A = P^T from TMEM) or dK += dS^T_g Q_g (A = dS^T, the K-major
        // view of dS buffer g & 1); B is the MN-major dO / Q tile.
        if (lane == 0) {
            const bool is_dv = warp == W_DV;
            const uint64_t b_mn = smem_desc_sw128(smem_u32(is_dv ? sdO : sQ), C::HALF, 1024);
            const uint64_t dst_k = smem_desc_sw128(smem_u32(sdS), 16, 1024);
            bool ok = true;
            int gi = 0, tn = 0;
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.n == 0) continue;
                for (int i = 0; i < it.n; ++i) {
                    const int g = gi + i, s = g % C::QS, b = g & 1;
                    if (!(is_dv ? mbar_wait(&bars->p_full, g & 1)
                                : mbar_wait(&bars->ds_full[b], (g >> 1) & 1)) ||
                        // dV and dK restart from zero: the previous item's epilogue has read them
                        (i == 0 && tn > 0 && !mbar_wait(&bars->dkv_empty, (tn - 1) & 1))) { ok = false; break; }
                    tc_fence_after();
                    if (is_dv) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ts(tmem + C::COL_DV,
                                   tmem + C::COL_P + (kk >> 2) * C::P_HALF_STRIDE + (kk & 3) * 8,
                                   b_mn + stage_off(s) + (uint64_t)(kk * 2048 >> 4), kIdescTs,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&bars->p_free);
                    } else {
                        // K step kk: queries 16kk..16kk+15, i.e. 32 bytes of the 128-byte rows
                        // of query half kk / 4
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tmem + C::COL_DK,
                                   dst_k + (uint64_t)((b * 32768 + (kk >> 2) * 16384 + (kk & 3) * 32) >> 4),
                                   b_mn + stage_off(s) + (uint64_t)(kk * 2048 >> 4), kIdescTs,
                                   (i > 0 || kk > 0) ? 1u : 0u);
                        mma_commit(&bars->dk_done[b]);
                    }
                    mma_commit(&bars->stage_empty[s]);
                }
                mma_commit(&bars->dkv_full);
                gi += it.n;
                ++tn;
            }
        }
    } else if (warp >= W_DQ0) {
        // ------------------------------ dQ products and drain ----------------------
        const int quarter = warp & 3;
        const int rrow = quarter * 32 + lane;       // query row in the tile = TMEM lane
        const int gt = threadIdx.x - W_DQ0 * 32;    // 0..127 inside this warpgroup
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const uint64_t ds_mn = smem_desc_sw128(smem_u32(sdS), 16384, 1024);
        const uint64_t k_mn0 = smem_desc_sw128(smem_u32(sK), C::HALF, 1024);
        bool ok = true;
        int gi = 0, tn = 0;
        Item it;
        for (int rr = 0; ok && item_at(rr, it); ++rr) {
        const int bh = it.bh;
        for (int i = 0, qi = it.q_first; i < it.n; ++i, qi = next_q(it, qi + 1)) {
            const int g = gi + i;
            if (warp == W_DQ0) {
                // dQ_g = dS_g K, issued by lane 0 of the first drain warp
                bool ok1 = true;
                if (lane == 0) {
                    const int b = g & 1, kb = tn & 1;
                    const uint64_t k_mn = k_mn0 + stage_off(kb);
                    ok1 = (i > 0 || mbar_wait(&bars->k_full[kb], (tn >> 1) & 1)) &&
                          mbar_wait(&bars->ds_full[b], (g >> 1) & 1) &&
                          (g == 0 || mbar_wait(&bars->dq_empty, (g - 1) & 1));
                    if (ok1) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            mma_ss(tmem + C::COL_DQ, ds_mn + (uint64_t)((b * 32768 + kk * 2048) >> 4),
                                   k_mn + (uint64_t)(kk * 2048 >> 4), kIdescDq, kk > 0 ? 1u : 0u);
                        mma_commit(&bars->dq_full);
                        mma_commit(&bars->ds_empty[b]);
                        if (i + 1 == it.n) mma_commit(&bars->k_empty[kb]);  // K_kb is free
                    }
                }
                __syncwarp();
                ok = __shfl_sync(0xffffffffu, ok1 ? 1 : 0, 0) != 0;
            }
            // The 128 drain threads agree on the wait's outcome before the warp-wide TMEM
            // loads and the named barriers below, so a timeout makes all of them leave.
            if (!named_bar_and(2, 128, ok && mbar_wait(&bars->dq_full, g & 1))) { ok = false; break; }
            tc_fence_after();
            // [128 rows][32 fp32] boxes, 16-byte chunks swizzled by row % 8, all D / 32 staged
            // and handed to one TMA reduce-add into the fp32 accumulator
            if (gt == 0) bulk_wait_group_read<0>();  // the previous reduce has read the stage
            named_bar_sync(2, 128);
#pragma unroll
            for (int bx = 0; bx < D / 32; ++bx) {
                uint32_t w[32];
                tmem_ld32(tmem + lane_base + C::COL_DQ + bx * 32, w);
                uint8_t *rowp = sDQ + bx * 16384 + rrow * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(rowp + ((c ^ (rrow & 7)) << 4)) =
                        make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
            }
            tc_fence_before();
            mbar_arrive(&bars->dq_empty);  // every dQ column is out of TMEM
            fence_proxy_async_smem();
            named_bar_sync(2, 128);
            if (gt == 0) {
#pragma unroll
                for (int bx = 0; bx < D / 32; ++bx)
                    tma_reduce_add_3d(&tmdQacc, sDQ + bx * 16384, bx * 32, qi * 128, bh);
                bulk_commit_group();
            }
        }
        gi += it.n;
        if (it.n > 0) ++tn;
        }
        if (gt == 0) bulk_wait_group<0>();
    } else {
        // ------------------------------ P / dS warps ------------------------------
        const int quarter = warp & 3;
        const int h = warp >> 2;             // query half: columns 64h .. 64h + 63
        const int t = quarter * 32 + lane;   // key row in the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const float sl2 = p.scale_log2;
        const float2 sl2x2 = make_float2(sl2, sl2);
        // dK (times the softmax scale) and dV of key tile kt, head bh, row t, columns
        // 32h .. 32h + 31, from TMEM (once the item's last dK / dV products are done) or
        // zero (a key tile no query visits), written as 16-bit values from registers.
        auto store_dkdv = [&](int kt, int bh, int etn, bool from_tmem) -> bool {
            if (from_tmem) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->dkv_full, etn & 1))) return false;
                tc_fence_after();
            }
            const int row = kt * 128 + t;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                uint32_t w[32];
                if (from_tmem) {
                    tmem_ld32(tmem + lane_base + (which == 0 ? C::COL_DV : C::COL_DK) + h * 32, w);
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) w[k] = 0u;
                }
                const float mul = which == 0 ? 1.f : p.scale;
                uint32_t wv[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    wv[k] = pack2<BF16>(__uint_as_float(w[2 * k]) * mul, __uint_as_float(w[2 * k + 1]) * mul);
                if (row < p.N) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        static_cast<uint16_t *>(which == 0 ? p.dv : p.dk) +
                        ((size_t)bh * p.N + row) * D + 32 * h);
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        dst[c] = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                }
            }
            if (from_tmem) {
                // dK, dV are out of TMEM: the next item's first dV / dK products may start
                tc_fence_before();
                mbar_arrive(&bars->dkv_empty);
            }
            return true;
        };
        bool ok = true;
        int gi = 0, tn = 0;
        int pend_kt = -1, pend_bh = 0, pend_tn = 0;  // item whose dK, dV are still in TMEM
        Item it;
        for (int rr = 0; ok && item_at(rr, it); ++rr) {
        const int kt = it.kt, bh = it.bh, L = it.L, n = it.n;
        const bool key_ok = kt * 128 + t < L;
        if (n == 0) {
            store_dkdv(kt, bh, 0, false);
            continue;
        }
        for (int i = 0, qi = it.q_first; ok && i < n; ++i, qi = next_q(it, qi + 1)) {
            const int g = gi + i;
            const int s = g % C::QS;
            // (waits are voted on per warp: the loop body has warp-wide TMEM loads and stores)
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, g & 1) &&
                                             mbar_wait(&bars->q_full[s], (g / C::QS) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // P^T for queries 64h .. 64h + 63 of this key row, packed in 16-bit pairs
            uint32_t Pw[32];
            {
                uint32_t w[64];
                tmem_ld64(tmem + lane_base + C::COL_S + h * 64, w);
                tc_fence_before();
                mbar_arrive(&bars->s_free);  // S^T may now be overwritten by S_{g+1}
                const float *nl2 = sLSE + s * 128 + h * 64;  // -LSE2 of the 64 queries
                const bool diag = p.causal && (qi == kt);
                const bool tile_masked = diag || (kt * 128 + 128 > L);
                if (!tile_masked) {
#pragma unroll
                    for (int k = 0; k < 64; k += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(nl2 + k);
                        const float2 x01 = __ffma2_rn(
                            make_float2(__uint_as_float(w[k]), __uint_as_float(w[k + 1])), sl2x2,
                            make_float2(l4.x, l4.y));
                        const float2 x23 = __ffma2_rn(
                            make_float2(__uint_as_float(w[k + 2]), __uint_as_float(w[k + 3])), sl2x2,
                            make_float2(l4.z, l4.w));
                        float2 e01, e23;
                        if (((k >> 2) & 7) < kBwd64EmuOf8) {
                            e01 = exp2_poly2(x01);
                            e23 = exp2_poly2(x23);
                        } else {
                            e01 = make_float2(ex2(x01.x), ex2(x01.y));
                            e23 = make_float2(ex2(x23.x), ex2(x23.y));
                        }
                        Pw[k >> 1] = pack2<BF16>(e01.x, e01.y);
                        Pw[(k >> 1) + 1] = pack2<BF16>(e23.x, e23.y);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 64; k += 4) {
                        const int c = h * 64 + k;  // query column in the tile
                        const float4 l4 = *reinterpret_cast<const float4 *>(nl2 + k);
                        float p0 = ex2(fmaf(__uint_as_float(w[k]), sl2, l4.x));
                        float p1 = ex2(fmaf(__uint_as_float(w[k + 1]), sl2, l4.y));
                        float p2 = ex2(fmaf(__uint_as_float(w[k + 2]), sl2, l4.z));
                        float p3 = ex2(fmaf(__uint_as_float(w[k + 3]), sl2, l4.w));
                        // keys past the valid length, and queries before the key (causal)
                        if (!key_ok || (diag && c < t)) p0 = 0.f;
                        if (!key_ok || (diag && c + 1 < t)) p1 = 0.f;
                        if (!key_ok || (diag && c + 2 < t)) p2 = 0.f;
                        if (!key_ok || (diag && c + 3 < t)) p3 = 0.f;
                        Pw[k >> 1] = pack2<BF16>(p0, p1);
                        Pw[(k >> 1) + 1] = pack2<BF16>(p2, p3);
                    }
                }
            }
            // the previous item's dK, dV, whose last products ran while P was formed
            if (i == 0 && pend_kt >= 0) {
                if (!store_dkdv(pend_kt, pend_bh, pend_tn, true)) {
                    ok = false;
                    break;
                }
                pend_kt = -1;
            }
            // the P^T columns: dV_{g-1} must have read P^T_{g-1}
            if (g > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->p_free, (g - 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            tmem_st32(tmem + lane_base + C::COL_P + h * C::P_HALF_STRIDE, Pw);
            tc_fence_before();
            mbar_arrive(&bars->p_full);

            if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full, g & 1) &&
                                             mbar_wait(&bars->do_full[s], (g / C::QS) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float *ndv = sDv + s * 128 + h * 64;  // -D of the 64 queries
            uint32_t wdp[64];
            tmem_ld64(tmem + lane_base + C::COL_DP + h * 64, wdp);
            tc_fence_before();
            mbar_arrive(&bars->dp_read);  // dP^T may now be overwritten by dP^T_{g+1}
            // dS buffer g & 1: dK_{g-2} and dQ_{g-2} have read it
            const int b = g & 1;
            if (g >= 2 && !__all_sync(0xffffffffu, mbar_wait(&bars->dk_done[b], ((g >> 1) - 1) & 1) &&
                                                       mbar_wait(&bars->ds_empty[b], ((g >> 1) - 1) & 1))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint32_t *w = wdp + cc * 32;
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float2 nd2 = *reinterpret_cast<const float2 *>(ndv + cc * 32 + k);
                    // dS = P o (dP - D): the difference in fp32 (one packed add), rounded to
                    // 16 bits, times the 16-bit P pair in one packed multiply
                    const float2 diff = __fadd2_rn(make_float2(__uint_as_float(w[k]),
                                                               __uint_as_float(w[k + 1])), nd2);
                    pk[k >> 1] = mul2<BF16>(Pw[cc * 16 + (k >> 1)], pack2<BF16>(diff.x, diff.y));
                }
                // dS -> shared memory: [query block h (64 queries)][key row t][128 bytes],
                // 128-byte swizzle (the K-major dS^T of dK, the MN-major dS of dQ)
                uint8_t *rowp = sdS + b * 32768 + h * 16384 + t * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int chunk = cc * 4 + q4;
                    *reinterpret_cast<uint4 *>(rowp + ((chunk ^ (t & 7)) << 4)) =
                        make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars->ds_full[b]);
        }

        if (!ok) break;
        pend_kt = kt;
        pend_bh = bh;
        pend_tn = tn;
        gi += n;
        ++tn;
        }  // items
        pdl_launch_dependents();
        if (ok && pend_kt >= 0) store_dkdv(pend_kt, pend_bh, pend_tn, true);  // the last item
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == W_SDP) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa
