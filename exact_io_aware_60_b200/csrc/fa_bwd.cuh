// fa_bwd.cuh -- backward pass of exact tiled attention on sm_100a.
//
// The method (anthology note "NOTE-005: FlashAttention", sections "Method" and "Key
// components"; aicassindra FlashAttention architecture page, "The architecture: every
// piece explained"): the backward pass does not read a stored N x N probability matrix;
// it recomputes each probability block on chip from Q, K and the statistics the forward
// pass kept (here LSE = m + ln l), then applies the chain rule of the op chain
//   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
// (The pages state the recomputation but print no gradient formulas; these are the
// textbook derivatives of softmax and of the two products.)
//
// Three kernels, all on the caller's stream:
//   1. fa_bwd_prep_kernel: D_i = rowsum(dO o O) in fp32 and LSE in base 2, both stored
//      negated (so that the main kernel's P = 2^(S scale log2e - LSE2) and dP - D are one
//      packed fused multiply-add or add each), padded to whole 128-row tiles (-inf for the
//      LSE where there is no row); and zeroes the fp32 dQ accumulator.
//   2. fa_bwd_kernel: persistent CTAs (one per SM) walking (128-key tile, head) items, each
//      looping over the 128-query tiles that can see its keys (causal: only tiles on or
//      below the diagonal).
//        warp 8      TMA producer: K, V once per item; Q_i, dO_i (+ LSE_i, D_i) into a
//                    2/3-stage ring.
//        warp 9      MMA issuer (one thread), all on tcgen05 with fp32 TMEM accumulators:
//                    S^T = K Q_i^T, dP^T = V dO_i^T, dV += P^T dO_i, dK += dS^T Q_i
//                    (P^T, dS^T read from TMEM), dQ_i = dS K (dS from shared memory).
//        warp 14     (d = 64 without the causal mask) a second MMA issuer, which takes dK_i
//                    and dP^T_{i+1} from warp 9 (see BwdCfg::TWO_ISS).
//        warps 0..7  one key row per thread and half of the query columns per warp
//                    (lane quarter w % 4, query half w / 4): P^T = 2^(S^T scale log2e -
//                    LSE2), written back to TMEM as 16-bit pairs; dS^T = P^T o (dP^T - D)
//                    to TMEM and, in the transposed operand layout, to shared memory;
//                    the item's epilogue writes dK, dV (in the non-causal d = 64 variant
//                    the dQ drain warps write them instead, see BwdCfg::DRAIN_EPI).
//        warps 10..13 drain dQ_i from TMEM through a swizzled shared-memory staging tile
//                    and a TMA reduce-add into the fp32 accumulator in global memory (own
//                    staging area at d = 64; at d = 128, where shared memory is full, the
//                    dS buffer in two 64-column rounds, free between the dQ MMA and dS_{i+1}).
//   3. fa_bwd_convert_kernel: dQ = scale * dQ_acc in the input dtype.
#pragma once

#include <cuda.h>

#include "dropout.cuh"
#include "sm100.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;

// --------------------------------------------------------------------------- prep

struct BwdPrepParams {
    const void *o;
    const void *dout;
    const float *lse;
    float *nlse2;  // [BH][Npad]: -LSE in base 2 (-inf for padding rows)
    float *ndvec;  // [BH][Npad]: -D (times dscale)
    float4 *dq_acc;
    long long dq_acc_vec4;  // number of float4 in dq_acc
    float dscale;           // D is stored times this (1, or 1 / keep_scale with dropout)
    int N;
    int Npad;
    long long BH;
};

// Each warp handles 32 / (D/8) consecutive padded rows per step (D/8 threads per row,
// 8 elements of O and dO each); every lane runs the same number of steps, so the
// group shuffles never diverge.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const BwdPrepParams p) {
    constexpr int G = D / 8;           // threads per row
    constexpr int RPW = 32 / G;        // rows per warp step
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    // The accumulator is the backward pass's own scratch, which no earlier kernel of the
    // stream reads or writes while this call runs: it is zeroed before the wait, so that
    // the zeroing overlaps the tail of the kernel before (the forward pass, in a training
    // step).  O and dO may be that kernel's outputs, so they are read after the wait.
    for (long long i = tid; i < p.dq_acc_vec4; i += nthreads)
        p.dq_acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    pdl_wait();
    pdl_launch_dependents();
    const long long rows_total = p.BH * p.Npad;
    const int lane = threadIdx.x & 31;
    const int g = lane % G;
    const long long warp_id = tid >> 5;
    const long long nwarps = nthreads >> 5;
    for (long long base = warp_id * RPW; base < rows_total; base += nwarps * RPW) {
        const long long rr = base + lane / G;
        float acc = 0.f;
        float l2 = INFINITY;  // LSE in base 2; +inf (P = 0) for rows that do not exist
        if (rr < rows_total) {
            const long long bh = rr / p.Npad;
            const int r = (int)(rr - bh * p.Npad);
            if (r < p.N) {
                const size_t off = ((size_t)bh * p.N + r) * D + g * 8;
                const uint4 a = *reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const uint16_t *>(p.o) + off);
                const uint4 bb = *reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const uint16_t *>(p.dout) + off);
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
                const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 x = unpack2<BF16>(aw[k]);
                    const float2 y = unpack2<BF16>(bw[k]);
                    acc = fmaf(x.x, y.x, acc);
                    acc = fmaf(x.y, y.y, acc);
                }
                const float lse = p.lse[(size_t)bh * p.N + r];
                l2 = (lse == -INFINITY) ? INFINITY : lse * kLog2e;
            }
        }
#pragma unroll
        for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (g == 0 && rr < rows_total) {
            p.ndvec[rr] = -acc * p.dscale;
            p.nlse2[rr] = -l2;
        }
    }
}

// --------------------------------------------------------------------------- convert

template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_convert_kernel(const float4 *acc, uint2 *out,
                                                             long long n_vec4, float scale) {
    pdl_wait();
    const long long nthreads = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec4; i += nthreads) {
        const float4 a = acc[i];
        out[i] = make_uint2(pack2<BF16>(a.x * scale, a.y * scale), pack2<BF16>(a.z * scale, a.w * scale));
    }
    // Only now may the next kernel start: the next backward call's preprocess zeroes this
    // accumulator before it waits (the same workspace, or the static one, may be reused).
    pdl_launch_dependents();
}

// --------------------------------------------------------------------------- main

struct BwdParams {
    const float *nlse2;  // [BH][Npad], minus the log2-domain LSE (-inf for padding rows)
    // Block-sparse attention: uint8 [heads][T][T]; key tile kt visits only the query tiles
    // qi with mask[qi][kt] != 0.  nullptr = dense.
    const uint8_t *bmask;
    long long bmask_bh_stride;  // 0: one mask for every (batch, head)
    const float *ndvec;  // [BH][Npad], -D
    float *dq_acc;      // [BH][N][D] fp32
    const int *kv_len;
    int N;
    int Npad;
    int BH;
    int H;
    int num_tiles;  // ceil(N / 128)
    float scale;
    float scale_log2;
    int causal;
    // Dropout variant only: the mask generator, and the epilogue multipliers of dV
    // (keep_scale) and dK (scale * keep_scale).
    DropoutParams drop;
    float dv_mul;
    float dk_mul;
};

// TWO: (d = 64) two MMA-issuing threads instead of one (see TWO_ISS).
template <int D, bool TWO = false>
struct BwdCfg {
    static constexpr int TILE = 128 * D * 2;  // one 128-row tile of Q / K / V / dO
    static constexpr int HALF = 128 * 128;    // one 128-byte column block of a tile
    static constexpr int HALVES = D / 64;
    // dQ leaves TMEM through a shared-memory staging area and a TMA reduce-add: its own
    // 32 KB at d = 64; at d = 128 (no room) the dS buffer, 64 columns at a time, which is
    // free between the dQ MMA that reads dS_i and the P/dS warps' writing of dS_{i+1}.
    static constexpr bool DQ_IN_DS = (D == 128);
    // d = 64: P^T gets its own TMEM columns, so S_{i+1} can overwrite S_i as soon as it
    // has been read.  d = 128: TMEM is full; P^T overwrites S^T and S_{i+1} waits for dV_i.
    static constexpr bool P_OWN = (D == 64);
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + TILE;
    // Q_i / dO_i ring: a stage is released only once dQ_i is done, and S_{i+2} needs its
    // refill right after, so d = 64 keeps three stages to hide the load latency; d = 128
    // has room for two.
    static constexpr int QS = (D == 64) ? 3 : 2;
    static constexpr int OFF_Q = OFF_V + TILE;        // QS stages
    static constexpr int OFF_DO = OFF_Q + QS * TILE;  // QS stages
    static constexpr int OFF_DS = OFF_DO + QS * TILE; // 128 x 128 16-bit, operand layout
    static constexpr int OFF_DQ = OFF_DS + 32768;    // fp32 staging (d = 64 only)
    static constexpr int DQ_BYTES = DQ_IN_DS ? 0 : 128 * D * 4;
    static constexpr int OFF_LSE = OFF_DQ + DQ_BYTES;  // QS x 512 B
    static constexpr int OFF_DV = OFF_LSE + QS * 512;  // QS x 512 B
    static constexpr int OFF_BAR = OFF_DV + QS * 512;
    static constexpr int USED = OFF_BAR + 512;  // barriers and the item cache
    // d = 128 uses all 227 KB: no room for alignment slack; the kernel checks instead.
    static constexpr int SLACK = (USED + 1024 <= 232448) ? 1024 : 0;
    static constexpr int SMEM = USED + SLACK;
    // warps 0..7: P / dS (lane quarter w % 4, query half w / 4); 8: TMA; 9: MMA;
    // 10..13: dQ drain (lane quarters 2, 3, 0, 1).
    // Two MMA-issuing threads (d = 64, used without the causal mask): A (warp 9) issues S^T,
    // dV and dQ; B (warp 14) issues dK_i and then dP^T_{i+1}, which overwrites the dS^T_i
    // that dK_i reads: in one thread's order no completion wait is needed between them.
    // Measured on B200, this shortens the long items of non-causal shapes by 2-3%, while the
    // short, uneven items of causal shapes end less evenly across CTAs with it.
    static constexpr bool TWO_ISS = TWO && (D == 64);
    // With TWO_ISS the dQ drain warps, idle at the end of an item, also write its dK and dV
    // (through their own staging area), so the P/dS warps go straight on to the next item:
    // non-causal backward 1.5-3% faster on B200.  On the short, uneven causal items it came
    // out 1% slower (dK and dV then leave TMEM later, after the last dQ drain), and at
    // d = 128 the drain's staging is the dS buffer: there the P/dS warps write dK and dV.
    static constexpr bool DRAIN_EPI = TWO_ISS;
    static constexpr int THREADS = TWO_ISS ? 480 : 448;
    static constexpr int W_TMA = 8, W_MMA = 9, W_DQ0 = 10, W_MMA2 = TWO_ISS ? 14 : 9;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t COL_S = 0;
    static constexpr uint32_t COL_DP = 128;
    static constexpr uint32_t COL_DV = 256;
    static constexpr uint32_t COL_DK = 256 + D;
    static constexpr uint32_t COL_DQ = (D == 64) ? 384 : 128;  // d = 128: aliases dP^T
    static constexpr uint32_t COL_P = P_OWN ? 448 : COL_S;
    // Column of the 16-bit pairs of queries 64h..64h+63 inside the P^T / dS^T areas:
    // each query half is written over columns its own warp has already read.
    static constexpr uint32_t P_HALF_STRIDE = P_OWN ? 32 : 64;
    static constexpr uint32_t DS_HALF_STRIDE = 64;
};

struct BwdBars {
    uint64_t kv_full;
    uint64_t q_full[3];
    uint64_t do_full[3];
    uint64_t stage_empty[3];
    uint64_t dq_stage_free;  // d = 128: the dQ drain has finished with the dS buffer
    uint64_t s_full, s_free, dp_full, p_full, p_free, ds_full, ds_empty, dq_full, dq_empty,
        dkv_full, dkv_empty;
    uint32_t tmem_base;
    ItemCache items;  // SCHED: this CTA's list of the launcher's schedule
};
static_assert(sizeof(BwdBars) <= 512, "the barrier block has 512 bytes of shared memory");

// DROP: dropout.  With K the keep mask and r = keep_scale, the chain rule gives
//   dV = r (P o K)^T dO,  dP = r K o (dO V^T),  D = rowsum(dO o O),  dS = P o (dP - D);
// the kernel computes dS' = P o (K o (dO V^T) - D / r) (D / r comes from the preprocess)
// and folds r into the dV, dK and dQ output multipliers.
// SCHED: the launcher passes a static schedule of the items (ItemSchedule).
template <int D, bool BF16, bool DROP, bool SCHED = false, bool TWO = false>
__global__ void __launch_bounds__(BwdCfg<D, TWO>::THREADS, 1)
fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
              const __grid_constant__ CUtensorMap tmdK, const __grid_constant__ CUtensorMap tmdV,
              const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p,
              const __grid_constant__ std::conditional_t<SCHED, ItemSchedule, NoSchedule> sched) {
    using C = BwdCfg<D, TWO>;
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
    BwdBars *bars = reinterpret_cast<BwdBars *>(smem + C::OFF_BAR);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Persistent CTA: work items are (key tile kt, head bh), numbered u = kt * BH + bh at
    // d = 64 so that heavier causal tiles (small kt) come first, and u = bh * T + kt at
    // d = 128 (head-major: the long-sequence case, where one head's fp32 dQ accumulator
    // should stay in L2).  Round r of CTA c takes item r * G + c on even rounds and
    // r * G + (G - 1 - c) on odd ones (G = grid size); the zigzag evens out the causal
    // work.  With a schedule from the launcher (dense and causal shapes of up to
    // kSchedMaxItems items), CTA c walks its list of items instead.  Every role walks the
    // same list on its own.

    if (warp == C::W_TMA && lane == 0) {
        if constexpr (SCHED) item_cache_fill(bars->items, sched);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmdK);
        tma_prefetch_desc(&tmdV);
        tma_prefetch_desc(&tmdQacc);
        mbar_init(&bars->kv_full, 1);
        for (int i = 0; i < C::QS; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->do_full[i], 1);
            mbar_init(&bars->stage_empty[i], C::TWO_ISS ? 2 : 1);  // each issuer's last reader
        }
        mbar_init(&bars->s_full, 1);
        mbar_init(&bars->s_free, 256);
        mbar_init(&bars->dp_full, 1);
        mbar_init(&bars->p_full, 256);
        mbar_init(&bars->p_free, 1);
        mbar_init(&bars->ds_full, 256);
        mbar_init(&bars->ds_empty, 1);
        mbar_init(&bars->dq_full, 1);
        mbar_init(&bars->dq_empty, 128);
        mbar_init(&bars->dq_stage_free, 1);
        mbar_init(&bars->dkv_full, C::TWO_ISS ? 2 : 1);  // each issuer's item end
        mbar_init(&bars->dkv_empty, C::DRAIN_EPI ? 128 : 256);
        fence_mbar_init();
    }
    if (warp == C::W_MMA) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_wait();  // the preprocess kernel's outputs are visible from here on

    // Inputs (key lengths, block mask) are read only after the wait above.
    struct Item {
        int kt, bh, L;        // key tile, head, valid keys of the sequence
        int q_first, n;       // first visited query tile, number of visited query tiles
        const uint8_t *mcol;  // block-mask column of kt (nullptr: dense)
    };
    // Block-sparse walk: next query tile at or after qi whose (qi, kt) entry is set.
    auto next_q = [&](const Item &it, int qi) -> int {
        if (it.mcol)
            while (qi < p.num_tiles && it.mcol[(size_t)qi * p.num_tiles] == 0) ++qi;
        return qi;
    };
    auto item_at = [&](int r, Item &it) -> bool {
        int u;
        if constexpr (SCHED) {  // the launcher's balanced assignment
            if (!item_cache_get(bars->items, sched, r, u)) return false;
        } else {
            const int G = (int)gridDim.x;
            u = r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        }
        if (u >= p.num_tiles * p.BH) return false;
        if (D == 128) {
            // head-major: the CTAs of a round share one or two heads, whose fp32 dQ
            // accumulator then stays in L2 while every key tile reduces into it
            it.bh = u / p.num_tiles;
            it.kt = u - it.bh * p.num_tiles;
        } else {
            it.kt = u / p.BH;
            it.bh = u - it.kt * p.BH;
        }
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

    if (warp == C::W_TMA) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0) {
            // Q_i, dO_i (+ LSE_i, D_i) of global iteration g into ring stage g % QS.
            auto load_q = [&](int g, int qi, int bh) -> bool {
                const int s = g % C::QS;
                if (g >= C::QS && !mbar_wait(&bars->stage_empty[s], ((g / C::QS) - 1) & 1))
                    return false;
                const size_t vec_off = (size_t)bh * p.Npad + (size_t)qi * 128;
                mbar_arrive_expect_tx(&bars->q_full[s], C::TILE + 512);
                for (int hf = 0; hf < C::HALVES; ++hf)
                    tma_load_3d(sQ + s * C::TILE + hf * C::HALF, &tmQ, &bars->q_full[s], hf * 64,
                                qi * 128, bh);
                bulk_load(sLSE + s * 128, p.nlse2 + vec_off, 512, &bars->q_full[s]);
                mbar_arrive_expect_tx(&bars->do_full[s], C::TILE + 512);
                for (int hf = 0; hf < C::HALVES; ++hf)
                    tma_load_3d(sdO + s * C::TILE + hf * C::HALF, &tmdO, &bars->do_full[s],
                                hf * 64, qi * 128, bh);
                bulk_load(sDv + s * 128, p.ndvec + vec_off, 512, &bars->do_full[s]);
                return true;
            };
            bool ok = true;
            int gi = 0, tn = 0;  // global iteration, items with work so far
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.n == 0) continue;
                // The first Q/dO tiles of this item go in as soon as their stages free up
                // (while the previous item still runs); K and V wait for the previous
                // item's last MMA.
                const int pre = min(it.n, C::QS - 1);
                int qi = it.q_first;
                for (int i = 0; ok && i < pre; ++i, qi = next_q(it, qi + 1)) ok = load_q(gi + i, qi, it.bh);
                if (ok && tn > 0) ok = mbar_wait(&bars->dkv_full, (tn - 1) & 1);
                if (!ok) break;
                mbar_arrive_expect_tx(&bars->kv_full, 2 * C::TILE);
                for (int hf = 0; hf < C::HALVES; ++hf) {
                    tma_load_3d(sK + hf * C::HALF, &tmK, &bars->kv_full, hf * 64, it.kt * 128, it.bh);
                    tma_load_3d(sV + hf * C::HALF, &tmV, &bars->kv_full, hf * 64, it.kt * 128, it.bh);
                }
                for (int i = pre; ok && i < it.n; ++i, qi = next_q(it, qi + 1)) ok = load_q(gi + i, qi, it.bh);
                gi += it.n;
                ++tn;
            }
        }
    } else if (warp == C::W_MMA || warp == C::W_MMA2) {
        // ------------------------------ MMA issuers -------------------------------
        if (lane == 0) {
            constexpr uint32_t kIdescSq = idesc_f16(BF16, false, false, 128, 128);  // S^T, dP^T
            constexpr uint32_t kIdescTs = idesc_f16(BF16, false, true, 128, D);     // dV, dK
            constexpr uint32_t kIdescDq = idesc_f16(BF16, true, true, 128, D);      // dQ
            // Descriptors are built once; per k-step and per stage only the 16-byte start
            // address field changes, by compile-time offsets.
            const uint64_t k_kmaj = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t v_kmaj = smem_desc_sw128(smem_u32(sV), 16, 1024);
            const uint64_t q_kmaj = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t do_kmaj = smem_desc_sw128(smem_u32(sdO), 16, 1024);
            const uint64_t q_mn = smem_desc_sw128(smem_u32(sQ), C::HALF, 1024);
            const uint64_t do_mn = smem_desc_sw128(smem_u32(sdO), C::HALF, 1024);
            const uint64_t k_mn = smem_desc_sw128(smem_u32(sK), C::HALF, 1024);
            const uint64_t ds_mn = smem_desc_sw128(smem_u32(sdS), 16384, 1024);
            // X^T = A B^T with A, B both [128 rows][D] K-major tiles.
            auto mma_square = [&](uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t off = (uint64_t)(((kk >> 2) * C::HALF + (kk & 3) * 32) >> 4);
                    mma_ss(d_tmem, a_desc + off, b_desc + off, kIdescSq, kk > 0 ? 1u : 0u);
                }
            };
            // D[128 x D] (+)= A_tmem[128 x 128] * B[128 rows][D] (MN-major B).  The A pairs
            // of queries 64..127 start `half_stride` columns after those of queries 0..63.
            auto mma_tmem_a = [&](uint32_t d_tmem, uint32_t a_tmem, uint32_t half_stride,
                                  uint64_t b_desc, bool acc) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ts(d_tmem, a_tmem + (kk >> 2) * half_stride + (kk & 3) * 8,
                           b_desc + (uint64_t)(kk * 2048 >> 4), kIdescTs,
                           (acc || kk > 0) ? 1u : 0u);
            };
            auto stage_off = [](int st) { return (uint64_t)((st * C::TILE) >> 4); };
            bool ok = true;
            int gi = 0, tn = 0;  // global iteration, items with work so far
            Item it;
            if constexpr (C::TWO_ISS) {
                const bool is_a = warp == C::W_MMA;
                for (int r = 0; ok && item_at(r, it); ++r) {
                    const int n = it.n;
                    if (n == 0) continue;
                    if (!mbar_wait(&bars->kv_full, tn & 1)) break;
                    tc_fence_after();
                    const int s0 = gi % C::QS;
                    if (is_a) {
                        // A: S^T, dV, dQ.  The item's first S^T overwrites the previous
                        // item's last once the P/dS warps have read it.
                        if (gi > 0 && !mbar_wait(&bars->s_free, (gi - 1) & 1)) break;
                        if (!mbar_wait(&bars->q_full[s0], (gi / C::QS) & 1)) break;
                        tc_fence_after();
                        mma_square(tmem + C::COL_S, k_kmaj, q_kmaj + stage_off(s0));
                        mma_commit(&bars->s_full);
                        for (int i = 0; i < n; ++i) {
                            const int g = gi + i;  // global iteration: stage and phases
                            const int s = g % C::QS;
                            const int s1 = (g + 1) % C::QS;
                            if (i + 1 < n) {
                                // S_{i+1} overwrites S_i as soon as the P/dS warps have read it.
                                if (!mbar_wait(&bars->s_free, g & 1) ||
                                    !mbar_wait(&bars->q_full[s1], ((g + 1) / C::QS) & 1)) { ok = false; break; }
                                tc_fence_after();
                                mma_square(tmem + C::COL_S, k_kmaj, q_kmaj + stage_off(s1));
                                mma_commit(&bars->s_full);
                            }
                            if (!mbar_wait(&bars->p_full, g & 1)) { ok = false; break; }
                            // dV starts from zero in this item: the previous item's epilogue
                            // must have read it out of TMEM.
                            if (i == 0 && tn > 0 && !mbar_wait(&bars->dkv_empty, (tn - 1) & 1)) { ok = false; break; }
                            tc_fence_after();
                            mma_tmem_a(tmem + C::COL_DV, tmem + C::COL_P, C::P_HALF_STRIDE,
                                       do_mn + stage_off(s), i > 0);
                            mma_commit(&bars->p_free);
                            mma_commit(&bars->stage_empty[s]);  // A's last reader of stage s
                            // dQ_i over dQ_{i-1}, which the drain has read
                            if (!mbar_wait(&bars->ds_full, g & 1) ||
                                (g > 0 && !mbar_wait(&bars->dq_empty, (g - 1) & 1))) { ok = false; break; }
                            tc_fence_after();
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk)
                                mma_ss(tmem + C::COL_DQ, ds_mn + (uint64_t)(kk * 2048 >> 4),
                                       k_mn + (uint64_t)(kk * 2048 >> 4), kIdescDq, kk > 0 ? 1u : 0u);
                            mma_commit(&bars->dq_full);
                            mma_commit(&bars->ds_empty);
                        }
                    } else {
                        // B: dP^T and dK.  The item's first dP^T follows the previous item's
                        // last dK in this thread's order (dK read the dS^T it overwrites).
                        if (!mbar_wait(&bars->do_full[s0], (gi / C::QS) & 1)) break;
                        tc_fence_after();
                        mma_square(tmem + C::COL_DP, v_kmaj, do_kmaj + stage_off(s0));
                        mma_commit(&bars->dp_full);
                        for (int i = 0; i < n; ++i) {
                            const int g = gi + i;
                            const int s = g % C::QS;
                            const int s1 = (g + 1) % C::QS;
                            if (!mbar_wait(&bars->ds_full, g & 1)) { ok = false; break; }
                            // dK starts from zero in this item: the previous item's epilogue
                            // must have read it out of TMEM.
                            if (i == 0 && tn > 0 && !mbar_wait(&bars->dkv_empty, (tn - 1) & 1)) { ok = false; break; }
                            tc_fence_after();
                            mma_tmem_a(tmem + C::COL_DK, tmem + C::COL_DP, C::DS_HALF_STRIDE,
                                       q_mn + stage_off(s), i > 0);
                            mma_commit(&bars->stage_empty[s]);  // B's last reader of stage s
                            if (i + 1 < n) {
                                // dP^T_{i+1} over dS^T_i, after dK_i in this thread's order
                                if (!mbar_wait(&bars->do_full[s1], ((g + 1) / C::QS) & 1)) { ok = false; break; }
                                tc_fence_after();
                                mma_square(tmem + C::COL_DP, v_kmaj, do_kmaj + stage_off(s1));
                                mma_commit(&bars->dp_full);
                            }
                        }
                    }
                    if (!ok) break;
                    mma_commit(&bars->dkv_full);
                    gi += n;
                    ++tn;
                }
            } else {
            for (int r = 0; ok && item_at(r, it); ++r) {
                const int n = it.n;
                if (n == 0) continue;
                if (!mbar_wait(&bars->kv_full, tn & 1)) break;
                tc_fence_after();
                // First S^T and dP^T of the item.  S^T overwrites the previous item's last
                // S^T once the P/dS warps have read it (d = 64); at d = 128 it overwrites the
                // previous P^T, which the (earlier issued) dV MMA has consumed.  dP^T at
                // d = 128 shares its columns with dQ: the previous dQ must be drained.
                {
                    const int s0 = gi % C::QS;
                    if (C::P_OWN && gi > 0 && !mbar_wait(&bars->s_free, (gi - 1) & 1)) break;
                    if (!mbar_wait(&bars->q_full[s0], (gi / C::QS) & 1)) break;
                    tc_fence_after();
                    mma_square(tmem + C::COL_S, k_kmaj, q_kmaj + stage_off(s0));
                    mma_commit(&bars->s_full);
                    if (D == 128 && gi > 0 && !mbar_wait(&bars->dq_empty, (gi - 1) & 1)) break;
                    if (!mbar_wait(&bars->do_full[s0], (gi / C::QS) & 1)) break;
                    tc_fence_after();
                    mma_square(tmem + C::COL_DP, v_kmaj, do_kmaj + stage_off(s0));
                    mma_commit(&bars->dp_full);
                }
                for (int i = 0; i < n; ++i) {
                    const int g = gi + i;  // global iteration: ring stage and barrier phases
                    const int s = g % C::QS;
                    const int s1 = (g + 1) % C::QS;
                    if (C::P_OWN && i + 1 < n) {
                        // S_{i+1} overwrites S_i as soon as every P/dS warp has read it.
                        if (!mbar_wait(&bars->s_free, g & 1) ||
                            !mbar_wait(&bars->q_full[s1], ((g + 1) / C::QS) & 1)) { ok = false; break; }
                        tc_fence_after();
                        mma_square(tmem + C::COL_S, k_kmaj, q_kmaj + stage_off(s1));
                        mma_commit(&bars->s_full);
                    }
                    if (!mbar_wait(&bars->p_full, g & 1)) { ok = false; break; }
                    // dV and dK start from zero in this item: the previous item's epilogue
                    // must have read them out of TMEM.
                    if (i == 0 && tn > 0 && !mbar_wait(&bars->dkv_empty, (tn - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    mma_tmem_a(tmem + C::COL_DV, tmem + C::COL_P, C::P_HALF_STRIDE,
                               do_mn + stage_off(s), i > 0);
                    mma_commit(&bars->p_free);
                    if (!C::P_OWN && i + 1 < n) {
                        // P^T_i lives in the S^T columns: S_{i+1} follows dV_i.
                        if (!mbar_wait(&bars->q_full[s1], ((g + 1) / C::QS) & 1)) { ok = false; break; }
                        tc_fence_after();
                        mma_square(tmem + C::COL_S, k_kmaj, q_kmaj + stage_off(s1));
                        mma_commit(&bars->s_full);
                    }
                    if (!mbar_wait(&bars->ds_full, g & 1)) { ok = false; break; }
                    tc_fence_after();
                    mma_tmem_a(tmem + C::COL_DK, tmem + C::COL_DP, C::DS_HALF_STRIDE,
                               q_mn + stage_off(s), i > 0);
                    if (D == 64 && g > 0) {
                        if (!mbar_wait(&bars->dq_empty, (g - 1) & 1)) { ok = false; break; }
                        tc_fence_after();
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + C::COL_DQ, ds_mn + (uint64_t)(kk * 2048 >> 4),
                               k_mn + (uint64_t)(kk * 2048 >> 4), kIdescDq, kk > 0 ? 1u : 0u);
                    mma_commit(&bars->dq_full);
                    mma_commit(&bars->ds_empty);
                    mma_commit(&bars->stage_empty[s]);
                    if (i + 1 < n) {
                        if (D == 128) {
                            // dQ_i lives in the dP^T columns: wait until it has been drained.
                            if (!mbar_wait(&bars->dq_empty, g & 1)) { ok = false; break; }
                        }
                        if (!mbar_wait(&bars->do_full[s1], ((g + 1) / C::QS) & 1)) { ok = false; break; }
                        tc_fence_after();
                        mma_square(tmem + C::COL_DP, v_kmaj, do_kmaj + stage_off(s1));
                        mma_commit(&bars->dp_full);
                    }
                }
                mma_commit(&bars->dkv_full);
                gi += n;
                ++tn;
            }
            }
        }
    } else if (warp >= C::W_DQ0) {
        // ------------------------------ dQ drain ----------------------------------
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;          // query row in the tile = TMEM lane
        const int gt = threadIdx.x - C::W_DQ0 * 32;  // 0..127 inside this warpgroup
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool ok = true;
        int gi = 0, tn = 0;  // global iteration, items with work so far
        Item it;
        for (int rr = 0; ok && item_at(rr, it); ++rr) {
        const int bh = it.bh;
        for (int i = 0, qi = it.q_first; i < it.n; ++i, qi = next_q(it, qi + 1)) {
            // The 128 drain threads agree on the wait's outcome before the warp-wide TMEM
            // loads and the named barriers below, so a timeout makes all of them leave.
            if (!named_bar_and(2, 128, mbar_wait(&bars->dq_full, (gi + i) & 1))) { ok = false; break; }
            tc_fence_after();
            // Boxes of [128 rows][32 fp32], 16-byte chunks swizzled by row % 8, staged
            // ROUND_BOXES at a time (all D/32 at d = 64; two per round in the dS buffer at
            // d = 128), each round handed to a TMA reduce-add into the fp32 accumulator.
            constexpr int ROUND_BOXES = C::DQ_IN_DS ? 2 : D / 32;
            uint8_t *stage = C::DQ_IN_DS ? sdS : sDQ;
#pragma unroll
            for (int b0 = 0; b0 < D / 32; b0 += ROUND_BOXES) {
                if (gt == 0) bulk_wait_group_read<0>();  // the previous reduce has read it
                named_bar_sync(2, 128);
#pragma unroll
                for (int bx = 0; bx < ROUND_BOXES; ++bx) {
                    uint32_t w[32];
                    tmem_ld32(tmem + lane_base + C::COL_DQ + (b0 + bx) * 32, w);
                    uint8_t *rowp = stage + bx * 16384 + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        *reinterpret_cast<uint4 *>(rowp + ((c ^ (r & 7)) << 4)) =
                            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                }
                if (b0 + ROUND_BOXES == D / 32) {  // every dQ column is out of TMEM
                    tc_fence_before();
                    mbar_arrive(&bars->dq_empty);
                }
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (gt == 0) {
#pragma unroll
                    for (int bx = 0; bx < ROUND_BOXES; ++bx)
                        tma_reduce_add_3d(&tmdQacc, stage + bx * 16384, (b0 + bx) * 32, qi * 128, bh);
                    bulk_commit_group();
                }
            }
            if (C::DQ_IN_DS && gt == 0) {
                bulk_wait_group_read<0>();  // the dS buffer may take dS_{i+1}
                mbar_arrive(&bars->dq_stage_free);
            }
        }
        if constexpr (C::DRAIN_EPI) {
            // ------------------------- epilogue of the item: dK, dV ----------------------
            // Every MMA of the item is done (dkv_full); the staging area is free once the
            // item's last dQ reduce-add has read it.  Row r of both 16-bit tiles, 128-byte
            // blocks with 16-byte chunks swizzled by r % 8 (the store maps' layout).
            if (ok) {
                const int n = it.n, kt = it.kt;
                Item nxt;
                if (!item_at(rr + 1, nxt)) pdl_launch_dependents();  // this CTA's last item
                const bool w_ok = n == 0 || mbar_wait(&bars->dkv_full, tn & 1);
                if (gt == 0) bulk_wait_group_read<0>();
                if (!named_bar_and(2, 128, w_ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int which = 0; which < 2; ++which) {
                    const uint32_t col = which == 0 ? C::COL_DV : C::COL_DK;
                    float mul = which == 0 ? 1.f : p.scale;
                    if constexpr (DROP) mul = which == 0 ? p.dv_mul : p.dk_mul;
                    uint8_t *rowp = sDQ + which * C::HALF + r * 128;
#pragma unroll
                    for (int c32 = 0; c32 < D / 32; ++c32) {
                        uint32_t w[32];
                        if (n > 0) {
                            tmem_ld32(tmem + lane_base + col + c32 * 32, w);
                        } else {
#pragma unroll
                            for (int k = 0; k < 32; ++k) w[k] = 0u;
                        }
                        uint32_t wv[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            wv[k] = pack2<BF16>(__uint_as_float(w[2 * k]) * mul,
                                                __uint_as_float(w[2 * k + 1]) * mul);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            *reinterpret_cast<uint4 *>(rowp + (((c32 * 4 + c) ^ (r & 7)) << 4)) =
                                make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                    }
                }
                if (n > 0) {
                    // dK, dV are out of TMEM: the next item's first dV / dK MMA may start
                    tc_fence_before();
                    mbar_arrive(&bars->dkv_empty);
                }
                fence_proxy_async_smem();
                named_bar_sync(2, 128);
                if (gt == 0) {
                    tma_store_3d(&tmdV, sDQ, 0, kt * 128, bh);
                    tma_store_3d(&tmdK, sDQ + C::HALF, 0, kt * 128, bh);
                    bulk_commit_group();
                }
            }
            if (it.n > 0) ++tn;
        }
        gi += it.n;
        }
        if (gt == 0) bulk_wait_group<0>();
    } else {
        // ------------------------------ P / dS warps ------------------------------
        const int quarter = warp & 3;
        const int h = warp >> 2;             // query half: columns 64h .. 64h + 63
        const int t = quarter * 32 + lane;   // key row in the tile = TMEM lane
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        const float sl2 = p.scale_log2;
        bool ok = true;
        bool store_pending = false;  // the last item's dK/dV stores may still read the dS buffer
        int gi = 0, tn = 0;  // global iteration, items with work so far
        Item it;
        for (int rr = 0; item_at(rr, it); ++rr) {
        const int kt = it.kt, bh = it.bh, L = it.L, n = it.n;
        const bool key_ok = kt * 128 + t < L;
        for (int i = 0, qi = it.q_first; ok && i < n; ++i, qi = next_q(it, qi + 1)) {
            const int g = gi + i;  // global iteration: ring stage and barrier phases
            const int s = g % C::QS;
            // Dropout keep bits of this key row against queries 64h .. 64h + 63 of tile qi:
            // bit m of kb[u] = query 32u + 2m, bit m + 16 = query 32u + 2m + 1.  Each lane
            // of a half-warp draws the Philox blocks of two queries for the half-warp's
            // 16-key group; a bit transpose hands every lane its own key's bits.
            uint32_t kb[2] = {0u, 0u};
            if constexpr (DROP) {
                const uint32_t grp = (uint32_t)(kt * 128 + quarter * 32 + (lane & 16)) >> 4;
                const uint32_t q0 = (uint32_t)(qi * 128 + h * 64 + 2 * (lane & 15));
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t a = keep_bits16(
                        philox4x32_10(grp, q0 + 32 * u, (uint32_t)bh, p.drop.offset, p.drop.seed_lo,
                                      p.drop.seed_hi), p.drop.add16);
                    const uint32_t c = keep_bits16(
                        philox4x32_10(grp, q0 + 32 * u + 1, (uint32_t)bh, p.drop.offset,
                                      p.drop.seed_lo, p.drop.seed_hi), p.drop.add16);
                    kb[u] = transpose16x16_halfwarp(a | (c << 16), lane);
                }
            }
            // (waits are voted on per warp: the loop body has warp-wide TMEM loads and stores)
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full, g & 1) &&
                                             mbar_wait(&bars->q_full[s], (g / C::QS) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            // P^T for queries 64h .. 64h + 63 of this key row, packed in 16-bit pairs
            // (exactly what the dV MMA consumes; dS below uses the same rounded values).
            uint32_t Pw[32];
            {
                const float *nl2 = sLSE + s * 128 + h * 64;  // -LSE2 of the 64 queries
                // Masks only on the causal diagonal tile and the key-padding tail tile.
                const bool diag = p.causal && (qi == kt);
                const bool tile_masked = diag || (kt * 128 + 128 > L);
                // P^T for queries 64h + k0 .. + 31 from the S^T values w
                auto p_half = [&](const uint32_t (&w)[32], int k0) {
                    if (!tile_masked) {
#pragma unroll
                        for (int k = 0; k < 32; k += 4) {
                            const float4 l4 = *reinterpret_cast<const float4 *>(nl2 + k0 + k);
                            const float p0 = ex2(fmaf(__uint_as_float(w[k]), sl2, l4.x));
                            const float p1 = ex2(fmaf(__uint_as_float(w[k + 1]), sl2, l4.y));
                            const float p2 = ex2(fmaf(__uint_as_float(w[k + 2]), sl2, l4.z));
                            const float p3 = ex2(fmaf(__uint_as_float(w[k + 3]), sl2, l4.w));
                            Pw[(k0 + k) >> 1] = pack2<BF16>(p0, p1);
                            Pw[((k0 + k) >> 1) + 1] = pack2<BF16>(p2, p3);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; k += 4) {
                            const int c = h * 64 + k0 + k;  // query column in the tile
                            const float4 l4 = *reinterpret_cast<const float4 *>(nl2 + k0 + k);
                            float p0 = ex2(fmaf(__uint_as_float(w[k]), sl2, l4.x));
                            float p1 = ex2(fmaf(__uint_as_float(w[k + 1]), sl2, l4.y));
                            float p2 = ex2(fmaf(__uint_as_float(w[k + 2]), sl2, l4.z));
                            float p3 = ex2(fmaf(__uint_as_float(w[k + 3]), sl2, l4.w));
                            // keys past the valid length, and queries before the key (causal)
                            if (!key_ok || (diag && c < t)) p0 = 0.f;
                            if (!key_ok || (diag && c + 1 < t)) p1 = 0.f;
                            if (!key_ok || (diag && c + 2 < t)) p2 = 0.f;
                            if (!key_ok || (diag && c + 3 < t)) p3 = 0.f;
                            Pw[(k0 + k) >> 1] = pack2<BF16>(p0, p1);
                            Pw[((k0 + k) >> 1) + 1] = pack2<BF16>(p2, p3);
                        }
                    }
                };
                // The second half of the S^T row loads while the first is exponentiated.
                uint32_t wa[32], wb[32];
                tmem_ld32(tmem + lane_base + C::COL_S + h * 64, wa);
                tmem_ld32_async(tmem + lane_base + C::COL_S + h * 64 + 32, wb);
                p_half(wa, 0);
                tmem_wait_ld(wb);
                if (C::P_OWN) {
                    tc_fence_before();
                    mbar_arrive(&bars->s_free);  // S^T may now be overwritten by S_{i+1}
                }
                p_half(wb, 32);
            }
            if (C::P_OWN && g > 0 &&  // dV_{g-1} has read P
                !__all_sync(0xffffffffu, mbar_wait(&bars->p_free, (g - 1) & 1))) {
                ok = false;
                break;
            }
            if constexpr (DROP) {
                // the dV operand is P o K; Pw (unmasked) stays for dS
                uint32_t Pm[32];
#pragma unroll
                for (int pi = 0; pi < 32; ++pi) {
                    const uint32_t x = kb[pi >> 4] << (15 - (pi & 15));
                    Pm[pi] = Pw[pi] & prmt(x, 0u, 0xBB99u);
                }
                tmem_st32(tmem + lane_base + C::COL_P + h * C::P_HALF_STRIDE, Pm);
            } else {
                tmem_st32(tmem + lane_base + C::COL_P + h * C::P_HALF_STRIDE, Pw);
            }
            tc_fence_before();
            mbar_arrive(&bars->p_full);

            if (!__all_sync(0xffffffffu,
                            mbar_wait(&bars->dp_full, g & 1) &&
                                mbar_wait(&bars->do_full[s], (g / C::QS) & 1) &&
                                (g == 0 || mbar_wait(&bars->ds_empty, (g - 1) & 1)) &&
                                // d = 128: the dQ drain has staged dQ_{g-1} through the dS
                                // buffer and let go
                                (!C::DQ_IN_DS || g == 0 ||
                                 mbar_wait(&bars->dq_stage_free, (g - 1) & 1)))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (store_pending) {
                // the previous item's dK/dV stores have read the dS buffer (this wait
                // overlapped P_0) before dS_0 goes there
                if (threadIdx.x == 0) bulk_wait_group_read<0>();
                named_bar_sync(1, 256);
                store_pending = false;
            }
            const float *ndv = sDv + s * 128 + h * 64;  // -D of the 64 queries
            // dS for queries 64h + 32cc .. + 31 from the dP^T values w
            auto ds_half = [&](const uint32_t (&w)[32], int cc) {
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float2 nd2 = *reinterpret_cast<const float2 *>(ndv + cc * 32 + k);
                    float dp0 = __uint_as_float(w[k]);
                    float dp1 = __uint_as_float(w[k + 1]);
                    if constexpr (DROP) {
                        if (!((kb[cc] >> (k >> 1)) & 1u)) dp0 = 0.f;
                        if (!((kb[cc] >> ((k >> 1) + 16)) & 1u)) dp1 = 0.f;
                    }
                    // dS = P o (dP - D): the difference in fp32, rounded to 16 bits, times
                    // the 16-bit P pair in one packed multiply
                    pk[k >> 1] = mul2<BF16>(Pw[cc * 16 + (k >> 1)],
                                            pack2<BF16>(dp0 + nd2.x, dp1 + nd2.y));
                }
                // dS^T pairs -> TMEM, over dP^T columns this warp has just read; A operand
                // of dK += dS^T Q.
                tmem_st16(tmem + lane_base + C::COL_DP + h * C::DS_HALF_STRIDE + cc * 16, pk);
                // dS -> shared memory as the MN-major A operand of dQ = dS K:
                // [query block h (64 queries)][key row t][128 bytes], 128-byte swizzle.
                uint8_t *rowp = sdS + h * 16384 + t * 128;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int chunk = cc * 4 + q4;
                    *reinterpret_cast<uint4 *>(rowp + ((chunk ^ (t & 7)) << 4)) =
                        make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
                }
            };
            // the second half of the dP^T row loads while the first is turned into dS
            uint32_t da[32], db[32];
            tmem_ld32(tmem + lane_base + C::COL_DP + h * 64, da);
            tmem_ld32_async(tmem + lane_base + C::COL_DP + h * 64 + 32, db);
            ds_half(da, 0);
            tmem_wait_ld(db);
            ds_half(db, 1);
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars->ds_full);
        }

        if constexpr (!C::DRAIN_EPI) {
        // ------------------------------ epilogue of the item: dK, dV ---------------------
        // All 256 threads agree on whether to go on (a bounded wait may have failed).
        ok = named_bar_and(1, 256, ok);
        Item nxt;
        if (!item_at(rr + 1, nxt)) pdl_launch_dependents();  // this CTA's last item
        if (ok && n > 0) {
            ok = mbar_wait(&bars->dkv_full, tn & 1) &&
                 // d = 128: the dQ drain of the item's last iteration is done with the dS buffer
                 (!C::DQ_IN_DS || mbar_wait(&bars->dq_stage_free, (gi + n - 1) & 1));
            tc_fence_after();
        }
        // An item without work has written no dS: the previous stores' reads of the dS
        // buffer are waited for here, before the staging below (the barrier orders it).
        if (store_pending && threadIdx.x == 0) bulk_wait_group_read<0>();
        store_pending = false;
        // Agree again, so that the `break` after the epilogue is taken by all 256 threads
        // or by none (the next item's epilogue barriers need every one of them).
        ok = named_bar_and(1, 256, ok);
        // Staging in the dS buffer (free: every MMA of the item is done; 32 KB): both
        // 16-bit tiles at d = 64, one tile per round at d = 128.  Each warp converts its
        // lane quarter's D/2 columns.
        constexpr int HCOLS = D / 2;  // columns of this warp's half
        constexpr int ROUNDS = (D == 64) ? 1 : 2;
#pragma unroll
        for (int round = 0; round < ROUNDS; ++round) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                if (ROUNDS == 2 && which != round) continue;
                const uint32_t col = (which == 0 ? C::COL_DV : C::COL_DK) + h * HCOLS;
                float mul = which == 0 ? 1.f : p.scale;
                if constexpr (DROP) mul = which == 0 ? p.dv_mul : p.dk_mul;
                uint8_t *stage = sdS + (ROUNDS == 1 ? which * C::HALF : 0);
#pragma unroll
                for (int c32 = 0; c32 < HCOLS / 32; ++c32) {
                    uint32_t w[32];
                    if (n > 0) {
                        tmem_ld32(tmem + lane_base + col + c32 * 32, w);
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) w[k] = 0u;
                    }
                    uint32_t wv[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        wv[k] = pack2<BF16>(__uint_as_float(w[2 * k]) * mul,
                                            __uint_as_float(w[2 * k + 1]) * mul);
                    // element e = h * HCOLS + c32 * 32 .. + 31 of row t: 128-byte block e / 64,
                    // 16-byte chunks (e % 64) / 8 .. + 3
                    const int e0 = h * HCOLS + c32 * 32;
                    uint8_t *rowp = stage + (e0 >> 6) * C::HALF + t * 128;
                    const int ch0 = (e0 & 63) >> 3;
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<uint4 *>(rowp + (((ch0 + c) ^ (t & 7)) << 4)) =
                            make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
                }
            }
            if (round == ROUNDS - 1 && n > 0) {
                // dK, dV are out of TMEM: the next item's first dV / dK MMA may start
                tc_fence_before();
                mbar_arrive(&bars->dkv_empty);
            }
            fence_proxy_async_smem();
            named_bar_sync(1, 256);
            if (threadIdx.x == 0) {
                for (int which = 0; which < 2; ++which) {
                    if (ROUNDS == 2 && which != round) continue;
                    const uint8_t *stage = sdS + (ROUNDS == 1 ? which * C::HALF : 0);
                    for (int hf = 0; hf < C::HALVES; ++hf)
                        tma_store_3d(which == 0 ? &tmdV : &tmdK, stage + hf * C::HALF, hf * 64,
                                     kt * 128, bh);
                }
                bulk_commit_group();
                // The next round reuses the dS buffer right away; after the last round the
                // next item writes it only for its first dS, which waits then (store_pending).
                if (round < ROUNDS - 1) bulk_wait_group_read<0>();
            }
            if (round < ROUNDS - 1) named_bar_sync(1, 256);
        }
        store_pending = true;
        }
        gi += n;
        if (n > 0) ++tn;
        if (!ok) break;
        }  // items
        if (threadIdx.x == 0) bulk_wait_group<0>();  // shared memory must outlive the stores
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::W_MMA) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fa
