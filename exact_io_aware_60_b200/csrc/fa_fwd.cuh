// fa_fwd.cuh -- forward pass of exact tiled attention on sm_100a.
//
// The method (anthology note "NOTE-005: FlashAttention", section "Method"; aicassindra
// FlashAttention architecture page, "End-to-end flow"): split Q into row blocks and
// K, V into key blocks, bring one block at a time on chip, form that block of scores
// there, and fold it into the output with an online softmax that carries a running row
// maximum m and normaliser l, rescaling the accumulated output whenever m grows.  Only
// O and the row statistics leave the chip; the N x N score matrix never exists in HBM.
//
// B200 mapping: persistent CTAs (two per SM at d = 64), each walking a static list of
// work items = 128-row query tiles of one (batch, head) (and one key range in split-KV
// mode).  Per CTA:
//   warp 4      TMA producer: Q of an item (two buffers at d = 64, so the next item's Q
//               is loaded while this one runs; one at d = 128, loaded once the previous
//               item's last S MMA is done), then K_j / V_j into an NS-stage shared-memory
//               ring (128-byte swizzle, mbarrier transaction counts) that runs on across
//               items.
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into TMEM, then O += P_j V_j with
//               P_j read straight from TMEM.
//   warps 0..3  softmax, one query row per thread (TMEM lane = row): load S_j, mask on
//               diagonal / tail blocks only, row max, p = 2^(s*scale*log2e - m) with the
//               MUFU ex2, row sum, P_j written back into TMEM as 16-bit pairs.
//               The output rescale is lazy: m only moves when the row max grows by more
//               than 2^8, which leaves the result exact because O and l always share the
//               same m.  Epilogue: O / l' -> 16-bit, written from registers row by row
//               (no staging, so the next item's Q can load early); LSE = ln2 * (m + log2 l).
//   Normaliser: the tensor core multiplies V by P rounded to 16 bits, so the output is
//   divided by l' = sum of exactly those rounded values, produced by the same PV MMA
//   (its B operand carries 16 extra columns of ones after V) in 16 extra TMEM columns.
//   The weights applied to the rows of V then sum to one exactly, which removes the bias
//   a fp32 l would leave when one key dominates a row.  LSE keeps the fp32 sum l of the
//   unrounded values.
//
// Two shapes of the same kernel:
//   d = 64  : 64-key blocks; TMEM holds S (64 columns), P (32), O and the sums (80): 176
//             of 256 columns, so two CTAs share an SM.  P has its own columns, so S_{j+1}
//             is computed as soon as the softmax has read S_j, while it works on P_j.
//   d = 128 : 128-key blocks; the CTA owns the SM's 512 columns: two score buffers (P_j is
//             written over S_j), so S_{j+1} is computed while softmax works on S_j.
// A tcgen05.mma instruction costs at least ~45 cycles whatever its N, so small MMAs are
// merged where possible (the row sums ride on the PV instruction).
//
// Block-sparse attention (promptingindex page, "Benchmark results"; NOTE-005, "Key
// components"): with a block mask, every role walks only the key blocks whose 128 x 128
// (query tile, key tile) entry is set; skipped blocks cost nothing.
//
// The loop order is query-block outer (each CTA writes its O rows once) instead of the
// key-block-outer order of the original algorithm; the result is the same up to
// floating-point ordering.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "dropout.cuh"
#include "sm100.cuh"

namespace fa {

struct FwdParams {
    void *o;  // [BH][N][D] 16-bit output (written from registers)
    float *lse;
    const int *kv_len;
    // Split-KV partial outputs (SPLIT only): the normalised O and the LSE of each split's
    // key range, fp32 [num_splits][BH][N][D] and [num_splits][BH][N].
    float *part_o;
    float *part_lse;
    int num_splits;          // 1 without splitting
    int kv_blocks_per_split; // key blocks per split (0: all)
    // Block-sparse attention: uint8 [heads][T128][T128] (T128 = ceil(N / 128)); a query
    // tile visits only key tiles whose byte is nonzero.  nullptr = dense.
    const uint8_t *bmask;
    long long bmask_bh_stride;  // 0: one mask for every (batch, head)
    int bmask_T;
    int N;           // query rows
    int Nk;          // key rows (= N except for the rectangular inference shape)
    int causal_off;  // Nk - N: query i sees keys j <= i + causal_off under causal masking
    int BH;
    int H;
    int num_q_tiles;
    float scale_log2;  // scale * log2(e)
    int causal;
    DropoutParams drop;  // used by the dropout variant only
    float out_scale;     // E4M3 variant: V's scale factor, applied to the output
};

template <int D>
struct FwdCfg {
    static constexpr int BM = 128;                      // query rows per tile
    static constexpr int BN = (D == 64) ? 64 : 128;     // keys per block
    static constexpr int HALVES = D / 64;               // 128-byte column blocks per row
    static constexpr int QTILE = BM * D * 2;            // bytes of the Q tile
    static constexpr int QHALF = BM * 128;              // one column block of Q
    static constexpr int KTILE = BN * D * 2;            // bytes of one K or V block
    static constexpr int KHALF = BN * 128;              // one column block of K or V
    static constexpr bool P_OWN = (D == 64);            // P in its own TMEM columns
    static constexpr int SBUF = (D == 64) ? 1 : 2;      // score buffers in TMEM
    static constexpr int CTAS_PER_SM = (D == 64) ? 2 : 1;
    // d = 64: two Q buffers and a 3-deep K/V ring fit two CTAs in an SM's shared memory
    static constexpr int QBUF = (D == 64) ? 2 : 1;      // Q buffers (items in flight)
    static constexpr int NS = (D == 64) ? 3 : 2;        // K/V ring depth
    // Each V stage is followed by a block of 16-bit ones, one 64-column block past the
    // tile: the PV MMA reads it as B columns D..D+15 and so also produces the row sums
    // of P (one N = D + 16 instruction instead of a second, equally costly N = 16 one).
    static constexpr int VSTAGE = (HALVES + 1) * KHALF;  // V block + its ones block
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QBUF * QTILE;
    static constexpr int OFF_V = OFF_K + NS * KTILE;
    static constexpr int OFF_BAR = OFF_V + NS * VSTAGE;
    static constexpr int USED = OFF_BAR + 512;  // barriers and the item cache
    // Two CTAs per SM leave no room for an alignment pad at d = 64: the kernel checks
    // that the dynamic shared-memory base is 1024-byte aligned instead.
    static constexpr int SLACK = (CTAS_PER_SM == 1) ? 1024 : 0;
    static constexpr int SMEM = USED + SLACK;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = (CTAS_PER_SM == 2) ? 256 : 512;
    static constexpr uint32_t COL_P = SBUF * BN;        // d = 64 only: 32 columns
    static constexpr uint32_t COL_O = P_OWN ? COL_P + BN / 2 : SBUF * BN;
    static constexpr uint32_t COL_SUM = COL_O + D;      // 16 columns: row sums of 16-bit P
    static constexpr int PV_N = D + 16;                 // O and the row sums in one MMA
    static constexpr int KS_S = D / 16;                 // MMA K steps of S (32 bytes each)
    static constexpr int KS_PV = BN / 16;               // MMA K steps of P V
    static constexpr int PV_STEP = 16 * 128;            // bytes of V rows per P V step
    static_assert(COL_SUM + 16 <= TMEM_COLS, "TMEM budget");
    // (an SM has 228 KB of shared memory and reserves 1 KB per resident CTA)
    static_assert(CTAS_PER_SM * (SMEM + 1024) <= 233472, "shared memory budget");
};

// E4M3 inputs, d = 128: a row of Q, K or V is one 128-byte swizzle block, an MMA step
// takes K = 32 one-byte elements, and P goes to TMEM as four E4M3 values per column.
struct FwdCfgF8 {
    static constexpr int D = 128;
    static constexpr int BM = 128;
    static constexpr int BN = 128;
    static constexpr int HALVES = 1;                    // 128-byte column blocks per row
    static constexpr int QTILE = BM * 128;
    static constexpr int QHALF = BM * 128;
    static constexpr int KTILE = BN * 128;
    static constexpr int KHALF = BN * 128;
    static constexpr bool P_OWN = false;
    static constexpr int SBUF = 2;
    static constexpr int CTAS_PER_SM = 1;
    static constexpr int QBUF = 1;
    static constexpr int NS = 4;
    static constexpr int VSTAGE = 2 * KHALF;            // V block + its block of E4M3 ones
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QTILE;
    static constexpr int OFF_V = OFF_K + NS * KTILE;
    static constexpr int OFF_BAR = OFF_V + NS * VSTAGE;
    static constexpr int USED = OFF_BAR + 512;  // barriers and the item cache
    static constexpr int SLACK = 1024;
    static constexpr int SMEM = USED + SLACK;
    static constexpr int THREADS = 192;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int PBUF = 1;
    static constexpr uint32_t COL_P = SBUF * BN;
    static constexpr uint32_t COL_O = SBUF * BN;
    static constexpr uint32_t COL_SUM = COL_O + D;
    static constexpr int PV_N = D + 16;
    static constexpr int KS_S = D / 32;
    static constexpr int KS_PV = BN / 32;
    static constexpr int PV_STEP = 32 * 128;
    static_assert(COL_SUM + 16 <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct FwdBars {
    uint64_t q_full[2];
    uint64_t q_empty[2];  // every S MMA of the item in this Q buffer is done: it may be reloaded
    uint64_t o_empty;  // the epilogue has read O: the next item's first P V may start
    uint64_t s_full[2];
    uint64_t s_read;
    uint64_t p_full[2];
    uint64_t o_full;
    uint64_t k_full[4];
    uint64_t v_full[4];
    uint64_t kv_empty[4];
    uint32_t tmem_base;
    ItemCache items;  // SCHED: this CTA's list of the launcher's schedule
};

// DROP: dropout on the probabilities (the mask is regenerated per element from the
// counter-based generator; the normaliser is the fp32 sum of the undropped values).
// SPLIT: the CTA covers one range of key blocks and writes an fp32 partial output (O
// normalised by that range's own l) and the range's LSE; a combine kernel merges them.
// F8: E4M3 Q, K, V (d = 128), kind::f8f6f4 MMAs, P rounded to E4M3 for the P V product,
// bf16 output (BF16 = true).
// SCHED: the launcher passes a static schedule of the items (ItemSchedule).
template <int D, bool BF16, bool DROP, bool SPLIT, bool F8 = false, bool SCHED = false>
__global__ void __launch_bounds__(192, FwdCfg<D>::CTAS_PER_SM)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const FwdParams p,
              const __grid_constant__ std::conditional_t<SCHED, ItemSchedule, NoSchedule> sched) {
    static_assert(!F8 || (D == 128 && BF16 && !DROP && !SPLIT), "E4M3 variant: d = 128 only");
    using C = std::conditional_t<F8, FwdCfgF8, FwdCfg<D>>;
    constexpr int BN = C::BN;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    if (pad > (uint32_t)C::SLACK) {  // cannot happen with a 1024-aligned dynamic base
        if (threadIdx.x == 0) atomicExch(&g_status, 5);
        return;
    }
    uint8_t *smem = smem_raw + pad;
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    FwdBars *bars = reinterpret_cast<FwdBars *>(smem + C::OFF_BAR);
    static_assert(sizeof(FwdBars) <= 512, "barrier area");

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 128) {
        if constexpr (SCHED) item_cache_fill(bars->items, sched);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->q_full[i], 1);
            mbar_init(&bars->q_empty[i], 1);
        }
        mbar_init(&bars->o_empty, 128);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 128);
        }
        mbar_init(&bars->s_read, 128);
        mbar_init(&bars->o_full, 1);
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&bars->k_full[i], 1);
            mbar_init(&bars->v_full[i], 1);
            mbar_init(&bars->kv_empty[i], 1);
        }
        fence_mbar_init();
    }
    if (warp == 4) {
        // 16-bit (or E4M3) ones after every V stage (layout-agnostic: every element is 1)
        const uint32_t one2 = F8 ? 0x38383838u : (BF16 ? 0x3F803F80u : 0x3C003C00u);
        for (int st = 0; st < C::NS; ++st) {
            uint4 *ones = reinterpret_cast<uint4 *>(sV + st * C::VSTAGE + C::HALVES * C::KHALF);
            for (int i = lane; i < C::KHALF / 16; i += 32) ones[i] = make_uint4(one2, one2, one2, one2);
        }
        fence_proxy_async_smem();
    }
    if (warp == 5) tmem_alloc(&bars->tmem_base, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars->tmem_base;
    pdl_wait();  // inputs written by the previous kernel are visible from here on

    // Persistent CTA: work items are (query tile, key split, head), numbered so that the
    // heaviest causal tiles come first.  With a schedule from the launcher (dense and
    // causal shapes of up to kSchedMaxItems items), CTA c walks its list of items;
    // otherwise round r of CTA c takes item r * G + c on even rounds and r * G + (G - 1 - c)
    // on odd ones (G = grid size).  Every role walks the same list; key lengths and block
    // masks are read only after the wait above.
    struct Item {
        int qt, split, bh, L;
        int T;            // end of this item's key-block range
        int j_first;      // first visited key block (T if none)
        const uint8_t *mrow;
    };
    // Block-sparse walk: next key block at or after j whose tile is set (T if none).
    auto next_block = [&](const Item &it, int j) -> int {
        if (it.mrow)
            while (j < it.T && it.mrow[(j * BN) >> 7] == 0) ++j;
        return j;
    };
    auto item_at = [&](int r, Item &it) -> bool {
        int u;
        if constexpr (SCHED) {  // the launcher's balanced assignment
            if (!item_cache_get(bars->items, sched, r, u)) return false;
        } else {
            const int G = (int)gridDim.x;
            u = r * G + ((r & 1) ? (G - 1 - (int)blockIdx.x) : (int)blockIdx.x);
        }
        if (u >= p.num_q_tiles * p.num_splits * p.BH) return false;
        it.bh = u % p.BH;
        const int rest = u / p.BH;
        it.split = rest % p.num_splits;
        const int tile_rank = rest / p.num_splits;
        it.qt = p.causal ? (p.num_q_tiles - 1 - tile_rank) : tile_rank;
        int L = p.Nk;
        if (p.kv_len != nullptr) {
            L = p.kv_len[it.bh / p.H];
            L = L < 0 ? 0 : (L > p.Nk ? p.Nk : L);
        }
        it.L = L;
        int kv_end = L;
        if (p.causal) kv_end = min(kv_end, (it.qt + 1) * C::BM + p.causal_off);
        it.T = kv_end > 0 ? (kv_end + BN - 1) / BN : 0;
        int j_lo = 0;
        if (p.kv_blocks_per_split > 0) {  // this split's blocks: [j_lo, T)
            j_lo = it.split * p.kv_blocks_per_split;
            it.T = min(it.T, j_lo + p.kv_blocks_per_split);
        }
        it.mrow = p.bmask ? p.bmask + (size_t)it.bh * p.bmask_bh_stride + (size_t)it.qt * p.bmask_T
                          : nullptr;
        it.j_first = next_block(it, j_lo);
        return true;
    };

    if (warp == 4) {
        // ------------------------------ TMA producer ------------------------------
        // Q of an item as soon as the previous item's last S MMA is done; K_j / V_j into
        // the ring, whose stages and phases run on the global block count gj.
        if (lane == 0) {
            bool ok = true;
            int gj = 0, t = 0;  // global block count, items with blocks
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.j_first >= it.T) continue;
                // Q buffer qb: the item QBUF back has issued its last S MMA
                const int qb = t % C::QBUF;
                if (t >= C::QBUF && !mbar_wait(&bars->q_empty[qb], ((t / C::QBUF) - 1) & 1)) break;
                mbar_arrive_expect_tx(&bars->q_full[qb], C::QTILE);
                for (int hf = 0; hf < C::HALVES; ++hf)
                    tma_load_3d(sQ + qb * C::QTILE + hf * C::QHALF, &tmQ, &bars->q_full[qb], hf * 64,
                                it.qt * C::BM, it.bh);
                for (int j = it.j_first; j < it.T; j = next_block(it, j + 1), ++gj) {
                    const int s = gj % C::NS;
                    if (gj >= C::NS && !mbar_wait(&bars->kv_empty[s], ((gj / C::NS) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->k_full[s], C::KTILE);
                    for (int hf = 0; hf < C::HALVES; ++hf)
                        tma_load_3d(sK + s * C::KTILE + hf * C::KHALF, &tmK, &bars->k_full[s],
                                    hf * 64, j * BN, it.bh);
                    mbar_arrive_expect_tx(&bars->v_full[s], C::KTILE);
                    for (int hf = 0; hf < C::HALVES; ++hf)
                        tma_load_3d(sV + s * C::VSTAGE + hf * C::KHALF, &tmV, &bars->v_full[s],
                                    hf * 64, j * BN, it.bh);
                }
                ++t;
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0) {
            constexpr uint32_t kIdescS =
                F8 ? idesc_e4m3(false, false, 128, BN) : idesc_f16(BF16, false, false, 128, BN);
            constexpr uint32_t kIdescO = F8 ? idesc_e4m3(false, true, 128, C::PV_N)
                                            : idesc_f16(BF16, false, true, 128, C::PV_N);
            // Descriptors are built once; per k-step and per stage only the 16-byte start
            // address field changes, by compile-time offsets.
            const uint64_t q_desc0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            uint64_t q_desc = q_desc0;  // the current item's Q buffer
            const uint64_t k_desc = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(smem_u32(sV), C::KHALF, 1024);
            // g: global block index (stages, phases and score buffers follow it)
            auto issue_s = [&](int g) -> bool {
                const int s = g % C::NS;
                if (!mbar_wait(&bars->k_full[s], (g / C::NS) & 1)) return false;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((g % C::SBUF) * BN);
                const uint64_t kd = k_desc + (uint64_t)((s * C::KTILE) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::KS_S; ++kk) {
                    const uint64_t qo = (uint64_t)(((kk >> 2) * C::QHALF + (kk & 3) * 32) >> 4);
                    const uint64_t ko = (uint64_t)(((kk >> 2) * C::KHALF + (kk & 3) * 32) >> 4);
                    if constexpr (F8) mma_ss_f8(d_tmem, q_desc + qo, kd + ko, kIdescS, kk > 0 ? 1u : 0u);
                    else mma_ss(d_tmem, q_desc + qo, kd + ko, kIdescS, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[g % C::SBUF]);
                return true;
            };
            bool ok = true;
            int gj = 0, t = 0;
            Item it;
            for (int r = 0; ok && item_at(r, it); ++r) {
                if (it.j_first >= it.T) continue;
                const int qb = t % C::QBUF;
                if (!mbar_wait(&bars->q_full[qb], (t / C::QBUF) & 1)) break;
                tc_fence_after();
                q_desc = q_desc0 + (uint64_t)((qb * C::QTILE) >> 4);
                // The item's first S overwrites the previous block's S once the softmax has
                // read it (d = 64); at d = 128 its buffer held P_{g-2}, consumed by an
                // earlier P V.
                if (C::P_OWN && gj > 0 && !mbar_wait(&bars->s_read, (gj - 1) & 1)) break;
                if (!issue_s(gj)) break;
                int jj = 0;
                for (int j = it.j_first; j < it.T; ++jj) {
                    const int g = gj + jj;
                    const int jn = next_block(it, j + 1);
                    if (jn < it.T) {
                        if (C::P_OWN) {
                            // S_{g+1} overwrites S_g as soon as the softmax has read it.
                            if (!mbar_wait(&bars->s_read, g & 1) || !issue_s(g + 1)) { ok = false; break; }
                        } else if (C::SBUF == 2) {
                            if (!issue_s(g + 1)) { ok = false; break; }  // other buffer is free
                        }
                    } else {
                        mma_commit(&bars->q_empty[qb]);  // every S of the item is issued: Q is free
                    }
                    const int s = g % C::NS;
                    if (!mbar_wait(&bars->p_full[g % C::SBUF], (g / C::SBUF) & 1) ||
                        !mbar_wait(&bars->v_full[s], (g / C::NS) & 1)) { ok = false; break; }
                    // the item's first P V restarts O: the previous epilogue must have read it
                    if (jj == 0 && t > 0 && !mbar_wait(&bars->o_empty, (t - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t p_tmem =
                        tmem + (C::P_OWN ? C::COL_P : (uint32_t)((g % C::SBUF) * BN));
                    const uint64_t vd = v_desc + (uint64_t)((s * C::VSTAGE) >> 4);
#pragma unroll
                    for (int kk = 0; kk < C::KS_PV; ++kk) {
                        const uint64_t vo = (uint64_t)(kk * C::PV_STEP >> 4);
                        if constexpr (F8)
                            mma_ts_f8(tmem + C::COL_O, p_tmem + kk * 8, vd + vo, kIdescO,
                                      (jj > 0 || kk > 0) ? 1u : 0u);
                        else
                            mma_ts(tmem + C::COL_O, p_tmem + kk * 8, vd + vo, kIdescO,
                                   (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    mma_commit(&bars->kv_empty[s]);
                    mma_commit(&bars->o_full);
                    j = jn;
                }
                gj += jj;
                ++t;
            }
        }
    } else {
        // ------------------------------ softmax warps ------------------------------
        const int t = threadIdx.x;  // 0..127: row in the tile and TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t ob = tmem + lane_base + C::COL_O;
        const float sl2 = p.scale_log2;
        bool ok = true;
        int gj = 0;  // global block count
        Item it;
        // (the next item is looked up at the start of each item's epilogue and carried over)
        bool have_item = item_at(0, it);
        for (int r = 0; have_item; ++r) {
        const int qt = it.qt, bh = it.bh, L = it.L, T = it.T, split = it.split;
        const int row = qt * C::BM + t;
        const bool any_block = it.j_first < T;
        float m = -INFINITY;  // running max, in units of log2 (already scaled)
        float l = 0.f;        // running normaliser
        int jj = 0;           // blocks of this item so far
        for (int j = it.j_first; ok && j < T; j = next_block(it, j + 1), ++jj) {
            const int g = gj + jj;
            // (waits are voted on, so that a warp leaves the loop together: the loop body
            // has warp-wide TMEM loads and votes)
            if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[g % C::SBUF], (g / C::SBUF) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t sb = tmem + lane_base + (uint32_t)((g % C::SBUF) * BN);
            float s[BN];
            {
                uint32_t rr[BN];
                if constexpr (BN == 64) tmem_ld64(sb, rr);
                else tmem_ld128(sb, rr);
#pragma unroll
                for (int i = 0; i < BN; ++i) s[i] = __uint_as_float(rr[i]);
            }
            if (C::P_OWN) {
                tc_fence_before();
                mbar_arrive(&bars->s_read);
            }
            const bool need_mask =
                ((j + 1) * BN > L) || (p.causal && (j + 1) * BN - 1 > qt * C::BM + p.causal_off);
            if (need_mask) {
                // keys < lim are visible
                const int lim = p.causal ? min(L, row + 1 + p.causal_off) : L;
                const int c0 = lim - j * BN;
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (c >= c0) s[c] = -INFINITY;
            }
            // row max: eight independent chains of three-input maxima, then a short tree
            float mxv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                mxv[e] = fmax3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
                for (int c = 24; c + 8 < BN; c += 16) mxv[e] = fmax3(mxv[e], s[c + e], s[c + 8 + e]);
                if constexpr ((BN / 8 - 3) % 2 == 1) mxv[e] = fmaxf(mxv[e], s[BN - 8 + e]);
            }
            const float mx = fmax3(fmax3(mxv[0], mxv[1], mxv[2]), fmax3(mxv[3], mxv[4], mxv[5]),
                                   fmaxf(mxv[6], mxv[7])) * sl2;
            // Lazy rescale: move m only when the max grew by more than 2^8.
            const bool grow = mx > m + 8.0f;
            const bool any_grow = __any_sync(0xffffffffu, grow);
            float alpha = 1.f;
            if (any_grow && mx > m) {
                alpha = ex2(m - mx);  // m == -inf gives 0
                m = mx;
            }
            const float m_use = (m == -INFINITY) ? 0.f : m;
            float sum0 = 0.f, sum1 = 0.f;
            // P in the P V operand format: 16-bit pairs, or (F8) four E4M3 per word
            constexpr int PW = F8 ? BN / 4 : BN / 2;
            uint32_t pk[PW];
            if constexpr (F8) {
#pragma unroll
                for (int c = 0; c < BN; c += 4) {
                    const float p0 = ex2(fmaf(s[c], sl2, -m_use));
                    const float p1 = ex2(fmaf(s[c + 1], sl2, -m_use));
                    const float p2 = ex2(fmaf(s[c + 2], sl2, -m_use));
                    const float p3 = ex2(fmaf(s[c + 3], sl2, -m_use));
                    sum0 += p0 + p2;
                    sum1 += p1 + p3;
                    pk[c >> 2] = pack_e4m3x4(p0, p1, p2, p3);
                }
            } else {
#pragma unroll
                for (int c = 0; c < BN; c += 2) {
                    const float p0 = ex2(fmaf(s[c], sl2, -m_use));
                    const float p1 = ex2(fmaf(s[c + 1], sl2, -m_use));
                    sum0 += p0;
                    sum1 += p1;
                    pk[c >> 1] = pack2<BF16>(p0, p1);
                }
            }
            if constexpr (DROP) {
                // Keys j*BN + 16u .. +15 of this row: one Philox block each; dropped
                // probabilities become 0 in the operand of the PV product.
                const uint32_t g0 = (uint32_t)(j * BN) >> 4;
#pragma unroll
                for (int u = 0; u < BN / 16; ++u) {
                    const uint4 rr = philox4x32_10(g0 + u, (uint32_t)row, (uint32_t)bh,
                                                   p.drop.offset, p.drop.seed_lo, p.drop.seed_hi);
                    const uint32_t w4[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        uint32_t m01, m23;
                        pair_masks(w4[k], p.drop.add16, m01, m23);
                        pk[8 * u + 2 * k] &= m01;
                        pk[8 * u + 2 * k + 1] &= m23;
                    }
                }
            }
            l = l * alpha + (sum0 + sum1);
            // Every phase of o_full is waited on, in order, so that a parity wait can never
            // alias a phase two ahead.  P_{g-1} V_{g-1} (possibly the previous item's last)
            // was issued a whole softmax block ago, so this wait is normally satisfied.  It
            // also frees P's columns (d = 64) before P_g is written there.
            if (g > 0) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full, (g - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            if (jj > 0 && any_grow) {
                // Rescale the accumulated output and row sums (P_{g-1} V_{g-1} is done).
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t rr[32];
                    tmem_ld32(ob + c * 32, rr);
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                    tmem_st32(ob + c * 32, rr);
                }
                {
                    uint32_t rr[16];
                    tmem_ld16(ob + D, rr);
#pragma unroll
                    for (int i = 0; i < 16; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
                    tmem_st16(ob + D, rr);
                }
            }
            {
                const uint32_t pb = C::P_OWN ? tmem + lane_base + C::COL_P : sb;
#pragma unroll
                for (int h = 0; h < PW / 32; ++h) {
                    uint32_t rr[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) rr[i] = pk[h * 32 + i];
                    tmem_st32(pb + h * 32, rr);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->p_full[g % C::SBUF]);
        }

        // ------------------------------ epilogue of the item ---------------------------
        Item nxt;
        const bool have_next = item_at(r + 1, nxt);
        if (!have_next) pdl_launch_dependents();  // this CTA's last item
        if (ok && jj > 0) {
            ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, (gj + jj - 1) & 1));
            tc_fence_after();
        }
        const bool have = any_block;  // warp-uniform: TMEM loads are warp-wide
        float l_round = 0.f;
        if (have) {
            uint32_t rr[16];
            tmem_ld16(ob + D, rr);
            l_round = __uint_as_float(rr[0]);
        }
        // Without dropout the output is divided by the sum of the rounded probabilities
        // the MMA used; with dropout those no longer sum the row, and the output is
        // (sum of kept P v) * keep_scale / l.
        float inv;
        if constexpr (DROP) inv = (l > 0.f) ? p.drop.keep_scale / l : 0.f;
        else inv = (l > 0.f && l_round > 0.f) ? 1.f / l_round : 0.f;
        if constexpr (F8) inv *= p.out_scale;
        const float lse_row = (l > 0.f) ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
        // O straight from TMEM to registers to global memory, 32 columns at a time; the
        // accumulator is released (o_empty) once every column has been read.
#pragma unroll
        for (int c32 = 0; c32 < D / 32; ++c32) {
            uint32_t rr[32];
            if (have) {
                tmem_ld32(ob + c32 * 32, rr);
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) rr[i] = 0u;
            }
            if (c32 == D / 32 - 1 && any_block) {
                tc_fence_before();
                mbar_arrive(&bars->o_empty);
            }
            if (row < p.N) {
                if constexpr (SPLIT) {
                    const size_t prow = ((size_t)split * p.BH + bh) * p.N + row;
                    float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * D) + c32 * 8;
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(
                            __uint_as_float(rr[4 * i]) * inv, __uint_as_float(rr[4 * i + 1]) * inv,
                            __uint_as_float(rr[4 * i + 2]) * inv, __uint_as_float(rr[4 * i + 3]) * inv);
                } else {
                    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.o) +
                                                           ((size_t)bh * p.N + row) * D) + c32 * 4;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_uint4(
                            pack2<BF16>(__uint_as_float(rr[8 * q4]) * inv, __uint_as_float(rr[8 * q4 + 1]) * inv),
                            pack2<BF16>(__uint_as_float(rr[8 * q4 + 2]) * inv, __uint_as_float(rr[8 * q4 + 3]) * inv),
                            pack2<BF16>(__uint_as_float(rr[8 * q4 + 4]) * inv, __uint_as_float(rr[8 * q4 + 5]) * inv),
                            pack2<BF16>(__uint_as_float(rr[8 * q4 + 6]) * inv, __uint_as_float(rr[8 * q4 + 7]) * inv));
                }
            }
        }
        if (row < p.N) {
            if constexpr (SPLIT) p.part_lse[((size_t)split * p.BH + bh) * p.N + row] = lse_row;
            else p.lse[(size_t)bh * p.N + row] = lse_row;
        }
        if (any_block) gj += jj;
        if (!ok) break;
        it = nxt;
        have_item = have_next;
        }  // items
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, C::TMEM_COLS);
}

// Merges the split-KV partial results: with the per-split LSE_s of a row,
//   LSE = M + ln sum_s e^(LSE_s - M)  (M = max_s LSE_s),   O = sum_s e^(LSE_s - LSE) O_s,
// which is the online-softmax (m, l) merge applied once to whole key ranges.  Rows whose
// every split saw no key get O = 0, LSE = -inf.  D / 4 threads per row, four columns each.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_splitkv_combine_kernel(const float *part_o,
                                                                const float *part_lse, void *o,
                                                                float *lse, long long rows,
                                                                int num_splits) {
    constexpr int G = D / 4;       // threads per row
    constexpr int RPW = 32 / G;    // rows per warp step
    pdl_wait();
    pdl_launch_dependents();
    const long long tid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane % G;
    for (long long base = (tid >> 5) * RPW; base < rows; base += nwarps * RPW) {
        const long long r = base + lane / G;
        if (r >= rows) continue;
        float mx = -INFINITY;
        for (int s = 0; s < num_splits; ++s) mx = fmaxf(mx, part_lse[(long long)s * rows + r]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float out_lse = -INFINITY;
        if (mx != -INFINITY) {
            float sum = 0.f;
            for (int s = 0; s < num_splits; ++s) {
                const float ls = part_lse[(long long)s * rows + r];
                if (ls == -INFINITY) continue;
                const float w = __expf(ls - mx);
                sum += w;
                const float4 v = reinterpret_cast<const float4 *>(part_o + ((long long)s * rows + r) * D)[g];
                acc.x = fmaf(w, v.x, acc.x);
                acc.y = fmaf(w, v.y, acc.y);
                acc.z = fmaf(w, v.z, acc.z);
                acc.w = fmaf(w, v.w, acc.w);
            }
            const float inv = 1.f / sum;
            acc = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
            out_lse = mx + __logf(sum);
        }
        reinterpret_cast<uint2 *>(o)[r * G + g] =
            make_uint2(pack2<BF16>(acc.x, acc.y), pack2<BF16>(acc.z, acc.w));
        if (g == 0) lse[r] = out_lse;
    }
}

}  // namespace fa
