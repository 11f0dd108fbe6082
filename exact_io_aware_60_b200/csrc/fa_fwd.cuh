// fa_fwd.cuh -- forward pass of exact tiled attention on sm_100a.
//
// The method (anthology note "NOTE-005: FlashAttention", section "Method"; aicassindra
// FlashAttention architecture page, "End-to-end flow"): split Q into row blocks and
// K, V into key blocks, bring one block at a time on chip, form that block of scores
// there, and fold it into the output with an online softmax that carries a running row
// maximum m and normaliser l, rescaling the accumulated output whenever m grows.  Only
// O and the row statistics leave the chip; the N x N score matrix never exists in HBM.
//
// B200 mapping (one CTA = one 128-row query tile of one (batch, head)):
//   warp 4      TMA producer: Q once, then K_j / V_j into an NS-stage shared-memory ring
//               (128-byte swizzle, mbarrier transaction counts).
//   warp 5      MMA issuer (one thread): S_j = Q K_j^T into TMEM, then O += P_j V_j with
//               P_j read straight from TMEM.
//   warps 0..3  softmax, one query row per thread (TMEM lane = row): load S_j, mask on
//               diagonal / tail blocks only, row max, p = 2^(s*scale*log2e - m) with the
//               MUFU ex2, row sum, P_j written back into TMEM as 16-bit pairs.
//               The output rescale is lazy: m only moves when the row max grows by more
//               than 2^8, which leaves the result exact because O and l always share the
//               same m.  Epilogue: O / l' -> 16-bit, staged swizzled in shared memory and
//               written with one TMA store; LSE = ln2 * (m + log2 l).
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
    static constexpr int NS = (D == 64) ? 4 : 2;        // K/V ring depth
    // Each V stage is followed by a block of 16-bit ones, one 64-column block past the
    // tile: the PV MMA reads it as B columns D..D+15 and so also produces the row sums
    // of P (one N = D + 16 instruction instead of a second, equally costly N = 16 one).
    static constexpr int VSTAGE = (HALVES + 1) * KHALF;  // V block + its ones block
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QTILE;
    static constexpr int OFF_V = OFF_K + NS * KTILE;
    static constexpr int OFF_BAR = OFF_V + NS * VSTAGE;
    static constexpr int USED = OFF_BAR + 256;
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
    static constexpr int NS = 4;
    static constexpr int VSTAGE = 2 * KHALF;            // V block + its block of E4M3 ones
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + QTILE;
    static constexpr int OFF_V = OFF_K + NS * KTILE;
    static constexpr int OFF_BAR = OFF_V + NS * VSTAGE;
    static constexpr int USED = OFF_BAR + 256;
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
    uint64_t q_full;
    uint64_t s_full[2];
    uint64_t s_read;
    uint64_t p_full[2];
    uint64_t o_full;
    uint64_t k_full[4];
    uint64_t v_full[4];
    uint64_t kv_empty[4];
    uint32_t tmem_base;
};

// DROP: dropout on the probabilities (the mask is regenerated per element from the
// counter-based generator; the normaliser is the fp32 sum of the undropped values).
// SPLIT: the CTA covers one range of key blocks and writes an fp32 partial output (O
// normalised by that range's own l) and the range's LSE; a combine kernel merges them.
// F8: E4M3 Q, K, V (d = 128), kind::f8f6f4 MMAs, P rounded to E4M3 for the P V product,
// bf16 output (BF16 = true).
template <int D, bool BF16, bool DROP, bool SPLIT, bool F8 = false>
__global__ void __launch_bounds__(192, FwdCfg<D>::CTAS_PER_SM)
fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const FwdParams p) {
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

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: (query tile, key split, head); heaviest causal tiles are launched first.
    const int bh = blockIdx.x % p.BH;
    const int rest = blockIdx.x / p.BH;
    const int split = rest % p.num_splits;
    const int tile_rank = rest / p.num_splits;
    const int qt = p.causal ? (p.num_q_tiles - 1 - tile_rank) : tile_rank;
    const int b = bh / p.H;
    // Softmax warps that hold at least one query row; the others skip the block loop, and
    // the per-block barriers count only the active ones.
    const int n_active = min(4, (p.N - qt * C::BM + 31) >> 5);

    if (threadIdx.x == 128) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmO);
        mbar_init(&bars->q_full, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars->s_full[i], 1);
            mbar_init(&bars->p_full[i], 32 * n_active);
        }
        mbar_init(&bars->s_read, 32 * n_active);
        mbar_init(&bars->o_full, 1);
        for (int i = 0; i < C::NS; ++i) {
            mbar_init(&bars->k_full[i], 1);
            mbar_init(&bars->v_full[i], 1);
            mbar_init(&bars->kv_empty[i], 1);
        }
        fence_mbar_init();
    }
    if (warp == 4) {
        // 16-bit ones after every V stage (layout-agnostic: every element is 1)
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

    int L = p.Nk;
    if (p.kv_len != nullptr) {
        L = p.kv_len[b];
        L = L < 0 ? 0 : (L > p.Nk ? p.Nk : L);
    }
    int kv_end = L;
    if (p.causal) kv_end = min(kv_end, (qt + 1) * C::BM + p.causal_off);
    int T = kv_end > 0 ? (kv_end + BN - 1) / BN : 0;  // key blocks in range
    int j_lo = 0;
    if (p.kv_blocks_per_split > 0) {  // this split's blocks: [j_lo, T)
        j_lo = split * p.kv_blocks_per_split;
        T = min(T, j_lo + p.kv_blocks_per_split);
    }
    // Block-sparse walk: next key block at or after j whose tile is set (T if none).
    const uint8_t *mrow =
        p.bmask ? p.bmask + (size_t)bh * p.bmask_bh_stride + (size_t)qt * p.bmask_T : nullptr;
    auto next_block = [&](int j) -> int {
        if (mrow)
            while (j < T && mrow[(j * BN) >> 7] == 0) ++j;
        return j;
    };
    const int j_first = next_block(j_lo);
    const bool any_block = j_first < T;

    if (warp == 4) {
        // ------------------------------ TMA producer ------------------------------
        if (lane == 0 && any_block) {
            mbar_arrive_expect_tx(&bars->q_full, C::QTILE);
            for (int hf = 0; hf < C::HALVES; ++hf)
                tma_load_3d(sQ + hf * C::QHALF, &tmQ, &bars->q_full, hf * 64, qt * C::BM, bh);
            int jj = 0;  // index among the visited blocks: drives stages and phases
            for (int j = j_first; j < T; j = next_block(j + 1), ++jj) {
                const int s = jj % C::NS;
                if (jj >= C::NS && !mbar_wait(&bars->kv_empty[s], ((jj / C::NS) - 1) & 1)) break;
                mbar_arrive_expect_tx(&bars->k_full[s], C::KTILE);
                for (int hf = 0; hf < C::HALVES; ++hf)
                    tma_load_3d(sK + s * C::KTILE + hf * C::KHALF, &tmK, &bars->k_full[s], hf * 64,
                                j * BN, bh);
                mbar_arrive_expect_tx(&bars->v_full[s], C::KTILE);
                for (int hf = 0; hf < C::HALVES; ++hf)
                    tma_load_3d(sV + s * C::VSTAGE + hf * C::KHALF, &tmV, &bars->v_full[s], hf * 64,
                                j * BN, bh);
            }
        }
    } else if (warp == 5) {
        // ------------------------------ MMA issuer --------------------------------
        if (lane == 0 && any_block) {
            constexpr uint32_t kIdescS =
                F8 ? idesc_e4m3(false, false, 128, BN) : idesc_f16(BF16, false, false, 128, BN);
            constexpr uint32_t kIdescO = F8 ? idesc_e4m3(false, true, 128, C::PV_N)
                                            : idesc_f16(BF16, false, true, 128, C::PV_N);
            // Descriptors are built once; per k-step and per stage only the 16-byte start
            // address field changes, by compile-time offsets.
            const uint64_t q_desc = smem_desc_sw128(smem_u32(sQ), 16, 1024);
            const uint64_t k_desc = smem_desc_sw128(smem_u32(sK), 16, 1024);
            const uint64_t v_desc = smem_desc_sw128(smem_u32(sV), C::KHALF, 1024);
            bool ok = mbar_wait(&bars->q_full, 0);
            tc_fence_after();
            // jj: index of the visited block (stages, phases and buffers follow it)
            auto issue_s = [&](int jj) -> bool {
                const int s = jj % C::NS;
                if (!mbar_wait(&bars->k_full[s], (jj / C::NS) & 1)) return false;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)((jj % C::SBUF) * BN);
                const uint64_t kd = k_desc + (uint64_t)((s * C::KTILE) >> 4);
#pragma unroll
                for (int kk = 0; kk < C::KS_S; ++kk) {
                    const uint64_t qo = (uint64_t)(((kk >> 2) * C::QHALF + (kk & 3) * 32) >> 4);
                    const uint64_t ko = (uint64_t)(((kk >> 2) * C::KHALF + (kk & 3) * 32) >> 4);
                    if constexpr (F8) mma_ss_f8(d_tmem, q_desc + qo, kd + ko, kIdescS, kk > 0 ? 1u : 0u);
                    else mma_ss(d_tmem, q_desc + qo, kd + ko, kIdescS, kk > 0 ? 1u : 0u);
                }
                mma_commit(&bars->s_full[jj % C::SBUF]);
                return true;
            };
            if (ok) ok = issue_s(0);
            int jj = 0;
            for (int j = j_first; ok && j < T; ++jj) {
                const int jn = next_block(j + 1);
                if (jn < T) {
                    if (C::P_OWN) {
                        // S_{jj+1} overwrites S_jj as soon as the softmax has read it.
                        if (!mbar_wait(&bars->s_read, jj & 1) || !issue_s(jj + 1)) break;
                    } else if (C::SBUF == 2) {
                        if (!issue_s(jj + 1)) break;  // the other score buffer is free
                    }
                }
                const int s = jj % C::NS;
                if (!mbar_wait(&bars->p_full[jj % C::SBUF], (jj / C::SBUF) & 1)) break;
                if (!mbar_wait(&bars->v_full[s], (jj / C::NS) & 1)) break;
                tc_fence_after();
                const uint32_t p_tmem =
                    tmem + (C::P_OWN ? C::COL_P : (uint32_t)((jj % C::SBUF) * BN));
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
        }
    } else {
        // ------------------------------ softmax warps ------------------------------
        const int t = threadIdx.x;  // 0..127: row in the tile and TMEM lane
        const int row = qt * C::BM + t;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const float sl2 = p.scale_log2;
        float m = -INFINITY;  // running max, in units of log2 (already scaled)
        float l = 0.f;        // running normaliser
        bool ok = true;
        int jj = 0;  // visited blocks so far
        const bool active = warp < n_active;
        for (int j = active ? j_first : T; j < T; j = next_block(j + 1), ++jj) {
            if (!mbar_wait(&bars->s_full[jj % C::SBUF], (jj / C::SBUF) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t sb = tmem + lane_base + (uint32_t)((jj % C::SBUF) * BN);
            float s[BN];
            {
                uint32_t r[BN];
                if constexpr (BN == 64) tmem_ld64(sb, r);
                else tmem_ld128(sb, r);
#pragma unroll
                for (int i = 0; i < BN; ++i) s[i] = __uint_as_float(r[i]);
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
                    const uint4 r = philox4x32_10(g0 + u, (uint32_t)row, (uint32_t)bh,
                                                  p.drop.offset, p.drop.seed_lo, p.drop.seed_hi);
                    const uint32_t w4[4] = {r.x, r.y, r.z, r.w};
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
            // Every phase of o_full is waited on, in order, so that a parity wait can
            // never alias a phase two ahead.  P_{j-1} V_{j-1} was issued a whole softmax
            // block ago, so this wait is normally already satisfied.  It also frees P's
            // columns (d = 64) before P_j is written there.
            if (jj > 0) {
                if (!mbar_wait(&bars->o_full, (jj - 1) & 1)) { ok = false; break; }
                tc_fence_after();
            }
            if (jj > 0 && any_grow) {
                // Rescale the accumulated output and row sums (P_{j-1} V_{j-1} is done).
                const uint32_t ob = tmem + lane_base + C::COL_O;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(ob + c * 32, r);
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st32(ob + c * 32, r);
                }
                {
                    uint32_t r[16];
                    tmem_ld16(ob + D, r);
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
                    tmem_st16(ob + D, r);
                }
            }
            {
                const uint32_t pb = C::P_OWN ? tmem + lane_base + C::COL_P : sb;
#pragma unroll
                for (int h = 0; h < PW / 32; ++h) {
                    uint32_t r[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = pk[h * 32 + i];
                    tmem_st32(pb + h * 32, r);
                }
            }
            tc_fence_before();
            mbar_arrive(&bars->p_full[jj % C::SBUF]);
        }

        // ------------------------------ epilogue ------------------------------
        pdl_launch_dependents();
        if (ok && jj > 0) {
            ok = mbar_wait(&bars->o_full, (jj - 1) & 1);
            tc_fence_after();
        }
        const uint32_t ob = tmem + lane_base + C::COL_O;
        const bool have = active && any_block;  // warp-uniform: TMEM loads are warp-wide
        float l_round = 0.f;
        if (have) {
            uint32_t r[16];
            tmem_ld16(ob + D, r);
            l_round = __uint_as_float(r[0]);
        }
        // Without dropout the output is divided by the sum of the rounded probabilities
        // the MMA used; with dropout those no longer sum the row, and the output is
        // (sum of kept P v) * keep_scale / l.
        float inv;
        if constexpr (DROP) inv = (l > 0.f) ? p.drop.keep_scale / l : 0.f;
        else inv = (l > 0.f && l_round > 0.f) ? 1.f / l_round : 0.f;
        if constexpr (F8) inv *= p.out_scale;
        const float lse_row = (l > 0.f) ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
        if constexpr (SPLIT) {
            // fp32 partial output of this key range, one contiguous row per thread
            const size_t prow = ((size_t)split * p.BH + bh) * p.N + row;
            float4 *dst = reinterpret_cast<float4 *>(p.part_o + prow * D);
#pragma unroll
            for (int c32 = 0; c32 < D / 32; ++c32) {
                uint32_t r[32];
                if (have) {
                    tmem_ld32(ob + c32 * 32, r);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
                if (row < p.N) {
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[c32 * 8 + i] = make_float4(
                            __uint_as_float(r[4 * i]) * inv, __uint_as_float(r[4 * i + 1]) * inv,
                            __uint_as_float(r[4 * i + 2]) * inv, __uint_as_float(r[4 * i + 3]) * inv);
                }
            }
            if (row < p.N) p.part_lse[prow] = lse_row;
        } else {
        // O staging: 16-bit [128 x D] in 64-column blocks of 16 KB, over Q (16-bit
        // inputs) or over the K ring (F8: the E4M3 Q tile is half the size; every K block
        // has been consumed once the last P V is done).
        uint8_t *stage = F8 ? sK : sQ;
        // Warps without query rows leave their staging rows alone: they have not waited
        // for the tile's MMAs, which may still be reading the staging area (their rows
        // would fall outside the tensor and be clipped by the store anyway).
#pragma unroll
        for (int hf = 0; hf < (active ? D / 64 : 0); ++hf) {
            uint32_t w[32];
            {
                uint32_t r[32];
                if (have) {
                    tmem_ld32(ob + hf * 64, r);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = 0u;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv,
                                       __uint_as_float(r[2 * i + 1]) * inv);
                if (have) {
                    tmem_ld32(ob + hf * 64 + 32, r);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    w[16 + i] = pack2<BF16>(__uint_as_float(r[2 * i]) * inv,
                                            __uint_as_float(r[2 * i + 1]) * inv);
            }
            // Row t of this 128-byte column block, 16-byte chunks XOR-swizzled by t % 8.
            uint8_t *rowp = stage + hf * 16384 + t * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint4 v4 = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
                *reinterpret_cast<uint4 *>(rowp + ((c ^ (t & 7)) << 4)) = v4;
            }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (t == 0) {
            for (int hf = 0; hf < D / 64; ++hf)
                tma_store_3d(&tmO, stage + hf * 16384, hf * 64, qt * C::BM, bh);
            bulk_commit_group();
            bulk_wait_group_read<0>();
        }
        if (row < p.N) p.lse[(size_t)bh * p.N + row] = lse_row;
        }  // !SPLIT
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
