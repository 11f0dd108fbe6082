/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library (libfa.so).
 *
 * The library computes exact attention O = softmax(scale * Q K^T + mask) V and its
 * gradients without ever forming the N x N score matrix in device memory:
 *   - the method: tile Q, K, V into on-chip blocks and update the output with an
 *     online softmax that carries a running row maximum m and normaliser l
 *     (anthology note "NOTE-005: FlashAttention", section "Method"; aicassindra
 *     FlashAttention architecture page, "End-to-end flow");
 *   - exactness: the result equals standard attention up to floating-point ordering
 *     (NOTE-005, Theorem 1; promptingindex page "FlashAttention: The IO-Aware
 *     Algorithm That Rewrote GPU Training Speed Records", section "Tiling");
 *   - the backward pass recomputes each probability block from the stored
 *     statistics instead of reading a saved matrix (NOTE-005, "Method" and "Key
 *     components"; aicassindra page, "The architecture: every piece explained").
 * The forward pass stores the two statistics as one array, the log-sum-exp
 * LSE_i = m_i + ln l_i (natural log).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout: Q, K, V, O, dO, dQ, dK, dV are contiguous row-major [B, H, N, d] arrays of
 *   the element type `dtype` (d innermost).  LSE is a contiguous fp32 [B, H, N] array.
 *   Q, K and V share the sequence length N (self-attention).
 * Mask: key j is visible to query i iff j < L_b and (causal == 0 or j <= i), with
 *   L_b = kv_len[b] clamped to [0, N], or L_b = N when kv_len is NULL.  kv_len, when
 *   given, is a DEVICE pointer to B int32 values.  Masked scores are -inf.  A query
 *   row that sees no key (only when L_b = 0) gets O = 0, LSE = -inf and zero gradient.
 * Scale: `scale` multiplies Q K^T before masking; it must be finite and > 0
 *   (typically 1/sqrt(d)).
 * Supported: d in {64, 128}; dtype FA_BF16 or FA_FP16 (fp32 accumulation inside);
 *   any N >= 1, B >= 1, H >= 1, B*H < 2^31, and at most FA_MAX_ELEMENTS elements in
 *   one [B, H, N, d] tensor.  Device: compute capability 10.0 (B200, sm_100a) only.
 * Pointers: all tensor pointers are DEVICE pointers, 16-byte aligned, owned by the
 *   caller; the library never allocates, frees or retains them after the call.
 * Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  Every entry
 *   point only enqueues work on `stream` and returns; results are ready once the
 *   stream is synchronised.
 * Errors: arguments are checked before anything is enqueued.  FA_ERR_INVALID_ARG:
 *   null or misaligned pointer, non-positive size, bad scale or dtype, workspace
 *   too small.  FA_ERR_UNSUPPORTED: d not 64/128, tensor too large, device not
 *   sm_100.  FA_ERR_CUDA: a CUDA call or launch failed (see fa_last_cuda_error()).
 *   There is no fallback of any kind: an unsupported call does no work.
 * Device-side waits are bounded.  A wait that gives up records FA_ERR_TIMEOUT in a
 *   per-device status word readable with fa_get_device_status().
 * Thread safety: every entry point may be called concurrently from several host
 *   threads; the only global state is a per-device status word and cached device
 *   properties.
 */
#ifndef FA_H
#define FA_H

#include <stddef.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1,
    FA_ERR_UNSUPPORTED = 2,
    FA_ERR_CUDA = 3,
    FA_ERR_TIMEOUT = 4,
    FA_ERR_SCRATCH_LIMIT = 5
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Largest element count of one [B, H, N, d] tensor the kernels index. */
#define FA_MAX_ELEMENTS ((long long)1 << 40)

/*
 * Forward pass (NOTE-005 "Method": tiles of Q against all K/V tiles, online softmax
 * with running m and l; output O and the row statistics).
 *   q, k, v : [B, H, N, d] dtype, read only.
 *   o       : [B, H, N, d] dtype, written.
 *   lse     : [B, H, N] fp32, written; LSE_i = ln sum_j exp(scale q_i.k_j) over the
 *             visible keys (-inf for a row that sees none).
 *   kv_len  : NULL or device int32[B] (see Mask above).
 * Returns FA_OK or an error code (nothing is enqueued on error).
 */
FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
           int B, int H, int N, int d, float scale, int causal, const int *kv_len,
           int dtype, void *stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes: an fp32 [B, H, N, d] dQ
 * accumulator, then two fp32 [B, H, ceil(N/128)*128] arrays (D_i = sum_c dO_ic O_ic
 * and the log-sum-exp in base 2), each 256-byte aligned.  Returns 0 for invalid sizes.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass of the loss sum(O * dO): recomputes every probability block from
 * q, k and the stored lse (NOTE-005 "Method": recompute rather than read a saved
 * matrix) and writes dQ, dK, dV.
 *   q, k, v, o, dout : [B, H, N, d] dtype, read only (o and lse from fa_fwd with the
 *                      same q, k, v, scale, causal and kv_len).
 *   lse              : [B, H, N] fp32, read only.
 *   dq, dk, dv       : [B, H, N, d] dtype, written (rows of dK/dV for keys >= L_b
 *                      are written as exact zeros).
 *   workspace        : device buffer of at least fa_bwd_workspace_bytes() bytes,
 *                      256-byte aligned; its contents on entry do not matter and
 *                      are clobbered.
 * Enqueues three kernels on `stream` (row-dot preprocess, main pass, dQ convert).
 */
FA_API int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
           float scale, int causal, const int *kv_len, int dtype, void *workspace,
           size_t workspace_bytes, void *stream);

/* Static, NUL-terminated description of a status code. */
FA_API const char *fa_strerror(int status);

/* Text of the last CUDA error this host thread saw inside the library ("" if none). */
FA_API const char *fa_last_cuda_error(void);

/*
 * Synchronises `stream`, then reads and clears the current device's status word.
 * Returns FA_OK, FA_ERR_TIMEOUT if some kernel gave up a bounded wait since the
 * last call, or FA_ERR_CUDA if the synchronisation failed.
 */
FA_API int fa_get_device_status(void *stream);

/*
 * Block-sparse attention (promptingindex page, "Benchmark results": the same tiling
 * applied to sparse patterns; NOTE-005, "Key components" and "Limitations": the
 * block-sparse extension, which is exact for its pattern and approximate as a stand-in
 * for dense attention).  Identical to fa_fwd / fa_bwd except that key j is visible to
 * query i only if, in addition to the Mask rule above,
 *     block_mask[i / 128][j / 128] != 0.
 * Skipped blocks are neither loaded nor multiplied.
 *   block_mask    : DEVICE pointer to uint8 [T][T] (T = ceil(N / 128)), row = query tile,
 *                   column = key tile; with mask_per_head = 1, [B * H][T][T] (index
 *                   b * H + h).  Read only.
 *   mask_per_head : 0 (one mask for every batch and head) or 1.
 * Rows whose visible set is empty get O = 0, LSE = -inf and zero gradients.  The backward
 * call must be given the same mask as the forward call that produced o and lse.
 * Returns FA_ERR_INVALID_ARG for a null mask or a bad mask_per_head; otherwise as fa_fwd /
 * fa_bwd.
 */
FA_API int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                              int B, int H, int N, int d, float scale, int causal,
                              const int *kv_len, const unsigned char *block_mask,
                              int mask_per_head, int dtype, void *stream);

FA_API int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o,
                              const void *dout, const float *lse, void *dq, void *dk, void *dv,
                              int B, int H, int N, int d, float scale, int causal,
                              const int *kv_len, const unsigned char *block_mask,
                              int mask_per_head, int dtype, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * Inference-shaped forward (stackzen.ai glossary entry "FlashAttention", which cites the
 * method's saving of memory traffic at inference as well as in training): Nq queries
 * against Nk keys, Nq usually much smaller than Nk (decoding, or a chunk of new tokens
 * against a long cache).  The
 * queries are the last Nq positions of the key sequence:
 *     key j is visible to query i  iff  j < kv_len[b]  and  (!causal or j <= i + Nk - Nq).
 * The key range is split into num_splits parts processed by separate CTAs (so that a
 * short query block still fills the GPU); each part produces its own normalised output
 * and LSE, and a second kernel merges them with the online-softmax (m, l) rule:
 *     LSE = M + ln sum_s e^(LSE_s - M),  O = sum_s e^(LSE_s - LSE) O_s,  M = max_s LSE_s.
 * The result equals fa_fwd's up to floating-point order (with Nq = Nk and num_splits = 1
 * it is fa_fwd).
 *   q, o       : DEVICE [B, H, Nq, d] 16-bit; lse: DEVICE [B, H, Nq] fp32.
 *   k, v       : DEVICE [B, H, Nk, d] 16-bit.
 *   num_splits : 0 = chosen by the library (the count, up to 128 with at least two key
 *                blocks per split, that minimises rounds x (blocks per split + 2) on a
 *                grid of one persistent CTA per SM slot), else 1 .. FA_MAX_SPLITS (capped
 *                by the number of key blocks: 64 keys at d = 64, 128 at d = 128).
 *   workspace  : DEVICE scratch of fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d,
 *                num_splits) bytes, 256-byte aligned, owned by the caller (may be NULL when
 *                that size is 0, i.e. when the call resolves to one split).  The size is
 *                computed for the current device; call both on the same device.
 * Returns FA_ERR_INVALID_ARG for the checks of fa_fwd, Nk < 1, num_splits outside
 * [0, FA_MAX_SPLITS], or a missing / small / misaligned workspace; otherwise as fa_fwd.
 * Not valid for training: there is no matching backward entry point.
 */
#define FA_MAX_SPLITS 256

FA_API size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits);

FA_API int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int H, int Nq, int Nk, int d, float scale, int causal,
                          const int *kv_len, int num_splits, int dtype, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * FP8 forward (the FlashAttention-3 low-precision variant the aicassindra page and the
 * promptingindex page, "Adoption", name): Q, K and V in E4M3 (one byte per element,
 * [B, H, N, d] like the 16-bit calls), each with one fp32 scale factor, so that the
 * represented values are q_scale * Q8, k_scale * K8, v_scale * V8.  Computes the same
 * attention as fa_fwd of those values: S = (scale * q_scale * k_scale) Q8 K8^T in fp32 on
 * E4M3 tensor cores (kind::f8f6f4), the online softmax in fp32, P rounded to E4M3 for the
 * P V product (its row sums come out of the same rounded values), O = v_scale * (P V) / l
 * written in bf16, LSE in fp32.
 *   q, k, v : DEVICE E4M3 bytes [B, H, N, d]; o: DEVICE bf16 [B, H, N, d]; lse: fp32.
 *   d       : 128 only (FA_ERR_UNSUPPORTED otherwise).
 * Accuracy: the inputs are exact (the reference is attention of the scaled E4M3 values);
 * the rounding of P to E4M3 (3 mantissa bits) perturbs each weight by up to 2^-4
 * relative, so |O - O_exact| <= 2^-3 max_j |v_j| in the worst case; in practice errors are
 * far smaller (see the parity tests).  Returns FA_ERR_INVALID_ARG for the fa_fwd checks
 * or a non-finite / non-positive scale factor.  Forward only (no FP8 backward).
 */
FA_API int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                      int H, int N, int d, float scale, int causal, const int *kv_len,
                      float q_scale, float k_scale, float v_scale, void *stream);

/*
 * Attention with dropout on the probabilities (promptingindex page, "Why attention is
 * memory-bound, not compute-bound": dropout is the op between the softmax and the
 * product with V).  Identical to fa_fwd / fa_bwd except that
 *     O_i = sum_j P_ij K_ij r v_j,   r = 256 / (256 - t),   t = rint(256 * p_drop),
 * where P is the softmax of the Mask rule above (LSE is unchanged) and K_ij = 1 when
 * the random byte of element (i, j) is >= t.  The backward call returns the gradients
 * of that O (dV = r (P o K)^T dO, dP = r K o (dO V^T), D = rowsum(dO o O), dS = P o
 * (dP - D)) and must be given the same p_drop, seed and offset as the forward call.
 * The mask is never stored: both calls regenerate it (the recomputation of NOTE-005,
 * "Method", applied to the random numbers).
 *   p_drop : drop probability, used as t / 256 (nearest multiple of 1/256, ties to
 *            even); t must lie in [0, 255], i.e. 0 <= p_drop < 255.5 / 256.  p_drop = 0
 *            keeps everything (same O as fa_fwd up to the normaliser's rounding).
 *   seed   : 64-bit key of the generator.
 *   offset : 32-bit stream number (e.g. layer or step), fourth word of the counter.
 * Random byte of element (i, j) of head bh = b * H + h: byte j mod 16 of the 16 output
 * bytes (byte k = bits 8 (k mod 4) .. +7 of word k / 4) of Philox4x32-10 (Salmon et al.,
 * "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011) with counter
 * (j / 16, i, bh, offset) and key (seed mod 2^32, seed >> 32).
 * Returns FA_ERR_INVALID_ARG for a p_drop outside the range; otherwise as fa_fwd / fa_bwd.
 */
FA_API int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse,
                          int B, int H, int N, int d, float scale, int causal,
                          const int *kv_len, float p_drop, unsigned long long seed,
                          unsigned int offset, int dtype, void *stream);

FA_API int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o,
                          const void *dout, const float *lse, void *dq, void *dk, void *dv,
                          int B, int H, int N, int d, float scale, int causal,
                          const int *kv_len, float p_drop, unsigned long long seed,
                          unsigned int offset, int dtype, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * The keep mask that fa_fwd_dropout / fa_bwd_dropout use, written out:
 *   keep : DEVICE pointer to uint8 [B * H][N][N], keep[bh][i][j] = K_ij (1 or 0),
 *          written by the call (asynchronously on `stream`).
 * For inspection and tests; it materialises N^2 bytes per head, which the attention
 * calls never do.  Returns FA_ERR_INVALID_ARG for a null pointer, B, H or N < 1, a bad
 * p_drop, or more than FA_MAX_ELEMENTS mask bytes.
 */
FA_API int fa_dropout_mask(int B, int H, int N, float p_drop, unsigned long long seed,
                           unsigned int offset, unsigned char *keep, void *stream);

/*
 * Backward pass for callers that cannot allocate device memory.  The FlashAttention
 * pages have no counterpart to this entry point: it exists for the environment, not the
 * method.  Some hosts of this library may not call cudaMalloc at all: plugins inside
 * an inference engine or framework that owns every byte of device memory and hands its
 * plugins no allocator, and serving loops that forbid device allocation once they have
 * started, because cudaMalloc can synchronise the device and stall every stream.  Such
 * callers can still provide their inputs and outputs but have nowhere to get the
 * backward pass's scratch from.
 *
 * fa_bwd_noalloc computes exactly what fa_bwd computes (same arguments, same kernels,
 * same results) but takes its scratch (the fp32 dQ accumulator and the two per-row
 * vectors described at fa_bwd_workspace_bytes) from one static device array of
 * FA_NOALLOC_SCRATCH_BYTES bytes inside the library.  Every GPU that loads the
 * library holds that array until the process exits.  The entry point itself calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Limit: the call is accepted only if fa_bwd_workspace_bytes(B, H, N, d) <=
 * FA_NOALLOC_SCRATCH_BYTES; with N a multiple of 128 that is up to B*H*N = 254080 rows
 * at d = 64 and 129024 rows at d = 128.  Larger problems return FA_ERR_SCRATCH_LIMIT and
 * enqueue nothing.
 *
 * Set-up: the first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream capture begins.
 * The cache is kept per device ordinal for the life of the process, so it assumes the
 * device's primary context (the one the CUDA runtime uses) and no cudaDeviceReset in
 * between: after a reset, or from another context on the same device, the cached
 * address would be stale.
 *
 * Sharing: all calls share the one array, and it keeps the previous call's contents;
 * the call clears what must start at zero itself.  Two calls whose kernels may overlap
 * on the GPU (different streams without ordering, or several host threads) race on the
 * array and produce wrong gradients: order them on one stream, or use fa_bwd with
 * separate workspaces.
 *
 * Arguments, layout, ownership and the other error codes are those of fa_bwd.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
FA_API int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                          const void *dout, const float *lse, void *dq, void *dk, void *dv,
                          int B, int H, int N, int d, float scale, int causal,
                          const int *kv_len, int dtype, void *stream);

/*
 * Optional timing hook for profiling.  After this call, every launch made by this host
 * thread of the selected kernel records `start` on the launch stream immediately
 * before the kernel and `stop` immediately after it, so cudaEventElapsedTime(start,
 * stop) is that kernel's device time.  which = 0: the forward kernel of fa_fwd;
 * which = 1: the main kernel of fa_bwd (not its preprocess and convert kernels).
 * start, stop: cudaEvent_t handles created by the caller, or both NULL to switch the
 * hook off.  Returns FA_OK or FA_ERR_INVALID_ARG.
 */
FA_API int fa_set_timing_events(int which, void *start, void *stop);

/*
 * Self-test of the bounded device waits: enqueues one kernel whose single thread waits
 * on a barrier that nothing ever completes, with a limit of `limit_us` microseconds
 * (1 .. 2000000).  The wait gives up and records FA_ERR_TIMEOUT in the device status
 * word, exactly as a stalled wait inside fa_fwd / fa_bwd would; the CUDA context stays
 * usable.  Returns FA_OK once enqueued.
 */
FA_API int fa_selftest_wait_timeout(int limit_us, void *stream);

/* The static schedule the launchers give the persistent kernels for causal shapes with
 * several work items per CTA (no key lengths, no block mask): items 0 .. n-1 with host
 * costs cost[i] (> 0) are split over `lists` lists so that the largest list total is small
 * (longest first onto the least loaded list, then moves and swaps out of the fullest
 * list); list c is ids[off[c]] .. ids[off[c + 1] - 1], heaviest item first.  Host memory:
 * cost[n], off[lists + 1], ids[n], all owned by the caller.  Pure host computation (no
 * GPU, no CUDA call).  FA_ERR_INVALID_ARG for a null pointer, n < 1 or n > 2048, lists < 1
 * or lists > 512, or a cost that is not a positive finite number. */
FA_API int fa_schedule_items(const float *cost, int n, int lists, unsigned short *off,
                             unsigned short *ids);

/* Library version, major * 10000 + minor * 100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H */
