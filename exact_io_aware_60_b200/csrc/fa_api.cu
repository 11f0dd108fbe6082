// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA descriptor
// encoding, grid selection and kernel launches.  All kernels live in this single
// translation unit (they are included below), so the device status word needs no
// relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "fa.h"
#include "fa_fwd.cuh"
#include "fa_bwd.cuh"

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int kMaxDevices = 64;

thread_local char t_last_error[256] = "";
thread_local cudaEvent_t t_timing[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};

// Records the profiling event of `which` (0 fwd, 1 bwd main), side 0 before / 1 after.
void timing_mark(int which, int side, cudaStream_t st) {
    if (t_timing[which][side] != nullptr) cudaEventRecord(t_timing[which][side], st);
}

void record_cuda_error(cudaError_t e, const char *where) {
    snprintf(t_last_error, sizeof(t_last_error), "%s: %s (%d)", where, cudaGetErrorString(e),
             (int)e);
}

// ---------------------------------------------------------------- device checks

std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other

int check_device(int *dev_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaGetDevice");
        return FA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    int st = g_dev_ok[dev].load(std::memory_order_relaxed);
    if (st == 0) {
        int major = 0, minor = 0;
        e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (e != cudaSuccess) {
            record_cuda_error(e, "cudaDeviceGetAttribute");
            return FA_ERR_CUDA;
        }
        st = (major == 10 && minor == 0) ? 1 : 2;
        g_dev_ok[dev].store(st, std::memory_order_relaxed);
    }
    *dev_out = dev;
    return st == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D view [BH][rows][cols] of a contiguous tensor; box = box_cols x box_rows x 1.
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem_bytes,
              long long cols, long long rows, long long bh, int box_cols, int box_rows,
              CUtensorMapSwizzle sw) {
    EncodeTiledFn enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)bh};
    cuuint64_t strides[2] = {(cuuint64_t)(cols * elem_bytes), (cuuint64_t)(cols * rows * elem_bytes)};
    cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return false;
    }
    return true;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(int B, int H, int N, int d, float scale, int dtype) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    const long long bh = (long long)B * H;
    if (bh >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
    if (bh * (long long)N * d > FA_MAX_ELEMENTS) return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

// Launches `kern` on `st` with programmatic stream serialization: the kernel may begin
// while the previous kernel in the stream finishes; it calls pdl_wait() before it reads
// anything that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <typename K>
cudaError_t set_smem(K kern, int bytes, std::atomic<int> *done, int dev) {
    if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev].store(1, std::memory_order_relaxed);
    return e;
}

// ---------------------------------------------------------------- static schedules

// Assigns work items 0 .. n-1 with estimated costs `cost` to `lists` persistent CTAs so
// that the largest list total is small: longest first onto the least loaded list (LPT),
// then, while it lowers the largest total, moves of an item out of the fullest list and
// swaps of an item of the fullest list with a smaller one of another list.  Each list is
// then walked heaviest item first.  Deterministic for given inputs.
bool balance_items(const std::vector<float> &cost, int lists, fa::ItemSchedule &s) {
    const int n = (int)cost.size();
    if (lists < 1 || lists > fa::kSchedMaxLists || n < 1 || n > fa::kSchedMaxItems) return false;
    std::vector<int> order(n);
    for (int i = 0; i < n; ++i) order[i] = i;
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
    std::vector<std::vector<int>> bins(lists);
    std::vector<double> load(lists, 0.0);
    for (int i : order) {
        int best = 0;
        for (int c = 1; c < lists; ++c)
            if (load[c] < load[best]) best = c;
        bins[best].push_back(i);
        load[best] += cost[i];
    }
    // (few items per list: there LPT can leave the largest total well above the mean)
    const int max_iter = (n <= 8 * lists) ? 4 * n : 0;
    for (int iter = 0; iter < max_iter; ++iter) {
        int hi = 0;
        for (int c = 1; c < lists; ++c)
            if (load[c] > load[hi]) hi = c;
        bool improved = false;
        // move: an item of the fullest list to a list that stays below the current maximum
        for (size_t a = 0; a < bins[hi].size() && !improved; ++a) {
            const float x = cost[bins[hi][a]];
            for (int c = 0; c < lists && !improved; ++c)
                if (c != hi && load[c] + x < load[hi] - 1e-6) {
                    bins[c].push_back(bins[hi][a]);
                    bins[hi].erase(bins[hi].begin() + a);
                    load[c] += x;
                    load[hi] -= x;
                    improved = true;
                }
        }
        // swap: an item of the fullest list with a smaller one elsewhere
        for (size_t a = 0; a < bins[hi].size() && !improved; ++a) {
            const float x = cost[bins[hi][a]];
            for (int c = 0; c < lists && !improved; ++c) {
                if (c == hi) continue;
                for (size_t b = 0; b < bins[c].size(); ++b) {
                    const float y = cost[bins[c][b]];
                    if (y < x && load[c] - y + x < load[hi] - 1e-6) {
                        std::swap(bins[hi][a], bins[c][b]);
                        load[hi] += y - x;
                        load[c] += x - y;
                        improved = true;
                        break;
                    }
                }
            }
        }
        if (!improved) break;
    }
    s.lists = lists;
    int k = 0;
    for (int c = 0; c < lists; ++c) {
        std::stable_sort(bins[c].begin(), bins[c].end(), [&](int a, int b) { return cost[a] > cost[b]; });
        s.off[c] = (uint16_t)k;
        for (int i : bins[c]) s.ids[k++] = (uint16_t)i;
    }
    s.off[lists] = (uint16_t)k;
    return true;
}

// Schedules by problem shape, computed once per shape and kept for the process.
std::mutex g_sched_mu;
std::map<std::vector<long long>, fa::ItemSchedule> g_sched;

// The schedule of a shape (lists = 0 when none applies), computed on first use from the
// items' estimated costs.
fa::ItemSchedule schedule_for(const std::vector<long long> &key, const std::vector<float> &cost,
                              int lists) {
    std::lock_guard<std::mutex> lock(g_sched_mu);
    auto f = g_sched.find(key);
    if (f != g_sched.end()) return f->second;
    fa::ItemSchedule s;
    std::memset(&s, 0, sizeof(s));
    if (!balance_items(cost, lists, s)) s.lists = 0;
    if (g_sched.size() > 256) g_sched.clear();  // bounded cache
    g_sched.emplace(key, s);
    return s;
}

fa::ItemSchedule no_schedule() {
    fa::ItemSchedule s;
    std::memset(&s, 0, sizeof(s));
    return s;
}

// Split-KV output of one launch: fp32 partial outputs and LSEs (see FwdParams).
struct SplitOut {
    float *part_o = nullptr;
    float *part_lse = nullptr;
    int num_splits = 1;
    int blocks_per_split = 0;
};

template <int D, bool BF16, bool DROP, bool SPLIT, bool F8 = false>
int launch_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
               int N, int Nk, float scale, int causal, const int *kv_len, const uint8_t *bmask,
               int mask_per_head, const fa::DropoutParams &drop, const SplitOut &so,
               cudaStream_t st, int dev, float out_scale = 1.f) {
    using C = std::conditional_t<F8, fa::FwdCfgF8, fa::FwdCfg<D>>;
    const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    // inputs: 16-bit with 64-element (128-byte) boxes, or E4M3 bytes with 128-element boxes
    const CUtensorMapDataType dti = F8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : dt;
    const int ie = F8 ? 1 : 2, ib = F8 ? 128 : 64;
    const long long bh = (long long)B * H;
    CUtensorMap mq, mk, mv;  // O is written from registers (or, split-KV, by the combine)
    if (!make_map(&mq, q, dti, ie, D, N, bh, ib, C::BM, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, k, dti, ie, D, Nk, bh, ib, C::BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, v, dti, ie, D, Nk, bh, ib, C::BN, CU_TENSOR_MAP_SWIZZLE_128B))
        return FA_ERR_CUDA;
    fa::FwdParams p;
    p.o = o;
    p.lse = lse;
    p.kv_len = kv_len;
    p.part_o = so.part_o;
    p.part_lse = so.part_lse;
    p.num_splits = so.num_splits;
    p.kv_blocks_per_split = so.blocks_per_split;
    p.Nk = Nk;
    p.causal_off = Nk - N;
    p.bmask = bmask;
    p.bmask_T = (N + 127) / 128;
    p.bmask_bh_stride = mask_per_head ? (long long)p.bmask_T * p.bmask_T : 0;
    p.N = N;
    p.BH = (int)bh;
    p.H = H;
    p.num_q_tiles = (N + C::BM - 1) / C::BM;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.drop = drop;
    p.out_scale = out_scale;
    // (a scheduled instance exists for the d = 64 forward without key splits only)
    constexpr bool kCanSched = (D == 64 && !SPLIT && !F8);
    auto kern = fa::fa_fwd_kernel<D, BF16, DROP, SPLIT, F8, false>;
    static std::atomic<int> smem_done[2][kMaxDevices];
    cudaError_t e = set_smem(kern, C::SMEM, smem_done[0], dev);
    if constexpr (kCanSched)
        if (e == cudaSuccess)
            e = set_smem(fa::fa_fwd_kernel<D, BF16, DROP, SPLIT, F8, true>, C::SMEM, smem_done[1], dev);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaFuncSetAttribute(fwd)");
        return FA_ERR_CUDA;
    }
    // Persistent: up to CTAS_PER_SM CTAs per SM walk the (query tile, split, head) items.
    const long long items = (long long)p.num_q_tiles * so.num_splits * bh;
    if (items >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    const long long grid = std::min<long long>(items, (long long)C::CTAS_PER_SM * sms);
    // Causal shapes (no key lengths or block mask) with several items per CTA: a balanced
    // static assignment.  Item u is (query tile, head) as the kernel numbers it; its cost
    // is its key blocks plus a per-item overhead (the epilogue and the next item's first
    // scores: about 1.8 blocks of 64 keys at d = 64, measured on B200; half that for
    // 128-key blocks).  Without the causal mask every item costs the same and the zigzag
    // is already balanced.
    fa::ItemSchedule sched = no_schedule();
    if (kCanSched && causal && kv_len == nullptr && bmask == nullptr && items > grid &&
        items <= fa::kSchedMaxItems) {
        std::vector<float> cost((size_t)items);
        for (long long u = 0; u < items; ++u) {
            const int rank = (int)(u / bh);
            const int qt = causal ? p.num_q_tiles - 1 - rank : rank;
            long long kv_end = Nk;
            if (causal) kv_end = std::min<long long>(kv_end, (long long)(qt + 1) * C::BM + p.causal_off);
            const long long T = kv_end > 0 ? (kv_end + C::BN - 1) / C::BN : 0;
            cost[(size_t)u] = (float)T + (C::BN == 64 ? 1.8f : 0.9f);
        }
        sched = schedule_for({0, D, N, Nk, bh, causal ? 1 : 0, grid}, cost, (int)grid);
    }
    timing_mark(0, 0, st);
    if constexpr (kCanSched) {
        if (sched.lists > 0)
            e = launch_pdl(fa::fa_fwd_kernel<D, BF16, DROP, SPLIT, F8, true>, dim3((unsigned)grid),
                           dim3(C::THREADS), C::SMEM, st, mq, mk, mv, p, sched);
        else
            e = launch_pdl(kern, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, st, mq, mk, mv, p,
                           fa::NoSchedule{0});
    } else {
        e = launch_pdl(kern, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, st, mq, mk, mv, p,
                       fa::NoSchedule{0});
    }
    if (e == cudaSuccess) e = cudaGetLastError();
    timing_mark(0, 1, st);
    if (e != cudaSuccess) {
        record_cuda_error(e, "fa_fwd launch");
        return FA_ERR_CUDA;
    }
    return FA_OK;
}


struct BwdWorkspace {
    float *dq_acc;
    float *nlse2;
    float *ndvec;
    size_t total;
};

size_t round256(size_t x) { return (x + 255) & ~(size_t)255; }

BwdWorkspace bwd_workspace_layout(void *base, long long BH, int N, int d) {
    const int npad = ((N + 127) / 128) * 128;
    const size_t dq = round256((size_t)BH * N * d * 4);
    const size_t vec = round256((size_t)BH * npad * 4);
    BwdWorkspace w;
    char *b = static_cast<char *>(base);
    w.dq_acc = reinterpret_cast<float *>(b);
    w.nlse2 = reinterpret_cast<float *>(b + dq);
    w.ndvec = reinterpret_cast<float *>(b + dq + vec);
    w.total = dq + 2 * vec;
    return w;
}

int grid_for(long long work, int threads) {
    long long g = (work + threads - 1) / threads;
    if (g < 1) g = 1;
    if (g > 148LL * 16) g = 148LL * 16;
    return (int)g;
}

template <int D, bool BF16, bool DROP>
int launch_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
               const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, float scale,
               int causal, const int *kv_len, const uint8_t *bmask, int mask_per_head,
               const fa::DropoutParams &drop, void *workspace, cudaStream_t st, int dev) {
    using C = fa::BwdCfg<D>;
    const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                        : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const long long bh = (long long)B * H;
    const int num_tiles = (N + 127) / 128;
    BwdWorkspace ws = bwd_workspace_layout(workspace, bh, N, D);

    CUtensorMap mq, mk, mv, mdo, mdk, mdv, mdq;
    if (!make_map(&mq, q, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, k, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, v, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mdo, dout, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mdk, dk, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mdv, dv, dt, 2, D, N, bh, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mdq, ws.dq_acc, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, N, bh, 32, 128,
                  CU_TENSOR_MAP_SWIZZLE_128B))
        return FA_ERR_CUDA;

    // 1. D = rowsum(dO o O), LSE in base 2, zeroed dQ accumulator.
    fa::BwdPrepParams pp;
    pp.o = o;
    pp.dout = dout;
    pp.lse = lse;
    pp.nlse2 = ws.nlse2;
    pp.ndvec = ws.ndvec;
    pp.dq_acc = reinterpret_cast<float4 *>(ws.dq_acc);
    pp.dq_acc_vec4 = bh * (long long)N * D / 4;
    pp.dscale = DROP ? 1.f / drop.keep_scale : 1.f;
    pp.N = N;
    pp.Npad = num_tiles * 128;
    pp.BH = bh;
    const long long prep_work = std::max(pp.dq_acc_vec4, bh * pp.Npad * (D / 8));
    cudaError_t e = launch_pdl(fa::fa_bwd_prep_kernel<D, BF16>, dim3(grid_for(prep_work, 256)),
                               dim3(256), 0, st, pp);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e, "fa_bwd prep launch");
        return FA_ERR_CUDA;
    }

    // 2. main pass
    fa::BwdParams p;
    p.nlse2 = ws.nlse2;
    p.ndvec = ws.ndvec;
    p.dq_acc = ws.dq_acc;
    p.bmask = bmask;
    p.bmask_bh_stride = mask_per_head ? (long long)num_tiles * num_tiles : 0;
    p.kv_len = kv_len;
    p.N = N;
    p.Npad = num_tiles * 128;
    p.BH = (int)bh;
    p.H = H;
    p.num_tiles = num_tiles;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.drop = drop;
    p.dv_mul = drop.keep_scale;
    p.dk_mul = scale * drop.keep_scale;
    // d = 64 without the causal mask: the two-issuer variant (BwdCfg::TWO_ISS).
    using C2 = fa::BwdCfg<D, true>;
    const bool two = (D == 64) && !causal;
    auto kern = fa::fa_bwd_kernel<D, BF16, DROP, false>;
    auto kern_s = fa::fa_bwd_kernel<D, BF16, DROP, true>;
    auto kern_2 = fa::fa_bwd_kernel<D, BF16, DROP, false, D == 64>;
    static std::atomic<int> smem_done[3][kMaxDevices];
    e = set_smem(kern, C::SMEM, smem_done[0], dev);
    if (e == cudaSuccess) e = set_smem(kern_s, C::SMEM, smem_done[1], dev);
    if (e == cudaSuccess && two) e = set_smem(kern_2, C2::SMEM, smem_done[2], dev);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaFuncSetAttribute(bwd)");
        return FA_ERR_CUDA;
    }
    // Persistent: one CTA per SM (or per work item, if fewer) walks the (key tile, head)
    // items; the kernel takes the grid size into its static schedule.
    const long long items = (long long)num_tiles * bh;
    if (items >= (1LL << 31)) return FA_ERR_UNSUPPORTED;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    const long long grid = std::min<long long>(items, sms);
    // Causal shapes (no key lengths or block mask) with several items per CTA: a balanced
    // static assignment.  Item u is (key tile, head) as the kernel numbers it; its cost is
    // the query tiles it visits plus the fixed cost of an item (its epilogue and the next
    // item's start) in units of one query tile: 1.8 at d = 64 (fitted to per-CTA end times
    // on B200: an item adds 3.1 us, a query tile 1.7 us), 0.9 at d = 128.  Without the
    // causal mask every item costs the same.
    fa::ItemSchedule sched = no_schedule();
    if (causal && kv_len == nullptr && bmask == nullptr && items > grid &&
        items <= fa::kSchedMaxItems) {
        std::vector<float> cost((size_t)items);
        for (long long u = 0; u < items; ++u) {
            const int kt = (D == 128) ? (int)(u % num_tiles) : (int)(u / bh);
            const int n = causal ? num_tiles - kt : num_tiles;
            cost[(size_t)u] = (float)n + (D == 64 ? 1.8f : 0.9f);
        }
        sched = schedule_for({1, D, N, bh, causal ? 1 : 0, grid}, cost, (int)grid);
    }
    timing_mark(1, 0, st);
    if (sched.lists > 0)
        e = launch_pdl(kern_s, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, st, mq, mk, mv,
                       mdo, mdk, mdv, mdq, p, sched);
    else if (two)
        e = launch_pdl(kern_2, dim3((unsigned)grid), dim3(C2::THREADS), C2::SMEM, st, mq, mk, mv,
                       mdo, mdk, mdv, mdq, p, fa::NoSchedule{0});
    else
        e = launch_pdl(kern, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, st, mq, mk, mv,
                       mdo, mdk, mdv, mdq, p, fa::NoSchedule{0});
    if (e == cudaSuccess) e = cudaGetLastError();
    timing_mark(1, 1, st);
    if (e != cudaSuccess) {
        record_cuda_error(e, "fa_bwd launch");
        return FA_ERR_CUDA;
    }

    // 3. dQ = scale * dQ_acc in the input dtype
    const long long nv4 = bh * (long long)N * D / 4;
    e = launch_pdl(fa::fa_bwd_convert_kernel<BF16>, dim3(grid_for(nv4, 256)), dim3(256), 0, st,
                   reinterpret_cast<const float4 *>(ws.dq_acc), reinterpret_cast<uint2 *>(dq), nv4,
                   DROP ? scale * drop.keep_scale : scale);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e, "fa_bwd convert launch");
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

// Static scratch of fa_bwd_noalloc.  In host code this name is only a stand-in for the
// device symbol: its device address is looked up with cudaGetSymbolAddress (once per
// device, with that device current) and that address is what the kernels get.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

std::atomic<void *> g_noalloc_ptr[kMaxDevices];

// Device address of g_noalloc_scratch on device `dev` (which must be current).
int noalloc_scratch(int dev, void **out) {
    void *p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            record_cuda_error(e, "cudaGetSymbolAddress(noalloc scratch)");
            return FA_ERR_CUDA;
        }
        g_noalloc_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return FA_OK;
}

// Dropout parameters of probability p_drop: the byte threshold t = rint(256 p) must lie
// in [0, 255].  Returns false for a p outside that range or not finite.
bool make_dropout(float p_drop, unsigned long long seed, unsigned int offset,
                  fa::DropoutParams *dp) {
    if (!std::isfinite(p_drop) || p_drop < 0.f) return false;
    const float tf = rintf(p_drop * 256.f);
    if (tf > 255.f) return false;
    const uint32_t t = (uint32_t)tf;
    dp->add16 = (0x8000u - t) * 0x00010001u;
    dp->seed_lo = (uint32_t)(seed & 0xFFFFFFFFull);
    dp->seed_hi = (uint32_t)(seed >> 32);
    dp->offset = offset;
    dp->keep_scale = 256.f / (float)(256u - t);
    return true;
}

const fa::DropoutParams kNoDropout = {0x8000u * 0x00010001u, 0u, 0u, 0u, 1.f};

// Key splits of the split-KV forward: `requested` (> 0) capped by the key blocks, or, for
// 0, enough splits that the grid fills about two waves of the SMs, with at least two key
// blocks per split.  Also returns the key blocks per split.
int resolve_splits(long long BH, int Nq, int Nk, int d, int requested, int sms, int *blocks_per) {
    const int BN = d == 64 ? 64 : 128;
    const int kblocks = (Nk + BN - 1) / BN;
    int splits;
    if (requested > 0) {
        splits = std::min(requested, kblocks);
    } else {
        // The split count that finishes first on a persistent grid of `slots` CTAs:
        // (query tile, split, head) items of bps key blocks each are dealt out in rounds
        // of `slots`; a round costs its blocks plus about two blocks' worth of per-item
        // work (the Q tile, the fp32 partial output).  Splits of fewer than two blocks,
        // and more than 128 splits, are not considered.
        const long long tiles = (long long)((Nq + 127) / 128) * BH;
        const long long slots = (long long)sms * (d == 64 ? 2 : 1);
        const int max_s = std::max(1, std::min(128, kblocks / 2));
        long long best = -1;
        splits = 1;
        for (int sp = 1; sp <= max_s; ++sp) {
            const int b = (kblocks + sp - 1) / sp;
            const long long items = tiles * ((kblocks + b - 1) / b);
            const long long cost = ((items + slots - 1) / slots) * (b + 2);
            if (best < 0 || cost < best) {
                best = cost;
                splits = sp;
            }
        }
    }
    const int bps = (kblocks + splits - 1) / splits;
    *blocks_per = bps;
    return (kblocks + bps - 1) / bps;
}

int current_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        return 148;
    return sms;
}

size_t splitkv_bytes(long long BH, int Nq, int d, int splits) {
    if (splits <= 1) return 0;
    return round256((size_t)splits * BH * Nq * d * 4) + round256((size_t)splits * BH * Nq * 4);
}

template <int D, bool BF16>
int launch_splitkv(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                   int Nq, int Nk, float scale, int causal, const int *kv_len, int splits, int bps,
                   void *workspace, cudaStream_t st, int dev) {
    if (splits <= 1) {
        const SplitOut whole;
        return launch_fwd<D, BF16, false, false>(q, k, v, o, lse, B, H, Nq, Nk, scale, causal,
                                                 kv_len, nullptr, 0, kNoDropout, whole, st, dev);
    }
    const long long bh = (long long)B * H;
    SplitOut so;
    so.part_o = static_cast<float *>(workspace);
    so.part_lse = reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                            round256((size_t)splits * bh * Nq * D * 4));
    so.num_splits = splits;
    so.blocks_per_split = bps;
    int rc = launch_fwd<D, BF16, false, true>(q, k, v, o, lse, B, H, Nq, Nk, scale, causal, kv_len,
                                              nullptr, 0, kNoDropout, so, st, dev);
    if (rc != FA_OK) return rc;
    const long long rows = bh * Nq;
    cudaError_t e = launch_pdl(fa::fa_splitkv_combine_kernel<D, BF16>,
                               dim3(grid_for(rows * (D / 4), 256)), dim3(256), 0, st,
                               (const float *)so.part_o, (const float *)so.part_lse, o, lse, rows,
                               splits);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e, "split-KV combine launch");
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return kVersion; }

int fa_schedule_items(const float *cost, int n, int lists, unsigned short *off,
                      unsigned short *ids) {
    if (cost == nullptr || off == nullptr || ids == nullptr) return FA_ERR_INVALID_ARG;
    if (n < 1 || n > fa::kSchedMaxItems || lists < 1 || lists > fa::kSchedMaxLists)
        return FA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!(cost[i] > 0.f) || !std::isfinite(cost[i])) return FA_ERR_INVALID_ARG;
    std::vector<float> c(cost, cost + n);
    fa::ItemSchedule s;
    std::memset(&s, 0, sizeof(s));
    if (!balance_items(c, lists, s)) return FA_ERR_INVALID_ARG;
    for (int i = 0; i <= lists; ++i) off[i] = s.off[i];
    for (int i = 0; i < n; ++i) ids[i] = s.ids[i];
    return FA_OK;
}

int fa_set_timing_events(int which, void *start, void *stop) {
    if (which < 0 || which > 1) return FA_ERR_INVALID_ARG;
    if ((start == nullptr) != (stop == nullptr)) return FA_ERR_INVALID_ARG;
    t_timing[which][0] = reinterpret_cast<cudaEvent_t>(start);
    t_timing[which][1] = reinterpret_cast<cudaEvent_t>(stop);
    return FA_OK;
}

const char *fa_strerror(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported configuration or device";
        case FA_ERR_CUDA: return "CUDA error";
        case FA_ERR_TIMEOUT: return "device-side wait timed out";
        case FA_ERR_SCRATCH_LIMIT: return "problem needs more scratch than fa_bwd_noalloc's static buffer";
        default: return "unknown status";
    }
}

const char *fa_last_cuda_error(void) { return t_last_error; }


static int fwd_common(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                      int H, int N, int d, float scale, int causal, const int *kv_len,
                      const uint8_t *bmask, int mask_per_head, const fa::DropoutParams *drop,
                      int dtype, void *stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID_ARG;
    int rc = check_common(B, H, N, d, scale, dtype);
    if (rc != FA_OK) return rc;
    int dev = 0;
    rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
#define FA_FWD_ARGS q, k, v, o, lse, B, H, N, N, scale, causal, kv_len, bmask, mask_per_head
    const SplitOut whole;
    if (drop) {
        if (d == 64)
            return bf16 ? launch_fwd<64, true, true, false>(FA_FWD_ARGS, *drop, whole, st, dev)
                        : launch_fwd<64, false, true, false>(FA_FWD_ARGS, *drop, whole, st, dev);
        return bf16 ? launch_fwd<128, true, true, false>(FA_FWD_ARGS, *drop, whole, st, dev)
                    : launch_fwd<128, false, true, false>(FA_FWD_ARGS, *drop, whole, st, dev);
    }
    if (d == 64)
        return bf16 ? launch_fwd<64, true, false, false>(FA_FWD_ARGS, kNoDropout, whole, st, dev)
                    : launch_fwd<64, false, false, false>(FA_FWD_ARGS, kNoDropout, whole, st, dev);
    return bf16 ? launch_fwd<128, true, false, false>(FA_FWD_ARGS, kNoDropout, whole, st, dev)
                : launch_fwd<128, false, false, false>(FA_FWD_ARGS, kNoDropout, whole, st, dev);
#undef FA_FWD_ARGS
}

int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N,
           int d, float scale, int causal, const int *kv_len, int dtype, void *stream) {
    return fwd_common(q, k, v, o, lse, B, H, N, d, scale, causal, kv_len, nullptr, 0, nullptr,
                      dtype, stream);
}

int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                       int H, int N, int d, float scale, int causal, const int *kv_len,
                       const unsigned char *block_mask, int mask_per_head, int dtype,
                       void *stream) {
    if (!block_mask || (mask_per_head != 0 && mask_per_head != 1)) return FA_ERR_INVALID_ARG;
    return fwd_common(q, k, v, o, lse, B, H, N, d, scale, causal, kv_len, block_mask,
                      mask_per_head, nullptr, dtype, stream);
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || (d != 64 && d != 128) || num_splits < 0 ||
        num_splits > FA_MAX_SPLITS)
        return 0;
    int bps = 0;
    const long long bh = (long long)B * H;
    const int splits = resolve_splits(bh, Nq, Nk, d, num_splits, current_sms(), &bps);
    return splitkv_bytes(bh, Nq, d, splits);
}

int fa_fwd_splitkv(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
                   int Nq, int Nk, int d, float scale, int causal, const int *kv_len,
                   int num_splits, int dtype, void *workspace, size_t workspace_bytes,
                   void *stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID_ARG;
    if (num_splits < 0 || num_splits > FA_MAX_SPLITS || Nk < 1) return FA_ERR_INVALID_ARG;
    int rc = check_common(B, H, Nq, d, scale, dtype);
    if (rc != FA_OK) return rc;
    if ((long long)B * H * (long long)Nk * d > FA_MAX_ELEMENTS) return FA_ERR_UNSUPPORTED;
    int dev = 0;
    rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    int bps = 0;
    const long long bh = (long long)B * H;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
        sms = 148;
    const int splits = resolve_splits(bh, Nq, Nk, d, num_splits, sms, &bps);
    const size_t need = splitkv_bytes(bh, Nq, d, splits);
    if (need > 0 && (!workspace || workspace_bytes < need ||
                     (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
        return FA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
#define FA_SPLIT_ARGS q, k, v, o, lse, B, H, Nq, Nk, scale, causal, kv_len, splits, bps, workspace, st, dev
    if (d == 64)
        return bf16 ? launch_splitkv<64, true>(FA_SPLIT_ARGS) : launch_splitkv<64, false>(FA_SPLIT_ARGS);
    return bf16 ? launch_splitkv<128, true>(FA_SPLIT_ARGS) : launch_splitkv<128, false>(FA_SPLIT_ARGS);
#undef FA_SPLIT_ARGS
}

int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
               int N, int d, float scale, int causal, const int *kv_len, float q_scale,
               float k_scale, float v_scale, void *stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_INVALID_ARG;
    if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID_ARG;
    for (float f : {q_scale, k_scale, v_scale})
        if (!std::isfinite(f) || !(f > 0.f)) return FA_ERR_INVALID_ARG;
    int rc = check_common(B, H, N, d, scale, FA_BF16);
    if (rc != FA_OK) return rc;
    if (d != 128) return FA_ERR_UNSUPPORTED;
    int dev = 0;
    rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    const SplitOut whole;
    // the scores see q_scale * k_scale through the softmax scale; V's scale multiplies O
    return launch_fwd<128, true, false, false, true>(
        q, k, v, o, lse, B, H, N, N, scale * q_scale * k_scale, causal, kv_len, nullptr, 0,
        kNoDropout, whole, reinterpret_cast<cudaStream_t>(stream), dev, v_scale);
}

int fa_fwd_dropout(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                   int H, int N, int d, float scale, int causal, const int *kv_len, float p_drop,
                   unsigned long long seed, unsigned int offset, int dtype, void *stream) {
    fa::DropoutParams dp;
    if (!make_dropout(p_drop, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
    return fwd_common(q, k, v, o, lse, B, H, N, d, scale, causal, kv_len, nullptr, 0, &dp, dtype,
                      stream);
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
    return bwd_workspace_layout(nullptr, (long long)B * H, N, d).total;
}

static int bwd_common(const void *q, const void *k, const void *v, const void *o,
                      const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                      int H, int N, int d, float scale, int causal, const int *kv_len,
                      const uint8_t *bmask, int mask_per_head, const fa::DropoutParams *drop,
                      int dtype, void *workspace, size_t workspace_bytes, void *stream) {
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace)
        return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
    if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID_ARG;
    int rc = check_common(B, H, N, d, scale, dtype);
    if (rc != FA_OK) return rc;
    if (workspace_bytes < fa_bwd_workspace_bytes(B, H, N, d)) return FA_ERR_INVALID_ARG;
    int dev = 0;
    rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
#define FA_BWD_ARGS q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, causal, kv_len, bmask, mask_per_head
    if (drop) {
        if (d == 64)
            return bf16 ? launch_bwd<64, true, true>(FA_BWD_ARGS, *drop, workspace, st, dev)
                        : launch_bwd<64, false, true>(FA_BWD_ARGS, *drop, workspace, st, dev);
        return bf16 ? launch_bwd<128, true, true>(FA_BWD_ARGS, *drop, workspace, st, dev)
                    : launch_bwd<128, false, true>(FA_BWD_ARGS, *drop, workspace, st, dev);
    }
    if (d == 64)
        return bf16 ? launch_bwd<64, true, false>(FA_BWD_ARGS, kNoDropout, workspace, st, dev)
                    : launch_bwd<64, false, false>(FA_BWD_ARGS, kNoDropout, workspace, st, dev);
    return bf16 ? launch_bwd<128, true, false>(FA_BWD_ARGS, kNoDropout, workspace, st, dev)
                : launch_bwd<128, false, false>(FA_BWD_ARGS, kNoDropout, workspace, st, dev);
#undef FA_BWD_ARGS
}

int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout,
           const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
           float scale, int causal, const int *kv_len, int dtype, void *workspace,
           size_t workspace_bytes, void *stream) {
    return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, kv_len,
                      nullptr, 0, nullptr, dtype, workspace, workspace_bytes, stream);
}

int fa_bwd_dropout(const void *q, const void *k, const void *v, const void *o, const void *dout,
                   const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                   float scale, int causal, const int *kv_len, float p_drop,
                   unsigned long long seed, unsigned int offset, int dtype, void *workspace,
                   size_t workspace_bytes, void *stream) {
    fa::DropoutParams dp;
    if (!make_dropout(p_drop, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
    return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, kv_len,
                      nullptr, 0, &dp, dtype, workspace, workspace_bytes, stream);
}

int fa_dropout_mask(int B, int H, int N, float p_drop, unsigned long long seed,
                    unsigned int offset, unsigned char *keep, void *stream) {
    if (!keep || B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    fa::DropoutParams dp;
    if (!make_dropout(p_drop, seed, offset, &dp)) return FA_ERR_INVALID_ARG;
    const long long bh = (long long)B * H;
    if ((double)bh * N * N > (double)FA_MAX_ELEMENTS) return FA_ERR_INVALID_ARG;
    int dev = 0;
    int rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    const long long work = bh * N * ((N + 15) / 16);
    fa::dropout_mask_kernel<<<grid_for(work, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        keep, bh, N, dp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e, "fa_dropout_mask launch");
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o,
                       const void *dout, const float *lse, void *dq, void *dk, void *dv, int B,
                       int H, int N, int d, float scale, int causal, const int *kv_len,
                       const unsigned char *block_mask, int mask_per_head, int dtype,
                       void *workspace, size_t workspace_bytes, void *stream) {
    if (!block_mask || (mask_per_head != 0 && mask_per_head != 1)) return FA_ERR_INVALID_ARG;
    return bwd_common(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, kv_len,
                      block_mask, mask_per_head, nullptr, dtype, workspace, workspace_bytes, stream);
}

int fa_selftest_wait_timeout(int limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 2000000) return FA_ERR_INVALID_ARG;
    int dev = 0;
    int rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    fa::wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)limit_us * 1000ull);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e, "selftest launch");
        return FA_ERR_CUDA;
    }
    return FA_OK;
}

int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const void *dout,
                   const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                   float scale, int causal, const int *kv_len, int dtype, void *stream) {
    if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
        !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
        return FA_ERR_INVALID_ARG;
    if (kv_len && (reinterpret_cast<uintptr_t>(kv_len) & 3u)) return FA_ERR_INVALID_ARG;
    int rc = check_common(B, H, N, d, scale, dtype);
    if (rc != FA_OK) return rc;
    if (fa_bwd_workspace_bytes(B, H, N, d) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
    int dev = 0;
    rc = check_device(&dev);
    if (rc != FA_OK) return rc;
    void *workspace = nullptr;
    rc = noalloc_scratch(dev, &workspace);
    if (rc != FA_OK) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const bool bf16 = dtype == FA_BF16;
#define FA_BWD_ARGS q, k, v, o, dout, lse, dq, dk, dv, B, H, N, scale, causal, kv_len, nullptr, 0, kNoDropout, workspace, st, dev
    if (d == 64)
        return bf16 ? launch_bwd<64, true, false>(FA_BWD_ARGS)
                    : launch_bwd<64, false, false>(FA_BWD_ARGS);
    return bf16 ? launch_bwd<128, true, false>(FA_BWD_ARGS)
                : launch_bwd<128, false, false>(FA_BWD_ARGS);
#undef FA_BWD_ARGS
}

int fa_get_device_status(void *stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) {
        record_cuda_error(e, "cudaStreamSynchronize");
        return FA_ERR_CUDA;
    }
    int val = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&val, fa::g_status, sizeof(int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) {
        record_cuda_error(e, "status word");
        return FA_ERR_CUDA;
    }
    return val == 0 ? FA_OK : FA_ERR_TIMEOUT;
}

}  // extern "C"
