// rkv_internal.h -- host-side declarations shared by the C-ABI layer and the
// kernel launchers.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "../../include/rkv.h"

namespace rkv {

// An NVTX range around one entry point (host side): profilers that record NVTX
// show each call of the library as a named span over the kernels it enqueues.
// Header-only NVTX: without an attached tool a push / pop costs a few ns.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

constexpr int kHeadDim = 128;
constexpr int kMaxLayersPerLaunch = 32;
constexpr int kMaxQCols = 64;          // G * window supported by the fused kernel
constexpr size_t kStatusBytes = 256;   // workspace header: status word and spare

// Flags of the fused per-unit kernel.
enum : int32_t {
    kFlagImportance = 1,   // compute importance (needs Q)
    kFlagSelect = 2,       // select + compact in place (the compression step)
    kFlagOutScores = 4,    // write I / inv_norm / r / R outputs (per-head entry points)
};

struct alignas(64) StepParams {
    CUtensorMap tmap_k[kMaxLayersPerLaunch];   // [B*Hkv*cap rows, 128] bf16, box 64x16, SW128
    CUtensorMap tmap_q[kMaxLayersPerLaunch];   // [B*Hq*w rows, 128] bf16, box 64xNQP, SW128
    uint16_t *k[kMaxLayersPerLaunch];          // cache bases for the in-place writes
    uint16_t *v[kMaxLayersPerLaunch];
    int32_t n_layers, layer_base, batch, n_kv, group, window, cap;
    int32_t cs;            // CTAs per unit (cluster size)
    int32_t rmax;          // rows per CTA the shared-memory layout holds
    int32_t rp;            // rows allocated per K half (>= max(rmax, 128), multiple of 16)
    int32_t tmem_cols;     // TMEM columns allocated per CTA
    int32_t n_tokens_fixed;  // > 0: per-head entry points, N fixed and every unit due
    int32_t budget_cfg;
    float lambda_cfg;
    float logit_scale_log2;  // log2(e) / sqrt(D)
    int32_t red_mode, gqa_pool, flags;
    const int32_t *budgets;  // device [batch] or null
    const float *lambdas;    // device [batch] or null
    const int32_t *n_eff;    // device [batch]: N of due sequences, 0 otherwise (plan kernel)
    const float *r_ext;      // MAX mode: raw r [units][cap] from the similarity kernel, or null
    int32_t *kept_out;       // optional [units][cap]
    float *scores_out;       // optional [units][4][cap]
    float *out_I, *out_inv, *out_r, *out_R;  // per-head outputs ([Hkv][M] / [Hkv][N])
    uint32_t *status;
};

constexpr int kStepThreads = 256;     // threads per CTA of the fused kernel

struct SmemLayout {
    uint32_t k, xstatm, xstatl, xs, hist, v, x, q, scratch, inv, ss, ihat, rr, dst, xp, gs, spart,
        gm, glinv, vis, red, misc, bars, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) {
    return (x + a - 1) / a * a;
}

// Offsets from a 1024-byte-aligned base; `total` includes 1024 bytes of slack
// for aligning the dynamic shared-memory pointer.  Regions whose names start
// with x are written by the other CTAs of the cluster (one slot per CTA).
// Lifetimes let regions share bytes:
//  * the select histograms (after barrier 2) reuse the barrier-1 exchange slots;
//  * region `x` first holds the query tile and the reduction scratch (both dead
//    before this CTA reaches barrier 1), then the (Ihat, r) pairs that the
//    cluster pushes after barrier 1, then, in place, the select keys.
__host__ __device__ inline SmemLayout make_layout(int rp, int rmax, int cap, int nqp, int cs) {
    SmemLayout L;
    uint32_t o = 0;
    L.k = o;      o += 2u * rp * 128u;                 // K rows, two 64-column swizzled halves
    const uint32_t u0 = o;
    L.xstatm = o; o += cs * nqp * 4u;                  // column max of every CTA
    L.xstatl = o; o += cs * nqp * 4u;                  // column sum of exp of every CTA
    L.xs = o;     o += cs * 128u * 4u;                 // S partial of every CTA
    L.hist = u0;                                       // 8 warps x 256 bins
    if (o - u0 < 8u * 256u * 4u) o = u0 + 8u * 256u * 4u;
    o = align_up(o, 1024);
    L.v = o;      o += static_cast<uint32_t>(rmax) * 256u;   // V rows, plain row-major
    o = align_up(o, 1024);
    L.x = o;
    L.q = o;                                           // window queries (swizzled, 1024-aligned)
    L.scratch = o + 2u * nqp * 128u;                   // 8 x 128 + 8 x nqp floats
    const uint32_t xbytes = cap * 8u;
    const uint32_t early = 2u * nqp * 128u + 8u * 128u * 4u + 8u * nqp * 4u;
    o += align_up(xbytes > early ? xbytes : early, 16);
    L.inv = o;    o += align_up(rmax * 4u, 16);
    L.ss = o;     o += align_up(rmax * 4u, 16);
    L.ihat = o;   o += align_up(rmax * 4u, 16);
    L.rr = o;     o += align_up(rmax * 4u, 16);
    L.dst = o;    o += align_up(rmax * 4u, 16);
    L.xp = o;     o += cs * 16u;                       // (sum Ihat, max r, sum exp r) of every CTA
    L.gs = o;     o += 128u * 4u;
    L.spart = o;  o += 128u * 4u;
    L.gm = o;     o += nqp * 4u;
    L.glinv = o;  o += nqp * 4u;
    L.vis = o;    o += 64u * 8u;
    L.red = o;    o += 64u * 4u;
    L.misc = o;   o += 64u * 4u;
    L.bars = o;   o += 64u;
    L.total = o + 1024u;
    return L;
}

// Launches `kernel` and returns that launch's own status.  (A <<< >>> launch has to be
// checked with cudaGetLastError, which would also report an error some unrelated
// earlier call of the caller left behind.)
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t stream, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit only when a launch needs more
// than any earlier one (so repeated and graph-captured launches make no
// attribute calls).  Per process; the value only grows.
template <class K>
inline cudaError_t ensure_smem_attr(K kernel, size_t bytes, std::atomic<int> &granted) {
    if (static_cast<int>(bytes) <= granted.load(std::memory_order_relaxed)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(bytes));
    if (e == cudaSuccess) {
        int cur = granted.load(std::memory_order_relaxed);
        while (cur < static_cast<int>(bytes) &&
               !granted.compare_exchange_weak(cur, static_cast<int>(bytes))) {
        }
    }
    return e;
}

// Caches with per-sequence capacities: each layer's K (and V) is one pool of
// pool_rows rows of 128 bf16, and sequence b's [Hkv][seq_cap[b]] block starts at
// row seq_row[b].  seq_row == null: the uniform [batch][Hkv][cap] layout.
struct RaggedLayout {
    const int64_t *seq_row = nullptr;   // device [batch]
    const int32_t *seq_cap = nullptr;   // device [batch]
    int64_t pool_rows = 0;
    int32_t n_kv = 0;
};

// First row of unit (b, h) in its layer's 2-D [rows, 128] view.
__device__ __forceinline__ int64_t unit_first_row(const int64_t *seq_row, const int32_t *seq_cap,
                                                  int b, int h, int n_kv, int cap) {
    return seq_row ? seq_row[b] + static_cast<int64_t>(h) * seq_cap[b]
                   : (static_cast<int64_t>(b) * n_kv + h) * cap;
}

// Launchers (defined in the .cu files); all return cudaSuccess or the launch error.
// cap: the uniform capacity, or with a ragged layout the largest seq_cap allowed.
cudaError_t launch_plan(int batch, const int32_t *budgets, int32_t budget_cfg, int32_t buffer,
                        int32_t window, int32_t cap, int32_t *cur_len, int32_t *n_eff,
                        uint32_t *status, cudaStream_t stream, bool update = true,
                        const RaggedLayout &rg = RaggedLayout{}, int32_t *order = nullptr);

// Unit `pos` of a launch over `n_layers` layers x `batch` sequences x `n_kv` heads, in
// the launch's order: by default layer-major (l, b, h); with `order` (the plan kernel's
// sequences by decreasing length) sequence-major (rank, l, h), so that the units of the
// longest sequences start first and a launch of many units ends on short ones.
struct UnitCoord {
    int l, b, h;
};
__host__ __device__ inline UnitCoord unit_coord(int pos, int n_kv, int batch, int n_layers,
                                                const int32_t *order) {
    UnitCoord c;
    c.h = pos % n_kv;
    if (order == nullptr) {
        c.b = (pos / n_kv) % batch;
        c.l = pos / (n_kv * batch);
    } else {
        c.l = (pos / n_kv) % n_layers;
        c.b = order[pos / (n_kv * n_layers)];
    }
    return c;
}
cudaError_t launch_step(const StepParams &p, int n_units, int nqp, size_t smem,
                        cudaStream_t stream);
size_t step_smem_bytes(int rp, int rmax, int cap, int nqp, int cs);
cudaError_t launch_select(const float *I, const float *R, int n_kv, int M, int N, int budget,
                          float lambda, int32_t *kept, float *Z, uint32_t *status,
                          cudaStream_t stream);
cudaError_t launch_compact(const uint16_t *k_src, const uint16_t *v_src, const int32_t *kept,
                           uint16_t *k_dst, uint16_t *v_dst, int64_t head_stride, int n_kv,
                           int budget, int n_tokens, bool in_place, int cs, uint32_t *status,
                           cudaStream_t stream);
int compact_in_place_cluster(int budget);   // 0: too large for the staged in-place path

// One-CTA-per-unit kernel (rkv_unit.cu): the whole (sequence, layer, KV head)
// in one CTA, K streamed through a two-stage TMA ring twice (HBM, then L2).
struct alignas(64) UnitParams {
    CUtensorMap tmap_k[kMaxLayersPerLaunch];   // [B*Hkv*cap rows, 128] bf16, box 64 x 128, SW128
    CUtensorMap tmap_q[kMaxLayersPerLaunch];   // [B*Hq*w rows, 128] bf16, box 64 x NQP, SW128
    uint16_t *k[kMaxLayersPerLaunch];
    uint16_t *v[kMaxLayersPerLaunch];
    int32_t layer_base, batch, n_kv, group, window, cap;
    int32_t nmax;          // rows the per-row arrays hold (= cap)
    int32_t tmem_cols;
    int32_t budget_cfg;
    float lambda_cfg;
    float logit_scale_log2;
    int32_t red_mode, gqa_pool;
    const int32_t *budgets;
    const float *lambdas;
    const int32_t *n_eff;
    const int32_t *order;  // sequences by decreasing length (plan kernel), or null: launch order
    const float *r_ext;
    int32_t *kept_out;
    float *scores_out;
    float *z_heads;        // shared selection: Z of every candidate [units][cap]; then no
                           // select, no compaction
    // paged caches: k / v are page pools [pages][Hkv][page_rows][128], tmap_k boxes are
    // one page; logical row i of sequence b is in page block_table[b][i / page_rows]
    const int32_t *block_table;   // [batch][max_blocks] or null (contiguous caches)
    int32_t max_blocks, page_rows;
    // per-sequence capacities (null: uniform [batch][Hkv][cap]; cap is then the largest)
    const int64_t *seq_row;
    const int32_t *seq_cap;
    uint32_t *status;
};

constexpr int kUnitThreads = 256;
constexpr int kUnitMaxPages = 512;     // pages of one sequence staged in shared memory
constexpr int kUnitMaxRows = 7680;     // keys + destinations + histograms fit the 64 KB ring

struct UnitLayout {
    uint32_t stage, b, bs, ss, ihat, r, scr, s, colm, colf, vis, red, bt, bars, total;
};

// Offsets from a 1024-byte-aligned base.  Lifetimes share bytes: the two 32 KB
// ring stages hold, after the last tile, the select keys, the destinations and
// the histograms; the B operand of the S UMMA (pass 1) shares bytes with the
// pass-2 arrays Ihat and r (the last S UMMA completes between the passes).  Per
// row only ||k||^2 crosses from pass 1 to pass 2 (the inverse norm is recomputed
// from it), and the two warpgroups' importance partials meet in one array, so
// that caches of up to about 2500 rows still fit two CTAs on an SM.
__host__ __device__ inline UnitLayout make_unit_layout(int nmax, int nqp) {
    UnitLayout L;
    uint32_t o = 0;
    L.stage = o;  o += 2u * 32768u;
    L.b = o;      o += 2u * (nqp + 16u) * 128u;        // queries + split S, two swizzled halves
    const uint32_t arr = align_up(static_cast<uint32_t>(nmax) * 4u, 16);
    L.ss = o;     o += arr;
    o = align_up(o, 1024);
    L.bs = o;                                          // pass 1: inv split, 2 x 4 KB
    L.ihat = o;                                        // pass 2: Ihat and r
    L.r = o + arr;
    o += (2u * arr > 8192u) ? 2u * arr : 8192u;
    L.scr = o;    o += 2048u;                          // column (max, sum) per warp
    L.s = o;      o += 512u;
    L.colm = o;   o += 256u;
    L.colf = o;   o += 256u;
    L.vis = o;    o += 512u;
    L.red = o;    o += 256u;
    L.bt = o;     o += 4u * kUnitMaxPages;             // the sequence's page list (paged caches)
    L.bars = o;   o += 128u;
    L.total = o + 1024u;
    return L;
}

cudaError_t launch_unit(const UnitParams &p, int n_units, int nqp, size_t smem,
                        cudaStream_t stream);

// Shared selection (rkv_shared.cu): pointers already offset to the launch's
// first layer.
struct SharedParams {
    uint16_t *k[kMaxLayersPerLaunch];
    uint16_t *v[kMaxLayersPerLaunch];
    int32_t batch, n_kv, window, cap, budget_cfg;
    const int32_t *budgets;
    const int32_t *n_eff;
    const float *z_heads;    // [layers][batch][Hkv][cap] per-head Z
    float *z_sum;            // [layers][batch][cap]
    int32_t *kept_out;       // optional [layers][batch][cap]
    uint32_t *status;
};
cudaError_t launch_head_sum(const SharedParams &p, int n_lb, cudaStream_t stream);
cudaError_t launch_shared_compact(const SharedParams &p, int n_units, cudaStream_t stream);
size_t shared_select_smem(int cap);

cudaError_t launch_freed_pages(int batch, const int32_t *budgets, int32_t budget_cfg,
                               const int32_t *n_eff, const int32_t *block_table, int max_blocks,
                               int page_rows, int32_t *freed, int32_t *n_freed,
                               cudaStream_t stream);

// MAX-mode similarity kernel: raw r of every candidate of every due unit.
struct alignas(64) GramParams {
    CUtensorMap tmap[kMaxLayersPerLaunch];   // [rows, 128] bf16, box 64 x 128 (paged: 64 x page_rows), SW128
    int32_t layer_base, batch, n_kv, window, cap;
    int32_t n_tokens_fixed;  // > 0: per-head entry point, N fixed
    const int32_t *n_eff;
    const int32_t *order;    // sequences by decreasing length (plan kernel), or null
    const int64_t *seq_row;  // per-sequence capacities, as in UnitParams (or null)
    const int32_t *seq_cap;
    const int32_t *block_table;   // paged caches, as in UnitParams (or null)
    int32_t max_blocks, page_rows;
    float *r_out;            // [units][cap]
    uint32_t *status;
};
// before_gram / after_gram (or null): recorded around the similarity kernel.
cudaError_t launch_gram_max(const GramParams &p, int n_units, cudaStream_t stream,
                            cudaEvent_t before_gram = nullptr, cudaEvent_t after_gram = nullptr);
int gram_max_rows();   // longest unit the similarity kernel holds

struct AppendParams {
    uint16_t *k[kMaxLayersPerLaunch];
    uint16_t *v[kMaxLayersPerLaunch];
    const uint16_t *k_new[kMaxLayersPerLaunch];
    const uint16_t *v_new[kMaxLayersPerLaunch];
    int32_t batch, n_kv, cap, n_new;
    const int32_t *cur_len;
    uint32_t *status;
};
cudaError_t launch_append(const AppendParams &p, int n_layers, cudaStream_t stream);
cudaError_t launch_bump(int batch, int n_new, int cap, int32_t *cur_len, cudaStream_t stream);

}  // namespace rkv
