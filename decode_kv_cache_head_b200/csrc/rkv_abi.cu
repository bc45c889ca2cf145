// rkv_abi.cu -- the extern "C" entry points declared in include/rkv.h:
// argument validation (synchronous, before anything is enqueued), TMA
// descriptor encoding, shape selection and kernel launches on the caller's
// stream.  No allocation, no synchronisation, no state kept between calls.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "rkv_internal.h"
#include "rkv_ptx.cuh"

using namespace rkv;

namespace {

constexpr int32_t kVersion = 1 * 10000 + 0 * 100 + 0;
constexpr int kSmemPerSM = 233472;            // 228 KB of shared memory per SM
constexpr int kSmemPerCtaMax = 232448;        // 227 KB opt-in limit per CTA
constexpr int kSmemTwoPerSM = kSmemPerSM / 2 - 1024;
constexpr int kB200SMs = 148;                 // launches with at least this many units use
                                              // the one-CTA-per-unit kernel

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// A [rows, 128] bf16 row-major matrix read in boxes of 64 columns x box_rows
// rows with the 128-byte swizzle (one box row = 128 bytes = one swizzle span).
bool encode_rows128(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim * 2)};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t es[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
              box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlap(const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

int nqp_of(int nq) { return (nq + 15) / 16 * 16; }

rkv_status check_cfg(const rkv_config *c) {
    if (!c) return RKV_ERR_NULL;
    if (c->head_dim != kHeadDim) return RKV_ERR_UNSUPPORTED;
    if (c->n_kv_heads < 1 || c->n_q_heads < 1 || c->n_q_heads % c->n_kv_heads != 0)
        return RKV_ERR_INVALID;
    if (c->window < 1) return RKV_ERR_INVALID;
    if (static_cast<int64_t>(c->n_q_heads / c->n_kv_heads) * c->window > kMaxQCols)
        return RKV_ERR_UNSUPPORTED;
    if (!std::isfinite(c->mix_lambda)) return RKV_ERR_INVALID;
    if (c->redundancy_mode != RKV_RED_MEAN && c->redundancy_mode != RKV_RED_MAX)
        return RKV_ERR_INVALID;
    if (c->gqa_pool != RKV_GQA_MAX && c->gqa_pool != RKV_GQA_MEAN) return RKV_ERR_INVALID;
    return RKV_OK;
}

struct Shape {
    int cs, rmax, rp, tmem_cols, nqp;
    size_t smem;
};

int pow2_at_least(int x) {
    int p = 32;
    while (p < x) p <<= 1;
    return p;
}

Shape shape_for(int cap, int nqp, int cs) {
    Shape s;
    s.cs = cs;
    s.nqp = nqp;
    s.rmax = ((cap + cs - 1) / cs + 15) / 16 * 16;
    s.rp = s.rmax < 128 ? 128 : s.rmax;
    const int ntiles = (s.rmax + 127) / 128;
    s.tmem_cols = pow2_at_least(ntiles * nqp);
    s.smem = step_smem_bytes(s.rp, s.rmax, cap, nqp, cs);
    // TMEM holds 512 columns per SM: never let more CTAs share an SM than fit,
    // by asking for enough shared memory to cap residency.
    const int max_res = 512 / s.tmem_cols;
    const size_t floor_smem = static_cast<size_t>(kSmemPerSM / (max_res + 1) - 1024 + 16);
    if (s.smem < floor_smem) s.smem = floor_smem;
    return s;
}

// Picks the cluster size: the smallest of 8, 16, 4, 2 whose layout lets two
// CTAs share an SM, else the smallest that fits at all.  cs = 0 if none fits.
Shape choose_shape(int cap, int nqp, int cs_req) {
    if (cs_req) {
        Shape s = shape_for(cap, nqp, cs_req);
        if (s.smem > static_cast<size_t>(kSmemPerCtaMax) || s.rmax > 512) s.cs = 0;
        return s;
    }
    const int order[4] = {8, 16, 4, 2};
    for (int i = 0; i < 4; ++i) {
        Shape s = shape_for(cap, nqp, order[i]);
        if (s.smem <= static_cast<size_t>(kSmemTwoPerSM) && s.rmax <= 512) return s;
    }
    for (int i = 0; i < 4; ++i) {
        Shape s = shape_for(cap, nqp, order[i]);
        if (s.smem <= static_cast<size_t>(kSmemPerCtaMax) && s.rmax <= 512) return s;
    }
    Shape none = {};
    return none;
}

// The one-CTA-per-unit kernel: dynamic shared memory and TMEM columns for
// caches of `cap` rows; ok = false when the unit does not fit one CTA.
struct UnitShape {
    bool ok;
    int tmem_cols;
    size_t smem;
};

UnitShape unit_shape(int cap, int nqp) {
    UnitShape u = {};
    if (cap > kUnitMaxRows) return u;
    u.tmem_cols = pow2_at_least(2 * (nqp + 16) + 16);   // two tile slots + the S accumulator
    u.smem = make_unit_layout(cap, nqp).total;
    const int max_res = 512 / u.tmem_cols;   // CTAs whose TMEM fits one SM
    const size_t floor_smem = static_cast<size_t>(kSmemPerSM / (max_res + 1) - 1024 + 16);
    if (u.smem < floor_smem) u.smem = floor_smem;
    u.ok = u.smem <= static_cast<size_t>(kSmemPerCtaMax);
    return u;
}

// cs_req: 0 = automatic, 1 = one CTA per unit, else the cluster size.
bool use_unit_kernel(int64_t n_units, int cap, int nqp, int cs_req) {
    if (cs_req == 1) return true;
    if (cs_req > 1) return false;
    return n_units >= kB200SMs && unit_shape(cap, nqp).ok;
}

// Paged caches: the page pools' geometry and the block table (null: contiguous).
struct PagedArgs {
    const int32_t *block_table;
    int32_t max_blocks, page_rows, num_pages;
};

// The one-CTA-per-unit kernel over all layers, 32 per launch.  z_heads != null:
// scores only (shared selection), no cache writes.
cudaError_t launch_unit_layers(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                               const rkv_bf16 *const *k_layers, rkv_bf16 *const *v_layers,
                               const rkv_bf16 *const *q_layers, const int32_t *budgets,
                               const float *lambdas, const int32_t *n_eff, const float *r_ext,
                               int32_t *kept_out, float *scores_out, float *z_heads,
                               uint32_t *status, const UnitShape &us, int nqp, cudaStream_t strm,
                               const PagedArgs &pg = PagedArgs{nullptr, 0, 0, 0},
                               const RaggedLayout &rg = RaggedLayout{},
                               const int32_t *order = nullptr) {
    UnitParams *up = new UnitParams();
    std::memset(up, 0, sizeof(*up));
    up->batch = batch;
    up->n_kv = cfg->n_kv_heads;
    up->group = cfg->n_q_heads / cfg->n_kv_heads;
    up->window = cfg->window;
    up->cap = cap;
    up->nmax = cap;
    up->tmem_cols = us.tmem_cols;
    up->budget_cfg = cfg->budget;
    up->lambda_cfg = cfg->mix_lambda;
    up->logit_scale_log2 =
        static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim)));
    up->red_mode = cfg->redundancy_mode;
    up->gqa_pool = cfg->gqa_pool;
    up->budgets = budgets;
    up->lambdas = lambdas;
    up->n_eff = n_eff;
    up->order = order;
    up->r_ext = r_ext;
    up->kept_out = kept_out;
    up->scores_out = scores_out;
    up->z_heads = z_heads;
    up->block_table = pg.block_table;
    up->max_blocks = pg.max_blocks;
    up->page_rows = pg.page_rows;
    up->seq_row = rg.seq_row;
    up->seq_cap = rg.seq_cap;
    up->status = status;
    const uint64_t k_rows = pg.block_table
                                ? static_cast<uint64_t>(pg.num_pages) * cfg->n_kv_heads * pg.page_rows
                            : rg.seq_row ? static_cast<uint64_t>(rg.pool_rows)
                                         : static_cast<uint64_t>(batch) * cfg->n_kv_heads * cap;
    const uint32_t k_box = pg.block_table ? static_cast<uint32_t>(pg.page_rows) : 128u;
    cudaError_t e = cudaSuccess;
    for (int l0 = 0; e == cudaSuccess && l0 < n_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = (n_layers - l0 < kMaxLayersPerLaunch) ? n_layers - l0 : kMaxLayersPerLaunch;
        up->layer_base = l0;
        for (int i = 0; i < nl; ++i) {
            const int l = l0 + i;
            if (!encode_rows128(&up->tmap_k[i], k_layers[l], k_rows, k_box) ||
                !encode_rows128(&up->tmap_q[i], q_layers[l],
                                static_cast<uint64_t>(batch) * cfg->n_q_heads * cfg->window,
                                static_cast<uint32_t>(nqp))) {
                e = cudaErrorInvalidValue;
                break;
            }
            up->k[i] = const_cast<uint16_t *>(k_layers[l]);
            up->v[i] = v_layers ? v_layers[l] : nullptr;
        }
        if (e == cudaSuccess) e = launch_unit(*up, nl * batch * cfg->n_kv_heads, nqp, us.smem, strm);
    }
    delete up;
    return e;
}

// MAX mode: raw r of every candidate of every due unit, by the similarity kernel.
// sim_begin / sim_end (or null): recorded before the first and after the last launch
// of the similarity kernel.
cudaError_t launch_gram_layers(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                               const rkv_bf16 *const *k_layers, const int32_t *n_eff, float *r_ext,
                               uint32_t *status, cudaStream_t strm, cudaEvent_t sim_begin = nullptr,
                               cudaEvent_t sim_end = nullptr,
                               const RaggedLayout &rg = RaggedLayout{},
                               const PagedArgs &pg = PagedArgs{nullptr, 0, 0, 0},
                               const int32_t *order = nullptr) {
    GramParams *gp = new GramParams();
    std::memset(gp, 0, sizeof(*gp));
    gp->batch = batch;
    gp->n_kv = cfg->n_kv_heads;
    gp->window = cfg->window;
    gp->cap = cap;
    gp->n_eff = n_eff;
    gp->order = order;
    gp->seq_row = rg.seq_row;
    gp->seq_cap = rg.seq_cap;
    gp->block_table = pg.block_table;
    gp->max_blocks = pg.max_blocks;
    gp->page_rows = pg.page_rows;
    gp->r_out = r_ext;
    gp->status = status;
    const uint64_t k_rows = pg.block_table
                                ? static_cast<uint64_t>(pg.num_pages) * cfg->n_kv_heads * pg.page_rows
                            : rg.seq_row ? static_cast<uint64_t>(rg.pool_rows)
                                         : static_cast<uint64_t>(batch) * cfg->n_kv_heads * cap;
    const uint32_t k_box = pg.block_table ? static_cast<uint32_t>(pg.page_rows) : 128u;
    cudaError_t e = cudaSuccess;
    for (int l0 = 0; e == cudaSuccess && l0 < n_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = (n_layers - l0 < kMaxLayersPerLaunch) ? n_layers - l0 : kMaxLayersPerLaunch;
        gp->layer_base = l0;
        for (int i = 0; i < nl && e == cudaSuccess; ++i)
            if (!encode_rows128(&gp->tmap[i], k_layers[l0 + i], k_rows, k_box)) e = cudaErrorInvalidValue;
        if (e == cudaSuccess)
            e = launch_gram_max(*gp, nl * batch * cfg->n_kv_heads, strm, l0 == 0 ? sim_begin : nullptr,
                                l0 + nl >= n_layers ? sim_end : nullptr);
    }
    delete gp;
    return e;
}

// Workspace of the shared-selection calls: the step's, then the per-head Z of
// every unit.
size_t ws_bytes_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap);

size_t ws_bytes_for(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap) {
    size_t n = kStatusBytes;
    n += align256(static_cast<size_t>(batch) * 4);
    if (cfg->redundancy_mode == RKV_RED_MAX)   // r per unit, from the similarity kernel
        n += align256(static_cast<size_t>(n_layers) * batch * cfg->n_kv_heads * cap * 4);
    return n;
}

size_t ws_bytes_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap) {
    const size_t units = static_cast<size_t>(n_layers) * batch * cfg->n_kv_heads;
    return ws_bytes_for(cfg, n_layers, batch, cap) + align256(units * cap * 4);
}

// Past the part a call needs (`base` bytes), a workspace may hold the plan kernel's
// order of the sequences by decreasing length (one int32 each); the batched kernels
// then start the longest sequences' units first.  rkv_workspace_size and
// rkv_workspace_size_shared include that room; a workspace without it runs the units in
// layer-major order (same results).
size_t order_bytes(int32_t batch) { return align256(static_cast<size_t>(batch) * 4); }

int32_t *order_slot(uint8_t *ws, size_t ws_bytes, size_t base, int32_t batch) {
    return ws_bytes >= base + order_bytes(batch) ? reinterpret_cast<int32_t *>(ws + base) : nullptr;
}

void fill_common(StepParams &p, const rkv_config *cfg, const Shape &s, int batch, int cap) {
    p.batch = batch;
    p.n_kv = cfg->n_kv_heads;
    p.group = cfg->n_q_heads / cfg->n_kv_heads;
    p.window = cfg->window;
    p.cap = cap;
    p.cs = s.cs;
    p.rmax = s.rmax;
    p.rp = s.rp;
    p.tmem_cols = s.tmem_cols;
    p.budget_cfg = cfg->budget;
    p.lambda_cfg = cfg->mix_lambda;
    p.logit_scale_log2 =
        static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(kHeadDim)));
    p.red_mode = cfg->redundancy_mode;
    p.gqa_pool = cfg->gqa_pool;
}

// The CUDA error behind the calling thread's latest RKV_ERR_CUDA.
thread_local int32_t g_last_cuda_error = 0;

rkv_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return RKV_OK;
    g_last_cuda_error = static_cast<int32_t>(e);
    return RKV_ERR_CUDA;
}

// Per-head entry points share this: one (sequence, layer), all KV heads.
rkv_status run_per_head_scores(const rkv_config *cfg, const rkv_bf16 *q, const rkv_bf16 *k,
                               int64_t head_stride, int32_t n_tokens, int32_t flags, float *I,
                               float *inv, float *r, float *R, void *ws, size_t ws_bytes,
                               cudaStream_t stream) {
    const int cap = static_cast<int>(head_stride / kHeadDim);
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    const Shape s = choose_shape(cap, nqp, 0);
    if (s.cs == 0) return RKV_ERR_UNSUPPORTED;
    const bool red_max = cfg->redundancy_mode == RKV_RED_MAX && (r || R);
    if (red_max && cap > gram_max_rows()) return RKV_ERR_UNSUPPORTED;
    StepParams *pp = new StepParams();
    StepParams &p = *pp;
    std::memset(&p, 0, sizeof(p));
    fill_common(p, cfg, s, 1, cap);
    p.n_layers = 1;
    p.n_tokens_fixed = n_tokens;
    p.flags = flags;
    p.out_I = I;
    p.out_inv = inv;
    p.out_r = r;
    p.out_R = R;
    p.status = static_cast<uint32_t *>(ws);
    p.red_mode = red_max ? RKV_RED_MAX : RKV_RED_MEAN;
    bool ok = encode_rows128(&p.tmap_k[0], k, static_cast<uint64_t>(cfg->n_kv_heads) * cap, 16);
    if (flags & kFlagImportance)
        ok = ok && encode_rows128(&p.tmap_q[0], q,
                                  static_cast<uint64_t>(cfg->n_q_heads) * cfg->window,
                                  static_cast<uint32_t>(nqp));
    GramParams *gp = nullptr;
    if (ok && red_max) {
        gp = new GramParams();
        std::memset(gp, 0, sizeof(*gp));
        ok = encode_rows128(&gp->tmap[0], k, static_cast<uint64_t>(cfg->n_kv_heads) * cap, 128);
        gp->batch = 1;
        gp->n_kv = cfg->n_kv_heads;
        gp->window = cfg->window;
        gp->cap = cap;
        gp->n_tokens_fixed = n_tokens;
        gp->r_out = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kStatusBytes + 256);
        gp->status = static_cast<uint32_t *>(ws);
        p.r_ext = gp->r_out;
    }
    if (!ok) {
        delete pp;
        delete gp;
        return RKV_ERR_CUDA;
    }
    p.k[0] = const_cast<uint16_t *>(k);
    cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, stream);
    if (e == cudaSuccess && gp) e = launch_gram_max(*gp, cfg->n_kv_heads, stream);
    if (e == cudaSuccess) e = launch_step(p, cfg->n_kv_heads, nqp, s.smem, stream);
    delete pp;
    delete gp;
    (void)ws_bytes;
    return cuda_status(e);
}

}  // namespace

// The part of a step's workspace the call cannot run without (no room for the order of
// the sequences); 0 for an invalid configuration.
namespace rkv {
size_t workspace_required_bytes(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                int32_t cap);
}  // namespace rkv

size_t rkv::workspace_required_bytes(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                     int32_t cap) {
    if (check_cfg(cfg) != RKV_OK || n_layers < 1 || batch < 1 || cap < 2) return 0;
    return ws_bytes_for(cfg, n_layers, batch, cap);
}

extern "C" {

const char *rkv_status_string(rkv_status s) {
    switch (s) {
        case RKV_OK: return "RKV_OK";
        case RKV_STATUS_DISABLED: return "RKV_STATUS_DISABLED: budget or buffer <= 0, compression off";
        case RKV_ERR_NULL: return "RKV_ERR_NULL: a required pointer is NULL";
        case RKV_ERR_INVALID: return "RKV_ERR_INVALID: inconsistent sizes";
        case RKV_ERR_ALIGN: return "RKV_ERR_ALIGN: a device pointer or stride is not 16-byte aligned";
        case RKV_ERR_ALIAS: return "RKV_ERR_ALIAS: outputs overlap inputs";
        case RKV_ERR_WORKSPACE: return "RKV_ERR_WORKSPACE: workspace missing or too small";
        case RKV_ERR_UNSUPPORTED: return "RKV_ERR_UNSUPPORTED: shape outside the supported range";
        case RKV_ERR_CUDA: return "RKV_ERR_CUDA: a CUDA call or launch failed";
        case RKV_STATUS_DEVICE_TIMEOUT: return "RKV_STATUS_DEVICE_TIMEOUT: a device-side wait ran out";
        case RKV_ERR_DEVICE_INPUT: return "RKV_ERR_DEVICE_INPUT: invalid device-side input";
    }
    return "unknown rkv_status";
}

int32_t rkv_version(void) { return kVersion; }

int32_t rkv_last_cuda_error(void) { return g_last_cuda_error; }

size_t rkv_workspace_size(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap) {
    if (check_cfg(cfg) != RKV_OK || n_layers < 1 || batch < 1 || cap < 2) return 0;
    return ws_bytes_for(cfg, n_layers, batch, cap) + order_bytes(batch);
}

rkv_status rkv_query_step_shape(const rkv_config *cfg, int64_t n_units, int32_t cap,
                                int32_t *cluster_size, int32_t *rows_per_cta, size_t *smem_bytes) {
    const rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cap < 2 || n_units < 1) return RKV_ERR_INVALID;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    if (use_unit_kernel(n_units, cap, nqp, 0)) {
        const UnitShape u = unit_shape(cap, nqp);
        if (cluster_size) *cluster_size = 1;
        if (rows_per_cta) *rows_per_cta = cap;
        if (smem_bytes) *smem_bytes = u.smem;
        return RKV_OK;
    }
    const Shape s = choose_shape(cap, nqp, 0);
    if (s.cs == 0) return RKV_ERR_UNSUPPORTED;
    if (cluster_size) *cluster_size = s.cs;
    if (rows_per_cta) *rows_per_cta = s.rmax;
    if (smem_bytes) *smem_bytes = s.smem;
    return RKV_OK;
}

rkv_status rkv_workspace_status(const void *workspace, rkv_stream_t stream) {
    if (!workspace) return RKV_ERR_NULL;
    uint32_t word = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e);
    if (word & kDevFlagTimeout) return RKV_STATUS_DEVICE_TIMEOUT;
    if (word) return RKV_ERR_DEVICE_INPUT;
    return RKV_OK;
}

rkv_status rkv_score_importance(const rkv_config *cfg, const rkv_bf16 *q, const rkv_bf16 *k,
                                int64_t k_head_stride, int32_t n_tokens, float *I,
                                float *inv_norm, void *workspace, size_t ws_bytes,
                                rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_score_importance");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (!q || !k || !I) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(workspace)) return RKV_ERR_ALIGN;
    if (k_head_stride % kHeadDim != 0) return RKV_ERR_ALIGN;
    if (n_tokens <= cfg->window || k_head_stride < static_cast<int64_t>(n_tokens) * kHeadDim)
        return RKV_ERR_INVALID;
    const int cap = static_cast<int>(k_head_stride / kHeadDim);
    if (ws_bytes < ws_bytes_for(cfg, 1, 1, cap)) return RKV_ERR_WORKSPACE;
    return run_per_head_scores(cfg, q, k, k_head_stride, n_tokens, kFlagImportance | kFlagOutScores,
                               I, inv_norm, nullptr, nullptr, workspace, ws_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

rkv_status rkv_score_redundancy(const rkv_config *cfg, const rkv_bf16 *k, int64_t k_head_stride,
                                int32_t n_tokens, float *r, float *R, void *workspace,
                                size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_score_redundancy");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (!k || (!r && !R)) return RKV_ERR_NULL;
    if (!aligned16(k) || !aligned16(workspace)) return RKV_ERR_ALIGN;
    if (k_head_stride % kHeadDim != 0) return RKV_ERR_ALIGN;
    if (n_tokens <= cfg->window || k_head_stride < static_cast<int64_t>(n_tokens) * kHeadDim)
        return RKV_ERR_INVALID;
    const int cap = static_cast<int>(k_head_stride / kHeadDim);
    if (ws_bytes < ws_bytes_for(cfg, 1, 1, cap)) return RKV_ERR_WORKSPACE;
    return run_per_head_scores(cfg, nullptr, k, k_head_stride, n_tokens, kFlagOutScores, nullptr,
                               nullptr, r, R, workspace, ws_bytes,
                               reinterpret_cast<cudaStream_t>(stream));
}

rkv_status rkv_select_topk(const rkv_config *cfg, const float *I, const float *R,
                           int32_t n_tokens, int32_t *kept, float *Z, void *workspace,
                           size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_select_topk");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->budget <= 0 || cfg->buffer <= 0) return RKV_STATUS_DISABLED;
    if (!I || !R || !kept) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (cfg->budget < cfg->window || cfg->budget > n_tokens || n_tokens <= cfg->window)
        return RKV_ERR_INVALID;
    const int M = n_tokens - cfg->window;
    if (static_cast<size_t>(M) * 4 > static_cast<size_t>(kSmemPerCtaMax) - 4096)
        return RKV_ERR_UNSUPPORTED;
    if (ws_bytes < kStatusBytes) return RKV_ERR_WORKSPACE;
    if (Z && (overlap(Z, static_cast<size_t>(M) * cfg->n_kv_heads * 4, I,
                      static_cast<size_t>(M) * cfg->n_kv_heads * 4) ||
              overlap(Z, static_cast<size_t>(M) * cfg->n_kv_heads * 4, R,
                      static_cast<size_t>(M) * cfg->n_kv_heads * 4)))
        return RKV_ERR_ALIAS;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess)
        e = launch_select(I, R, cfg->n_kv_heads, M, n_tokens, cfg->budget, cfg->mix_lambda, kept, Z,
                          static_cast<uint32_t *>(workspace), s);
    return cuda_status(e);
}

rkv_status rkv_compact_kv(const rkv_config *cfg, const rkv_bf16 *k_src, const rkv_bf16 *v_src,
                          const int32_t *kept, rkv_bf16 *k_dst, rkv_bf16 *v_dst,
                          int64_t head_stride, int32_t n_tokens, void *workspace,
                          size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_compact_kv");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->budget <= 0 || cfg->buffer <= 0) return RKV_STATUS_DISABLED;
    if (!k_src || !v_src || !kept || !k_dst || !v_dst) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (ws_bytes < kStatusBytes) return RKV_ERR_WORKSPACE;
    if (!aligned16(k_src) || !aligned16(v_src) || !aligned16(k_dst) || !aligned16(v_dst))
        return RKV_ERR_ALIGN;
    if (head_stride % 8 != 0) return RKV_ERR_ALIGN;
    if (cfg->budget > n_tokens || head_stride < static_cast<int64_t>(n_tokens) * kHeadDim)
        return RKV_ERR_INVALID;
    const size_t extent =
        (static_cast<size_t>(cfg->n_kv_heads - 1) * head_stride + static_cast<size_t>(n_tokens) * kHeadDim) * 2;
    const bool k_same = k_dst == k_src, v_same = v_dst == v_src;
    if (k_same != v_same) return RKV_ERR_ALIAS;
    if (overlap(k_dst, extent, v_dst, extent) || overlap(k_src, extent, v_src, extent))
        return RKV_ERR_ALIAS;
    int cs = 0;
    if (k_same) {
        cs = compact_in_place_cluster(cfg->budget);
        if (cs == 0) return RKV_ERR_UNSUPPORTED;
    } else if (overlap(k_dst, extent, k_src, extent) || overlap(k_dst, extent, v_src, extent) ||
               overlap(v_dst, extent, k_src, extent) || overlap(v_dst, extent, v_src, extent)) {
        return RKV_ERR_ALIAS;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess)
        e = launch_compact(k_src, v_src, kept, k_dst, v_dst, head_stride, cfg->n_kv_heads,
                           cfg->budget, n_tokens, k_same, cs, static_cast<uint32_t *>(workspace), s);
    return cuda_status(e);
}

rkv_status rkv_compress_step(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                             rkv_bf16 *const *k_layers, rkv_bf16 *const *v_layers,
                             const rkv_bf16 *const *q_layers, const int32_t *budgets,
                             const float *lambdas, int32_t *cur_len,
                             const rkv_step_options *opts, void *workspace, size_t ws_bytes,
                             rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_compress_step");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->buffer <= 0 || (!budgets && cfg->budget <= 0)) return RKV_STATUS_DISABLED;
    if (!k_layers || !v_layers || !q_layers || !cur_len) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (n_layers < 1 || batch < 1 || cap < 2) return RKV_ERR_INVALID;
    if (!budgets && (cfg->budget < cfg->window || cfg->budget >= cap)) return RKV_ERR_INVALID;
    if (static_cast<int64_t>(batch) * cfg->n_kv_heads * cap > INT32_MAX ||
        static_cast<int64_t>(batch) * cfg->n_q_heads * cfg->window > INT32_MAX)
        return RKV_ERR_UNSUPPORTED;
    const size_t layer_bytes = static_cast<size_t>(batch) * cfg->n_kv_heads * cap * kHeadDim * 2;
    for (int l = 0; l < n_layers; ++l) {
        if (!k_layers[l] || !v_layers[l] || !q_layers[l]) return RKV_ERR_NULL;
        if (!aligned16(k_layers[l]) || !aligned16(v_layers[l]) || !aligned16(q_layers[l]))
            return RKV_ERR_ALIGN;
        if (overlap(k_layers[l], layer_bytes, v_layers[l], layer_bytes)) return RKV_ERR_ALIAS;
    }
    if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return RKV_ERR_ALIGN;
    if (ws_bytes < ws_bytes_for(cfg, n_layers, batch, cap)) return RKV_ERR_WORKSPACE;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    const int cs_req = opts ? opts->cluster_size : 0;
    if (cs_req != 0 && cs_req != 1 && cs_req != 2 && cs_req != 4 && cs_req != 8 && cs_req != 16)
        return RKV_ERR_INVALID;
    const bool unit_path =
        use_unit_kernel(static_cast<int64_t>(n_layers) * batch * cfg->n_kv_heads, cap, nqp, cs_req);
    const UnitShape us = unit_path ? unit_shape(cap, nqp) : UnitShape{};
    if (unit_path && !us.ok) return RKV_ERR_UNSUPPORTED;
    const Shape s = unit_path ? Shape{} : choose_shape(cap, nqp, cs_req);
    if (!unit_path && s.cs == 0) return RKV_ERR_UNSUPPORTED;
    if (cfg->redundancy_mode == RKV_RED_MAX && cap > gram_max_rows()) return RKV_ERR_UNSUPPORTED;

    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    int32_t *n_eff = reinterpret_cast<int32_t *>(ws + kStatusBytes);
    float *r_ext = reinterpret_cast<float *>(ws + kStatusBytes + align256(static_cast<size_t>(batch) * 4));
    const bool red_max = cfg->redundancy_mode == RKV_RED_MAX;
    int32_t *order = unit_path ? order_slot(ws, ws_bytes, ws_bytes_for(cfg, n_layers, batch, cap), batch)
                               : nullptr;

    StepParams *pp = new StepParams();
    StepParams &p = *pp;
    std::memset(&p, 0, sizeof(p));
    fill_common(p, cfg, s, batch, cap);
    p.budgets = budgets;
    p.lambdas = lambdas;
    p.n_eff = n_eff;
    p.flags = kFlagImportance | kFlagSelect;
    p.kept_out = opts ? opts->kept_out : nullptr;
    p.scores_out = opts ? opts->scores_out : nullptr;
    p.status = status;
    p.r_ext = red_max ? r_ext : nullptr;

    // the plan kernel clears the status words first
    cudaError_t e = launch_plan(batch, budgets, cfg->budget, cfg->buffer, cfg->window, cap, cur_len,
                                n_eff, status, strm, true, RaggedLayout{}, order);
    if (red_max && e == cudaSuccess)   // raw r of every candidate: the tcgen05 similarity kernel
        e = launch_gram_layers(cfg, n_layers, batch, cap,
                               const_cast<const rkv_bf16 *const *>(k_layers), n_eff, r_ext, status,
                               strm, opts ? reinterpret_cast<cudaEvent_t>(opts->sim_begin) : nullptr,
                               opts ? reinterpret_cast<cudaEvent_t>(opts->sim_end) : nullptr,
                               RaggedLayout{}, PagedArgs{nullptr, 0, 0, 0}, order);
    if (e == cudaSuccess && opts && opts->main_begin)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_begin), strm);
    if (unit_path && e == cudaSuccess)
        e = launch_unit_layers(cfg, n_layers, batch, cap, k_layers, v_layers, q_layers, budgets,
                               lambdas, n_eff, p.r_ext, p.kept_out, p.scores_out, nullptr, status,
                               us, nqp, strm, PagedArgs{nullptr, 0, 0, 0}, RaggedLayout{}, order);
    for (int l0 = 0; !unit_path && e == cudaSuccess && l0 < n_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = (n_layers - l0 < kMaxLayersPerLaunch) ? n_layers - l0 : kMaxLayersPerLaunch;
        p.n_layers = nl;
        p.layer_base = l0;
        for (int i = 0; i < nl; ++i) {
            const int l = l0 + i;
            if (!encode_rows128(&p.tmap_k[i], k_layers[l],
                                static_cast<uint64_t>(batch) * cfg->n_kv_heads * cap, 16) ||
                !encode_rows128(&p.tmap_q[i], q_layers[l],
                                static_cast<uint64_t>(batch) * cfg->n_q_heads * cfg->window,
                                static_cast<uint32_t>(nqp))) {
                e = cudaErrorInvalidValue;
                break;
            }
            p.k[i] = k_layers[l];
            p.v[i] = v_layers[l];
        }
        if (e == cudaSuccess) e = launch_step(p, nl * batch * cfg->n_kv_heads, nqp, s.smem, strm);
    }
    if (e == cudaSuccess && opts && opts->main_end)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_end), strm);
    delete pp;
    return cuda_status(e);
}

rkv_status rkv_append_kv(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                         rkv_bf16 *const *k_layers, rkv_bf16 *const *v_layers,
                         const rkv_bf16 *const *k_new_layers, const rkv_bf16 *const *v_new_layers,
                         int32_t n_new, int32_t *cur_len, void *workspace, size_t ws_bytes,
                         rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_append_kv");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (!k_layers || !v_layers || !k_new_layers || !v_new_layers || !cur_len) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (ws_bytes < kStatusBytes) return RKV_ERR_WORKSPACE;
    if (n_layers < 1 || batch < 1 || cap < 2 || n_new < 1 || n_new > cap) return RKV_ERR_INVALID;
    const size_t layer_bytes = static_cast<size_t>(batch) * cfg->n_kv_heads * cap * kHeadDim * 2;
    const size_t new_bytes = static_cast<size_t>(batch) * cfg->n_kv_heads * n_new * kHeadDim * 2;
    for (int l = 0; l < n_layers; ++l) {
        if (!k_layers[l] || !v_layers[l] || !k_new_layers[l] || !v_new_layers[l]) return RKV_ERR_NULL;
        if (!aligned16(k_layers[l]) || !aligned16(v_layers[l]) || !aligned16(k_new_layers[l]) ||
            !aligned16(v_new_layers[l]))
            return RKV_ERR_ALIGN;
        if (overlap(k_layers[l], layer_bytes, v_layers[l], layer_bytes) ||
            overlap(k_new_layers[l], new_bytes, k_layers[l], layer_bytes) ||
            overlap(k_new_layers[l], new_bytes, v_layers[l], layer_bytes) ||
            overlap(v_new_layers[l], new_bytes, k_layers[l], layer_bytes) ||
            overlap(v_new_layers[l], new_bytes, v_layers[l], layer_bytes))
            return RKV_ERR_ALIAS;
    }
    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint32_t *status = static_cast<uint32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, strm);
    AppendParams p;
    std::memset(&p, 0, sizeof(p));
    p.batch = batch;
    p.n_kv = cfg->n_kv_heads;
    p.cap = cap;
    p.n_new = n_new;
    p.cur_len = cur_len;
    p.status = status;
    for (int l0 = 0; e == cudaSuccess && l0 < n_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = (n_layers - l0 < kMaxLayersPerLaunch) ? n_layers - l0 : kMaxLayersPerLaunch;
        for (int i = 0; i < nl; ++i) {
            p.k[i] = k_layers[l0 + i];
            p.v[i] = v_layers[l0 + i];
            p.k_new[i] = k_new_layers[l0 + i];
            p.v_new[i] = v_new_layers[l0 + i];
        }
        e = launch_append(p, nl, strm);
    }
    if (e == cudaSuccess) e = launch_bump(batch, n_new, cap, cur_len, strm);
    return cuda_status(e);
}

size_t rkv_workspace_size_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                 int32_t cap) {
    if (check_cfg(cfg) != RKV_OK || n_layers < 1 || batch < 1 || cap < 2) return 0;
    return ws_bytes_shared(cfg, n_layers, batch, cap) + order_bytes(batch);
}

}  // extern "C"

namespace {

// Checks shared by the two shared-selection calls (q_layers / v_layers may be
// absent in one of them).
rkv_status check_shared_args(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                             const rkv_bf16 *const *k_layers, const rkv_bf16 *const *v_layers,
                             const rkv_bf16 *const *q_layers, const int32_t *budgets,
                             const void *cur_len, const void *z_sum, const void *workspace,
                             size_t ws_bytes) {
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->buffer <= 0 || (!budgets && cfg->budget <= 0)) return RKV_STATUS_DISABLED;
    if (!k_layers || !cur_len || !z_sum) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (n_layers < 1 || batch < 1 || cap < 2) return RKV_ERR_INVALID;
    if (!budgets && (cfg->budget < cfg->window || cfg->budget >= cap)) return RKV_ERR_INVALID;
    if (static_cast<int64_t>(batch) * cfg->n_kv_heads * cap > INT32_MAX ||
        static_cast<int64_t>(batch) * cfg->n_q_heads * cfg->window > INT32_MAX)
        return RKV_ERR_UNSUPPORTED;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    if (!unit_shape(cap, nqp).ok) return RKV_ERR_UNSUPPORTED;
    if (cfg->redundancy_mode == RKV_RED_MAX && cap > gram_max_rows()) return RKV_ERR_UNSUPPORTED;
    const size_t layer_bytes = static_cast<size_t>(batch) * cfg->n_kv_heads * cap * kHeadDim * 2;
    for (int l = 0; l < n_layers; ++l) {
        if (!k_layers[l] || (v_layers && !v_layers[l]) || (q_layers && !q_layers[l]))
            return RKV_ERR_NULL;
        if (!aligned16(k_layers[l]) || (v_layers && !aligned16(v_layers[l])) ||
            (q_layers && !aligned16(q_layers[l])))
            return RKV_ERR_ALIGN;
        if (v_layers && overlap(k_layers[l], layer_bytes, v_layers[l], layer_bytes))
            return RKV_ERR_ALIAS;
    }
    if (!aligned16(z_sum)) return RKV_ERR_ALIGN;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RKV_ERR_ALIGN;
    if (ws_bytes < ws_bytes_shared(cfg, n_layers, batch, cap)) return RKV_ERR_WORKSPACE;
    return RKV_OK;
}

}  // namespace

extern "C" {

rkv_status rkv_score_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch, int32_t cap,
                            const rkv_bf16 *const *k_layers, const rkv_bf16 *const *q_layers,
                            const int32_t *budgets, const float *lambdas, const int32_t *cur_len,
                            float *z_sum, void *workspace, size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_score_shared");
    if (!q_layers) return check_cfg(cfg) != RKV_OK ? check_cfg(cfg) : RKV_ERR_NULL;
    rkv_status st = check_shared_args(cfg, n_layers, batch, cap, k_layers, nullptr, q_layers,
                                      budgets, cur_len, z_sum, workspace, ws_bytes);
    if (st != RKV_OK) return st;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    const UnitShape us = unit_shape(cap, nqp);
    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    int32_t *n_eff = reinterpret_cast<int32_t *>(ws + kStatusBytes);
    const size_t base = ws_bytes_for(cfg, n_layers, batch, cap);
    float *r_ext = reinterpret_cast<float *>(ws + kStatusBytes + align256(static_cast<size_t>(batch) * 4));
    float *z_heads = reinterpret_cast<float *>(ws + base);
    const bool red_max = cfg->redundancy_mode == RKV_RED_MAX;
    int32_t *order = order_slot(ws, ws_bytes, ws_bytes_shared(cfg, n_layers, batch, cap), batch);
    // the plan kernel clears the status words first
    cudaError_t e = launch_plan(batch, budgets, cfg->budget, cfg->buffer, cfg->window, cap,
                                const_cast<int32_t *>(cur_len), n_eff, status, strm, false,
                                RaggedLayout{}, order);
    if (red_max && e == cudaSuccess)
        e = launch_gram_layers(cfg, n_layers, batch, cap, k_layers, n_eff, r_ext, status, strm,
                               nullptr, nullptr, RaggedLayout{}, PagedArgs{nullptr, 0, 0, 0}, order);
    if (e == cudaSuccess)
        e = launch_unit_layers(cfg, n_layers, batch, cap, k_layers, nullptr, q_layers, budgets,
                               lambdas, n_eff, red_max ? r_ext : nullptr, nullptr, nullptr, z_heads,
                               status, us, nqp, strm, PagedArgs{nullptr, 0, 0, 0}, RaggedLayout{},
                               order);
    SharedParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.batch = batch;
    sp.n_kv = cfg->n_kv_heads;
    sp.window = cfg->window;
    sp.cap = cap;
    sp.n_eff = n_eff;
    sp.z_heads = z_heads;
    sp.z_sum = z_sum;
    sp.status = status;
    if (e == cudaSuccess) e = launch_head_sum(sp, n_layers * batch, strm);
    return cuda_status(e);
}

rkv_status rkv_select_compact_shared(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                     int32_t cap, rkv_bf16 *const *k_layers,
                                     rkv_bf16 *const *v_layers, const int32_t *budgets,
                                     int32_t *cur_len, const float *z_sum, int32_t *kept_out,
                                     void *workspace, size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_select_compact_shared");
    if (!v_layers) return check_cfg(cfg) != RKV_OK ? check_cfg(cfg) : RKV_ERR_NULL;
    rkv_status st = check_shared_args(cfg, n_layers, batch, cap,
                                      const_cast<const rkv_bf16 *const *>(k_layers),
                                      const_cast<const rkv_bf16 *const *>(v_layers), nullptr,
                                      budgets, cur_len, z_sum, workspace, ws_bytes);
    if (st != RKV_OK) return st;
    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    int32_t *n_eff = reinterpret_cast<int32_t *>(ws + kStatusBytes);
    const size_t units = static_cast<size_t>(n_layers) * batch * cfg->n_kv_heads;
    // the plan kernel clears the status words first
    cudaError_t e = launch_plan(batch, budgets, cfg->budget, cfg->buffer, cfg->window, cap, cur_len,
                                n_eff, status, strm, true);
    SharedParams sp;
    std::memset(&sp, 0, sizeof(sp));
    sp.batch = batch;
    sp.n_kv = cfg->n_kv_heads;
    sp.window = cfg->window;
    sp.cap = cap;
    sp.budget_cfg = cfg->budget;
    sp.budgets = budgets;
    sp.n_eff = n_eff;
    sp.status = status;
    for (int l0 = 0; e == cudaSuccess && l0 < n_layers; l0 += kMaxLayersPerLaunch) {
        const int nl = (n_layers - l0 < kMaxLayersPerLaunch) ? n_layers - l0 : kMaxLayersPerLaunch;
        const size_t off = static_cast<size_t>(l0) * batch * cap;
        sp.z_sum = const_cast<float *>(z_sum) + off;
        sp.kept_out = kept_out ? kept_out + off : nullptr;
        for (int i = 0; i < nl; ++i) {
            sp.k[i] = k_layers[l0 + i];
            sp.v[i] = v_layers[l0 + i];
        }
        e = launch_shared_compact(sp, nl * batch * cfg->n_kv_heads, strm);
    }
    return cuda_status(e);
}

rkv_status rkv_compress_step_paged(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                   const rkv_paged_kv *pg, rkv_bf16 *const *k_pools,
                                   rkv_bf16 *const *v_pools, const rkv_bf16 *const *q_layers,
                                   const int32_t *budgets, const float *lambdas, int32_t *cur_len,
                                   const rkv_step_options *opts, void *workspace, size_t ws_bytes,
                                   rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_compress_step_paged");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->buffer <= 0 || (!budgets && cfg->budget <= 0)) return RKV_STATUS_DISABLED;
    if (!pg || !k_pools || !v_pools || !q_layers || !cur_len) return RKV_ERR_NULL;
    if (!pg->block_table || !pg->freed_pages || !pg->n_freed) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    const int P = pg->page_rows;
    if (P != 16 && P != 32 && P != 64 && P != 128) return RKV_ERR_UNSUPPORTED;
    if (n_layers < 1 || batch < 1 || pg->max_blocks < 1 || pg->num_pages < 1) return RKV_ERR_INVALID;
    if (opts && opts->cluster_size != 0 && opts->cluster_size != 1) return RKV_ERR_UNSUPPORTED;
    const int64_t cap64 = static_cast<int64_t>(pg->max_blocks) * P;
    if (cap64 > kUnitMaxPages * static_cast<int64_t>(P) ||
        static_cast<int64_t>(pg->num_pages) * cfg->n_kv_heads * P > INT32_MAX)
        return RKV_ERR_UNSUPPORTED;
    const int cap = static_cast<int>(cap64);
    if (!budgets && (cfg->budget < cfg->window || cfg->budget >= cap)) return RKV_ERR_INVALID;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    const UnitShape us = unit_shape(cap, nqp);
    if (!us.ok) return RKV_ERR_UNSUPPORTED;
    const size_t pool_bytes = static_cast<size_t>(pg->num_pages) * cfg->n_kv_heads * P * kHeadDim * 2;
    for (int l = 0; l < n_layers; ++l) {
        if (!k_pools[l] || !v_pools[l] || !q_layers[l]) return RKV_ERR_NULL;
        if (!aligned16(k_pools[l]) || !aligned16(v_pools[l]) || !aligned16(q_layers[l]))
            return RKV_ERR_ALIGN;
        if (overlap(k_pools[l], pool_bytes, v_pools[l], pool_bytes)) return RKV_ERR_ALIAS;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RKV_ERR_ALIGN;
    if (ws_bytes < ws_bytes_for(cfg, n_layers, batch, cap)) return RKV_ERR_WORKSPACE;

    if (cfg->redundancy_mode == RKV_RED_MAX && cap > gram_max_rows()) return RKV_ERR_UNSUPPORTED;

    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    int32_t *n_eff = reinterpret_cast<int32_t *>(ws + kStatusBytes);
    float *r_ext = reinterpret_cast<float *>(ws + kStatusBytes + align256(static_cast<size_t>(batch) * 4));
    const bool red_max = cfg->redundancy_mode == RKV_RED_MAX;
    const PagedArgs pa{pg->block_table, pg->max_blocks, P, pg->num_pages};
    int32_t *order = order_slot(ws, ws_bytes, ws_bytes_for(cfg, n_layers, batch, cap), batch);
    // the plan kernel clears the status words first
    cudaError_t e = launch_plan(batch, budgets, cfg->budget, cfg->buffer, cfg->window, cap, cur_len,
                                n_eff, status, strm, true, RaggedLayout{}, order);
    if (red_max && e == cudaSuccess)   // raw r of every candidate, through the block table
        e = launch_gram_layers(cfg, n_layers, batch, cap,
                               const_cast<const rkv_bf16 *const *>(k_pools), n_eff, r_ext, status,
                               strm, opts ? reinterpret_cast<cudaEvent_t>(opts->sim_begin) : nullptr,
                               opts ? reinterpret_cast<cudaEvent_t>(opts->sim_end) : nullptr,
                               RaggedLayout{}, pa, order);
    if (e == cudaSuccess)
        e = launch_freed_pages(batch, budgets, cfg->budget, n_eff, pg->block_table, pg->max_blocks,
                               P, pg->freed_pages, pg->n_freed, strm);
    if (e == cudaSuccess && opts && opts->main_begin)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_begin), strm);
    if (e == cudaSuccess)
        e = launch_unit_layers(cfg, n_layers, batch, cap,
                               const_cast<const rkv_bf16 *const *>(k_pools), v_pools, q_layers,
                               budgets, lambdas, n_eff, red_max ? r_ext : nullptr,
                               opts ? opts->kept_out : nullptr,
                               opts ? opts->scores_out : nullptr, nullptr, status, us, nqp, strm, pa,
                               RaggedLayout{}, order);
    if (e == cudaSuccess && opts && opts->main_end)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_end), strm);
    return cuda_status(e);
}

rkv_status rkv_compress_step_ragged(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                    const rkv_ragged_kv *rg, rkv_bf16 *const *k_pools,
                                    rkv_bf16 *const *v_pools, const rkv_bf16 *const *q_layers,
                                    const int32_t *budgets, const float *lambdas,
                                    int32_t *cur_len, const rkv_step_options *opts,
                                    void *workspace, size_t ws_bytes, rkv_stream_t stream) {
    NvtxRange nvtx_range("rkv_compress_step_ragged");
    rkv_status st = check_cfg(cfg);
    if (st != RKV_OK) return st;
    if (cfg->buffer <= 0 || (!budgets && cfg->budget <= 0)) return RKV_STATUS_DISABLED;
    if (!rg || !k_pools || !v_pools || !q_layers || !cur_len) return RKV_ERR_NULL;
    if (!rg->seq_row || !rg->seq_cap) return RKV_ERR_NULL;
    if (!workspace) return RKV_ERR_WORKSPACE;
    if (n_layers < 1 || batch < 1 || rg->max_cap < 2 || rg->pool_rows < 1) return RKV_ERR_INVALID;
    if (rg->pool_rows > INT32_MAX || static_cast<int64_t>(batch) * cfg->n_q_heads * cfg->window > INT32_MAX)
        return RKV_ERR_UNSUPPORTED;
    const int cap = rg->max_cap;
    if (!budgets && (cfg->budget < cfg->window || cfg->budget >= cap)) return RKV_ERR_INVALID;
    if (opts && opts->cluster_size != 0 && opts->cluster_size != 1) return RKV_ERR_UNSUPPORTED;
    const int nqp = nqp_of((cfg->n_q_heads / cfg->n_kv_heads) * cfg->window);
    const UnitShape us = unit_shape(cap, nqp);
    if (!us.ok) return RKV_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(rg->seq_row) & 7u) || (reinterpret_cast<uintptr_t>(rg->seq_cap) & 3u))
        return RKV_ERR_ALIGN;
    const size_t pool_bytes = static_cast<size_t>(rg->pool_rows) * kHeadDim * 2;
    for (int l = 0; l < n_layers; ++l) {
        if (!k_pools[l] || !v_pools[l] || !q_layers[l]) return RKV_ERR_NULL;
        if (!aligned16(k_pools[l]) || !aligned16(v_pools[l]) || !aligned16(q_layers[l]))
            return RKV_ERR_ALIGN;
        if (overlap(k_pools[l], pool_bytes, v_pools[l], pool_bytes)) return RKV_ERR_ALIAS;
    }
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return RKV_ERR_ALIGN;
    if (ws_bytes < ws_bytes_for(cfg, n_layers, batch, cap)) return RKV_ERR_WORKSPACE;
    if (cfg->redundancy_mode == RKV_RED_MAX && cap > gram_max_rows()) return RKV_ERR_UNSUPPORTED;

    cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws);
    int32_t *n_eff = reinterpret_cast<int32_t *>(ws + kStatusBytes);
    float *r_ext = reinterpret_cast<float *>(ws + kStatusBytes + align256(static_cast<size_t>(batch) * 4));
    const bool red_max = cfg->redundancy_mode == RKV_RED_MAX;
    RaggedLayout lay;
    lay.seq_row = rg->seq_row;
    lay.seq_cap = rg->seq_cap;
    lay.pool_rows = rg->pool_rows;
    lay.n_kv = cfg->n_kv_heads;
    int32_t *order = order_slot(ws, ws_bytes, ws_bytes_for(cfg, n_layers, batch, cap), batch);
    // the plan kernel clears the status words first, then checks every due sequence's
    // block against the pool
    cudaError_t e = launch_plan(batch, budgets, cfg->budget, cfg->buffer, cfg->window, cap, cur_len,
                                n_eff, status, strm, true, lay, order);
    if (red_max && e == cudaSuccess)
        e = launch_gram_layers(cfg, n_layers, batch, cap,
                               const_cast<const rkv_bf16 *const *>(k_pools), n_eff, r_ext, status,
                               strm, opts ? reinterpret_cast<cudaEvent_t>(opts->sim_begin) : nullptr,
                               opts ? reinterpret_cast<cudaEvent_t>(opts->sim_end) : nullptr, lay,
                               PagedArgs{nullptr, 0, 0, 0}, order);
    if (e == cudaSuccess && opts && opts->main_begin)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_begin), strm);
    if (e == cudaSuccess)
        e = launch_unit_layers(cfg, n_layers, batch, cap,
                               const_cast<const rkv_bf16 *const *>(k_pools), v_pools, q_layers,
                               budgets, lambdas, n_eff, red_max ? r_ext : nullptr,
                               opts ? opts->kept_out : nullptr, opts ? opts->scores_out : nullptr,
                               nullptr, status, us, nqp, strm, PagedArgs{nullptr, 0, 0, 0}, lay,
                               order);
    if (e == cudaSuccess && opts && opts->main_end)
        e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(opts->main_end), strm);
    return cuda_status(e);
}

}  // extern "C"
