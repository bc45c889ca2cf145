// rkv_internal.h -- host-side declarations shared by the C-ABI layer and the
// kernel launchers.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/rkv.h"

namespace rkv {

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

struct SmemLayout {
    uint32_t k, q, v, inv, ss, ihat, rr, dst, keys, spart, gs, reds, statm, statl, gm, glinv,
        red, hist, misc, bars, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) {
    return (x + a - 1) / a * a;
}

// Offsets from a 1024-byte-aligned base; `total` includes 1024 bytes of slack
// for aligning the dynamic shared-memory pointer.
__host__ __device__ inline SmemLayout make_layout(int rp, int rmax, int cap, int nqp) {
    SmemLayout L;
    uint32_t o = 0;
    L.k = o;      o += 2u * rp * 128u;
    L.q = o;      o += 2u * nqp * 128u;
    L.v = o;      o += static_cast<uint32_t>(rmax) * 256u;
    L.inv = o;    o += align_up(rmax * 4u, 16);
    L.ss = o;     o += align_up(rmax * 4u, 16);
    L.ihat = o;   o += align_up(rmax * 4u, 16);
    L.rr = o;     o += align_up(rmax * 4u, 16);
    L.dst = o;    o += align_up(rmax * 4u, 16);
    L.keys = o;   o += align_up(cap * 4u, 16);
    L.spart = o;  o += 128u * 4u;
    L.gs = o;     o += 128u * 4u;
    L.reds = o;   o += 4u * 128u * 4u;
    L.statm = o;  o += nqp * 4u;
    L.statl = o;  o += nqp * 4u;
    L.gm = o;     o += nqp * 4u;
    L.glinv = o;  o += nqp * 4u;
    L.red = o;    o += 4u * nqp * 4u;
    L.hist = o;   o += 256u * 4u;
    L.misc = o;   o += 64u * 4u;
    L.bars = o;   o += 64u;
    L.total = o + 1024u;
    return L;
}

// Launchers (defined in the .cu files); all return cudaSuccess or the launch error.
cudaError_t launch_plan(int batch, const int32_t *budgets, int32_t budget_cfg, int32_t buffer,
                        int32_t window, int32_t cap, int32_t *cur_len, int32_t *n_eff,
                        uint32_t *status, cudaStream_t stream);
cudaError_t launch_step(const StepParams &p, int n_units, int nqp, size_t smem,
                        cudaStream_t stream);
size_t step_smem_bytes(int rp, int rmax, int cap, int nqp);
cudaError_t launch_select(const float *I, const float *R, int n_kv, int M, int N, int budget,
                          float lambda, int32_t *kept, float *Z, uint32_t *status,
                          cudaStream_t stream);
cudaError_t launch_compact(const uint16_t *k_src, const uint16_t *v_src, const int32_t *kept,
                           uint16_t *k_dst, uint16_t *v_dst, int64_t head_stride, int n_kv,
                           int budget, int n_tokens, bool in_place, int cs, uint32_t *status,
                           cudaStream_t stream);
int compact_in_place_cluster(int budget);   // 0: too large for the staged in-place path

}  // namespace rkv
