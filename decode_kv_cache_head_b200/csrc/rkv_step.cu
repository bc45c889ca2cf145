// rkv_step.cu -- the R-KV compression step on sm_100a: the plan kernel (which
// sequences are due) and the fused per-unit kernel (importance, redundancy,
// joint score, selection and in-place compaction of one (sequence, layer,
// KV head) by one thread-block cluster).
//
// Method: "R-KV: Redundancy-aware KV Cache Compression for Reasoning Models"
// (atlas.scime.ai summary, "Approach": Z = lambda I - (1 - lambda) R,
// applied periodically during decoding with a fixed buffer; "Measured
// effects" table: max pooling over the GQA group), the hysenlabs write-up
// "R-KV: decoding-time KV cache compression for reasoning models" (section
// on decode-time scoring: budget, window_size, mix_lambda, divide_length;
// protected recent window) and the sourcepulse summary ("How It Works":
// importance from attention weights, cosine similarity for near-duplicates,
// top-k within the budget).
//
// Work decomposition.  One cluster of `cs` CTAs (128 threads each) handles one
// unit of N cached rows; CTA c owns rows [c*R, c*R + R) with R = ceil16(N/cs).
//   1. TMA loads the CTA's K rows and the unit's G*w query rows into shared
//      memory (128-byte swizzle), once; K is never read from HBM again.
//   2. One thread issues tcgen05 UMMAs: logits[rows, G*w] = K_rows . Q^T into
//      TMEM (M = 128 key rows per tile, N = G*w padded to 16, K = 128).
//   3. Meanwhile all threads compute ||k_i||^2, 1/max(||k_i||, 1e-12) and the
//      CTA's part of S = sum_i khat_i (for the mean-redundancy row sum).
//   4. TMEM epilogue: per-query-column max and sum of exp over the CTA's
//      visible keys; exchanged over DSMEM (cluster barrier 1).
//   5. Per row: p = softmax probabilities, mean over the window, max over the
//      group -> Ihat_i; r_i = (khat_i . S - khat_i . khat_i) / (N - 1) (MEAN)
//      or r from the similarity kernel (MAX).  Partial sum Ihat, max r and
//      sum exp(r - max) exchanged (cluster barrier 2).
//   6. Every CTA pulls all candidates' Ihat and r over DSMEM, forms
//      Z = lambda Ihat/sum - (1-lambda) exp(r - rmax)/rsum, and runs the same
//      deterministic radix select (the k-th largest key, ties to the lower
//      index), so all CTAs agree on the kept set without another exchange.
//   7. Each CTA stages the V rows of its kept rows that move (bulk copies),
//      cluster barrier 3 (all K and V reads of the unit are done), then writes
//      its kept K rows (from shared memory) and V rows to their destinations.
//      Reading everything before any write makes the in-place gather safe.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace cg = cooperative_groups;

namespace rkv {

// ----------------------------------------------------------------------------
// Plan: which sequences are due; snapshot their length; set cur_len = budget.
// ----------------------------------------------------------------------------
__global__ void rkv_plan_kernel(int batch, const int32_t *__restrict__ budgets,
                                int32_t budget_cfg, int32_t buffer, int32_t window,
                                int32_t cap, int32_t *__restrict__ cur_len,
                                int32_t *__restrict__ n_eff, uint32_t *__restrict__ status) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    const int32_t bud = budgets ? budgets[b] : budget_cfg;
    const int32_t n = cur_len[b];
    // Compression is active only when budget and buffer are both positive.
    bool due = bud > 0 && buffer > 0 && n >= bud + buffer;
    if (due && (bud < window || n > cap)) {
        record_flag(status, kDevFlagBadSeq);
        due = false;
    }
    n_eff[b] = due ? n : 0;
    if (due) cur_len[b] = bud;
}

cudaError_t launch_plan(int batch, const int32_t *budgets, int32_t budget_cfg, int32_t buffer,
                        int32_t window, int32_t cap, int32_t *cur_len, int32_t *n_eff,
                        uint32_t *status, cudaStream_t stream) {
    const int threads = 128;
    const int blocks = (batch + threads - 1) / threads;
    rkv_plan_kernel<<<blocks, threads, 0, stream>>>(batch, budgets, budget_cfg, buffer, window,
                                                    cap, cur_len, n_eff, status);
    return cudaGetLastError();
}

// ----------------------------------------------------------------------------
// The fused per-unit kernel.
// ----------------------------------------------------------------------------
template <int NQP>
__global__ void __launch_bounds__(kThreads, 1) rkv_step_kernel(const __grid_constant__ StepParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    cg::cluster_group cluster = cg::this_cluster();
    const int cs = p.cs;
    const uint32_t rank = cluster.block_rank();
    const int unit = blockIdx.x / cs;
    const int h = unit % p.n_kv;
    const int b = (unit / p.n_kv) % p.batch;
    const int l = unit / (p.n_kv * p.batch);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int N = p.n_tokens_fixed > 0 ? p.n_tokens_fixed : p.n_eff[b];
    if (N <= 0) return;  // not due: the whole cluster leaves before any exchange

    const int w = p.window;
    const int G = p.group;
    const int NQ = G * w;
    const int M = N - w;
    const int budget = p.budgets ? p.budgets[b] : p.budget_cfg;
    const float lam = p.lambdas ? p.lambdas[b] : p.lambda_cfg;
    const int kk = budget - w;
    const bool do_imp = (p.flags & kFlagImportance) != 0;
    const bool do_sel = (p.flags & kFlagSelect) != 0;
    const bool red_max = p.red_mode == RKV_RED_MAX;

    const int R = ((N + cs - 1) / cs + 15) / 16 * 16;
    const int row0 = static_cast<int>(rank) * R;
    const int nrows = max(0, min(R, N - row0));
    const int nbox = (nrows + 15) / 16;
    const int nrows_pad = nbox * 16;
    const int ntiles = (nrows_pad + 127) / 128;
    const int64_t krow0 = (static_cast<int64_t>(b) * p.n_kv + h) * p.cap;   // row in the layer's 2D view
    const int64_t unit_g = (static_cast<int64_t>(p.layer_base + l) * p.batch + b) * p.n_kv + h;

    const SmemLayout L = make_layout(p.rp, p.rmax, p.cap, NQP);
    uint8_t *sK = base + L.k;
    uint8_t *sQ = base + L.q;
    uint8_t *sV = base + L.v;
    float *sInv = reinterpret_cast<float *>(base + L.inv);
    float *sSS = reinterpret_cast<float *>(base + L.ss);
    float *sIhat = reinterpret_cast<float *>(base + L.ihat);
    float *sRr = reinterpret_cast<float *>(base + L.rr);
    int32_t *sDst = reinterpret_cast<int32_t *>(base + L.dst);
    uint32_t *sKeys = reinterpret_cast<uint32_t *>(base + L.keys);
    float *sSpart = reinterpret_cast<float *>(base + L.spart);
    float *sGS = reinterpret_cast<float *>(base + L.gs);
    float *sRedS = reinterpret_cast<float *>(base + L.reds);
    float *sStatM = reinterpret_cast<float *>(base + L.statm);
    float *sStatL = reinterpret_cast<float *>(base + L.statl);
    float *sGM = reinterpret_cast<float *>(base + L.gm);
    float *sGLinv = reinterpret_cast<float *>(base + L.glinv);
    float *sRed = reinterpret_cast<float *>(base + L.red);
    uint32_t *sHist = reinterpret_cast<uint32_t *>(base + L.hist);
    float *sMisc = reinterpret_cast<float *>(base + L.misc);   // [0..2]: published partials
    float *sRed4 = sMisc + 8;                                   // block reduction scratch
    int *sInt = reinterpret_cast<int *>(sMisc + 16);            // scan / select scratch
    float *sGlob = sMisc + 32;                                  // cluster-wide scalars
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L.bars);
    uint64_t *bar_tma = bars + 0, *bar_mma = bars + 1, *bar_v = bars + 2;
    uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 4);

    bool ok = true;  // false after a timed-out wait: keep joining barriers, skip the writes

    // ---- set-up: TMEM, barriers, loads
    if (do_imp && warp == 0) {
        tmem_alloc(sTmem, static_cast<uint32_t>(p.tmem_cols));
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        mbar_init(bar_v, 1);
        fence_mbar_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = do_imp ? *sTmem : 0u;

    if (tid == 0 && nrows > 0) {
        const CUtensorMap *mk = &p.tmap_k[l];
        const uint32_t bytes = static_cast<uint32_t>(nbox) * 4096u +
                               (do_imp ? static_cast<uint32_t>(NQP) * 256u : 0u);
        mbar_arrive_expect_tx(bar_tma, bytes);
        for (int bx = 0; bx < nbox; ++bx) {
            const int32_t y = static_cast<int32_t>(krow0 + row0 + bx * 16);
            tma_load_2d(sK + bx * 16 * 128, mk, bar_tma, 0, y);
            tma_load_2d(sK + p.rp * 128 + bx * 16 * 128, mk, bar_tma, 64, y);
        }
        if (do_imp) {
            const CUtensorMap *mq = &p.tmap_q[l];
            const int32_t yq = (b * p.n_kv + h) * NQ;   // rows of this KV head's query group
            tma_load_2d(sQ, mq, bar_tma, 0, yq);
            tma_load_2d(sQ + NQP * 128, mq, bar_tma, 64, yq);
        }
    }
    if (nrows > 0) {
        if (!mbar_wait(bar_tma, 0)) {
            ok = false;
            record_flag(p.status, kDevFlagTimeout);
        }
    }

    // ---- UMMA: logits of every row against the G*w window queries
    auto tile_start = [&](int t) { return t < ntiles - 1 ? t * 128 : max(0, nrows_pad - 128); };
    if (do_imp && nrows > 0 && tid == 0) {
        tc_fence_after();
        constexpr uint32_t idesc = idesc_bf16_f32(128, NQP);
        const uint32_t k_base = smem_u32(sK), q_base = smem_u32(sQ);
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t a_row = static_cast<uint32_t>(tile_start(t)) * 128u;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint32_t half = ks >> 2, koff = (ks & 3) * 32u;
                const uint64_t ad = desc_kmajor_sw128(k_base + half * p.rp * 128u + a_row + koff);
                const uint64_t bd = desc_kmajor_sw128(q_base + half * NQP * 128u + koff);
                umma_bf16(tmem_base + static_cast<uint32_t>(t * NQP), ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
        }
        umma_commit(bar_mma);
    }

    // ---- norms (thread per row) while the tensor cores work
    for (int t = 0; t < ntiles; ++t) {
        const int row = tile_start(t) + tid;
        if (row < t * 128 || row >= nrows) continue;
        float ss = 0.f;
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            const uint8_t *src = sK + (c >> 3) * p.rp * 128 + sw128_offset(row, c & 7);
            const uint4 raw = *reinterpret_cast<const uint4 *>(src);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
            }
        }
        sSS[row] = ss;
        sInv[row] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();

    // ---- this CTA's part of S = sum_i khat_i (warp w takes rows w, w+4, ...; lane: 4 columns)
    if (!red_max) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        const int half = lane >> 4, cc = (lane & 15) >> 1, sub = lane & 1;
        for (int row = warp; row < nrows; row += kWarps) {
            const uint8_t *src = sK + half * p.rp * 128 + sw128_offset(row, cc) + sub * 8;
            const uint2 raw = *reinterpret_cast<const uint2 *>(src);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
            const float iv = sInv[row];
            const float2 f0 = __bfloat1622float2(h2[0]);
            const float2 f1 = __bfloat1622float2(h2[1]);
            acc[0] = fmaf(f0.x, iv, acc[0]);
            acc[1] = fmaf(f0.y, iv, acc[1]);
            acc[2] = fmaf(f1.x, iv, acc[2]);
            acc[3] = fmaf(f1.y, iv, acc[3]);
        }
        const int col = half * 64 + (lane & 15) * 4;
#pragma unroll
        for (int e = 0; e < 4; ++e) sRedS[warp * 128 + col + e] = acc[e];
        __syncthreads();
        sSpart[tid] = ((sRedS[tid] + sRedS[128 + tid]) + sRedS[256 + tid]) + sRedS[384 + tid];
    }

    // ---- softmax statistics of the CTA's rows for every query column
    const float sc = p.logit_scale_log2;
    if (do_imp) {
        if (nrows > 0) {
            if (!mbar_wait(bar_mma, 0)) {
                ok = false;
                record_flag(p.status, kDevFlagTimeout);
            }
            tc_fence_after();
        }
        // pass 1: column max (log2 domain)
        float cm[NQP];
#pragma unroll
        for (int q = 0; q < NQP; ++q) cm[q] = -INFINITY;
        if (nrows > 0) {
            for (int t = 0; t < ntiles; ++t) {
                const int row = tile_start(t) + tid;
                const bool valid = row >= t * 128 && row < nrows;
                const int gi = row0 + row;
#pragma unroll
                for (int c0 = 0; c0 < NQP; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem_base + ((32u * warp) << 16) + t * NQP + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int q = c0 + i;
                        const bool vis = valid && q < NQ && gi <= M + (q % w);
                        cm[q] = fmaxf(cm[q], vis ? v[i] * sc : -INFINITY);
                    }
                }
            }
        }
#pragma unroll
        for (int c0 = 0; c0 < NQP; c0 += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = cm[c0 + i];
            warp_transpose_reduce16(v, OpMax());
            if (lane < 16) sRed[warp * NQP + c0 + lane] = v[0];
        }
        __syncthreads();
        if (tid < NQP)
            sStatM[tid] = fmaxf(fmaxf(sRed[tid], sRed[NQP + tid]),
                                fmaxf(sRed[2 * NQP + tid], sRed[3 * NQP + tid]));
        __syncthreads();
        // pass 2: column sum of exp2(s - max) over the visible rows
        float cl[NQP];
#pragma unroll
        for (int q = 0; q < NQP; ++q) cl[q] = 0.f;
        if (nrows > 0) {
            for (int t = 0; t < ntiles; ++t) {
                const int row = tile_start(t) + tid;
                const bool valid = row >= t * 128 && row < nrows;
                const int gi = row0 + row;
#pragma unroll
                for (int c0 = 0; c0 < NQP; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem_base + ((32u * warp) << 16) + t * NQP + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int q = c0 + i;
                        const bool vis = valid && q < NQ && gi <= M + (q % w);
                        if (vis) cl[q] += exp2f(v[i] * sc - sStatM[q]);
                    }
                }
            }
        }
#pragma unroll
        for (int c0 = 0; c0 < NQP; c0 += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = cl[c0 + i];
            warp_transpose_reduce16(v, OpSum());
            if (lane < 16) sRed[warp * NQP + c0 + lane] = v[0];
        }
        __syncthreads();
        if (tid < NQP)
            sStatL[tid] = ((sRed[tid] + sRed[NQP + tid]) + sRed[2 * NQP + tid]) + sRed[3 * NQP + tid];
    }
    __syncthreads();

    // ================= cluster barrier 1: column statistics and S partials published
    cluster.sync();

    if (do_imp && tid < NQP) {
        float m = -INFINITY;
        for (int c = 0; c < cs; ++c) m = fmaxf(m, cluster.map_shared_rank(sStatM, c)[tid]);
        float lsum = 0.f;
        for (int c = 0; c < cs; ++c) {
            const float mc = cluster.map_shared_rank(sStatM, c)[tid];
            const float lc = cluster.map_shared_rank(sStatL, c)[tid];
            if (mc != -INFINITY) lsum += lc * exp2f(mc - m);
        }
        sGM[tid] = m;
        sGLinv[tid] = (lsum > 0.f) ? 1.0f / lsum : 0.f;
    }
    if (!red_max) {
        float s = 0.f;
        for (int c = 0; c < cs; ++c) s += cluster.map_shared_rank(sSpart, c)[tid];
        sGS[tid] = s;
    }
    __syncthreads();

    // ---- per row: importance Ihat_i, redundancy r_i
    const float inv_w = 1.0f / static_cast<float>(w);
    const float inv_nm1 = 1.0f / static_cast<float>(N - 1);
    float sumI = 0.f, rmax_loc = -INFINITY;
    for (int t = 0; t < ntiles; ++t) {
        const int row = tile_start(t) + tid;
        const bool valid = row >= t * 128 && row < nrows;
        const int gi = row0 + row;
        float ihat = 0.f;
        if (do_imp) {
            // loads are warp-collective: every lane takes part, valid or not
            float run = 0.f, best = (p.gqa_pool == RKV_GQA_MAX) ? -INFINITY : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < NQP; c0 += 16) {
                float v[16];
                tmem_ld16(tmem_base + ((32u * warp) << 16) + t * NQP + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int q = c0 + i;
                    if (q < NQ) {
                        const int j = q % w;
                        const float pr = (gi <= M + j) ? exp2f(v[i] * sc - sGM[q]) * sGLinv[q] : 0.f;
                        run += pr;
                        if (j == w - 1) {
                            const float a = run * inv_w;
                            best = (p.gqa_pool == RKV_GQA_MAX) ? fmaxf(best, a) : best + a;
                            run = 0.f;
                        }
                    }
                }
            }
            ihat = (p.gqa_pool == RKV_GQA_MAX) ? best : best / static_cast<float>(G);
        }
        if (!valid || gi >= M) continue;
        float r;
        if (red_max) {
            r = p.r_ext[unit_g * p.cap + gi];
        } else {
            float dot = 0.f;
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                const uint8_t *src = sK + (c >> 3) * p.rp * 128 + sw128_offset(row, c & 7);
                const uint4 raw = *reinterpret_cast<const uint4 *>(src);
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                const float4 s0 = *reinterpret_cast<const float4 *>(sGS + c * 8);
                const float4 s1 = *reinterpret_cast<const float4 *>(sGS + c * 8 + 4);
                const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
                const float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
                dot = fmaf(f0.x, s0.x, dot); dot = fmaf(f0.y, s0.y, dot);
                dot = fmaf(f1.x, s0.z, dot); dot = fmaf(f1.y, s0.w, dot);
                dot = fmaf(f2.x, s1.x, dot); dot = fmaf(f2.y, s1.y, dot);
                dot = fmaf(f3.x, s1.z, dot); dot = fmaf(f3.y, s1.w, dot);
            }
            const float iv = sInv[row];
            r = (iv * dot - iv * iv * sSS[row]) * inv_nm1;
        }
        sIhat[row] = ihat;
        sRr[row] = r;
        sumI += ihat;
        rmax_loc = fmaxf(rmax_loc, r);
    }
    sumI = block_allreduce(sumI, OpSum(), sRed4);
    rmax_loc = block_allreduce(rmax_loc, OpMax(), sRed4);
    float rsum = 0.f;
    for (int t = 0; t < ntiles; ++t) {
        const int row = tile_start(t) + tid;
        const int gi = row0 + row;
        if (row < t * 128 || row >= nrows || gi >= M) continue;
        rsum += exp2f((sRr[row] - rmax_loc) * 1.4426950408889634f);
    }
    rsum = block_allreduce(rsum, OpSum(), sRed4);
    if (tid == 0) {
        sMisc[0] = sumI;
        sMisc[1] = rmax_loc;
        sMisc[2] = rsum;
    }
    __syncthreads();

    // ================= cluster barrier 2: per-row scores and partial normalisers published
    cluster.sync();

    if (tid == 0) {
        float si = 0.f, rm = -INFINITY;
        for (int c = 0; c < cs; ++c) {
            const float *pm = cluster.map_shared_rank(sMisc, c);
            si += pm[0];
            rm = fmaxf(rm, pm[1]);
        }
        float rs = 0.f;
        for (int c = 0; c < cs; ++c) {
            const float *pm = cluster.map_shared_rank(sMisc, c);
            if (pm[1] != -INFINITY) rs += pm[2] * exp2f((pm[1] - rm) * 1.4426950408889634f);
        }
        sGlob[0] = si;
        sGlob[1] = rm;
        sGlob[2] = rs;
    }
    __syncthreads();
    const float sumI_g = sGlob[0], rmax_g = sGlob[1], rsum_g = sGlob[2];
    const float inv_rsum = 1.0f / rsum_g;

    if (p.flags & kFlagOutScores) {
        // per-head entry points: write this CTA's rows and stop
        for (int t = 0; t < ntiles; ++t) {
            const int row = tile_start(t) + tid;
            const int gi = row0 + row;
            if (row < t * 128 || row >= nrows) continue;
            if (p.out_inv) p.out_inv[static_cast<int64_t>(h) * N + gi] = sInv[row];
            if (gi < M) {
                const int64_t o = static_cast<int64_t>(h) * M + gi;
                if (p.out_I) p.out_I[o] = sIhat[row] / sumI_g;
                if (p.out_r) p.out_r[o] = sRr[row];
                if (p.out_R)
                    p.out_R[o] = exp2f((sRr[row] - rmax_g) * 1.4426950408889634f) * inv_rsum;
            }
        }
    }

    if (do_sel) {
        // ---- every CTA: keys of all M candidates (pulled over DSMEM), then the same select
        for (int j = tid; j < M; j += kThreads) {
            const int c = j / R, lr = j - c * R;
            const float ih = cluster.map_shared_rank(sIhat, c)[lr];
            const float rr = cluster.map_shared_rank(sRr, c)[lr];
            const float I = ih / sumI_g;
            const float Rv = exp2f((rr - rmax_g) * 1.4426950408889634f) * inv_rsum;
            sKeys[j] = ordered_key(joint_score(lam, I, Rv));
        }
        __syncthreads();
        uint32_t T = 0xffffffffu;
        int n_gt = 0;
        if (kk > 0) block_select_kth(sKeys, M, kk, sHist, sInt, T, n_gt);
        const int need_eq = (kk > 0) ? kk - n_gt : 0;

        // kept rows before this CTA's range
        const int lim = min(row0, M);
        int c_gt = 0, c_eq = 0;
        for (int j = tid; j < lim; j += kThreads) {
            const uint32_t key = sKeys[j];
            c_gt += (kk > 0 && key > T) ? 1 : 0;
            c_eq += (kk > 0 && key == T) ? 1 : 0;
        }
        const int gt_before = static_cast<int>(block_allreduce(static_cast<float>(c_gt), OpSum(), sRed4));
        const int eq_before = static_cast<int>(block_allreduce(static_cast<float>(c_eq), OpSum(), sRed4));
        const int kept_before = gt_before + min(eq_before, need_eq) + max(0, row0 - M);

        int eq_run = 0, kept_run = 0;
        for (int c0 = 0; c0 < nrows; c0 += kThreads) {
            const int row = c0 + tid;
            const int gi = row0 + row;
            const bool in = row < nrows;
            const bool cand = in && gi < M;
            const uint32_t key = cand ? sKeys[gi] : 0u;
            const bool eq = cand && kk > 0 && key == T;
            int eq_tot;
            const int eq_rank = eq_before + eq_run + block_excl_scan_flag(eq, sInt + 4, eq_tot);
            const bool kept = in && (!cand || (kk > 0 && (key > T || (eq && eq_rank < need_eq))));
            int kept_tot;
            const int dst = kept_before + kept_run + block_excl_scan_flag(kept, sInt + 4, kept_tot);
            if (in) sDst[row] = kept ? dst : -1;
            eq_run += eq_tot;
            kept_run += kept_tot;
        }
        __syncthreads();

        // optional outputs
        if (p.kept_out || p.scores_out) {
            for (int row = tid; row < nrows; row += kThreads) {
                const int gi = row0 + row;
                const int d = sDst[row];
                if (p.kept_out && d >= 0) p.kept_out[unit_g * p.cap + d] = gi;
                if (p.scores_out && gi < M) {
                    float *so = p.scores_out + unit_g * 4 * p.cap;
                    const float I = sIhat[row] / sumI_g;
                    const float Rv = exp2f((sRr[row] - rmax_g) * 1.4426950408889634f) * inv_rsum;
                    so[gi] = I;
                    so[p.cap + gi] = sRr[row];
                    so[2 * p.cap + gi] = Rv;
                    so[3 * p.cap + gi] = joint_score(lam, I, Rv);
                }
            }
        }

        // ---- stage the V rows that move, then wait until the whole unit has read
        const uint16_t *vsrc = p.v[l] + krow0 * kHeadDim;
        int moved = 0;
        for (int row = tid; row < nrows; row += kThreads) {
            const int d = sDst[row];
            if (d >= 0 && d != row0 + row) {
                bulk_g2s(sV + row * 256, vsrc + static_cast<int64_t>(row0 + row) * kHeadDim, 256u,
                         bar_v);
                ++moved;
            }
        }
        moved = static_cast<int>(block_allreduce(static_cast<float>(moved), OpSum(), sRed4));
        if (tid == 0) mbar_arrive_expect_tx(bar_v, static_cast<uint32_t>(moved) * 256u);
        if (!mbar_wait(bar_v, 0)) {
            ok = false;
            record_flag(p.status, kDevFlagTimeout);
        }
        ok = __syncthreads_and(ok);
    }

    // ================= cluster barrier 3: every read of this unit's K and V is done
    cluster.sync();

    if (do_sel && ok) {
        uint16_t *kdst = p.k[l] + krow0 * kHeadDim;
        uint16_t *vdst = p.v[l] + krow0 * kHeadDim;
        for (int idx = tid; idx < nrows * 16; idx += kThreads) {
            const int row = idx >> 4, c = idx & 15;
            const int d = sDst[row];
            if (d < 0 || d == row0 + row) continue;
            const uint4 kx = *reinterpret_cast<const uint4 *>(sK + (c >> 3) * p.rp * 128 +
                                                              sw128_offset(row, c & 7));
            const uint4 vx = *reinterpret_cast<const uint4 *>(sV + row * 256 + c * 16);
            *reinterpret_cast<uint4 *>(kdst + static_cast<int64_t>(d) * kHeadDim + c * 8) = kx;
            *reinterpret_cast<uint4 *>(vdst + static_cast<int64_t>(d) * kHeadDim + c * 8) = vx;
        }
    }

    __syncthreads();
    if (do_imp && warp == 0) {
        tc_fence_before();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
    }
}

size_t step_smem_bytes(int rp, int rmax, int cap, int nqp) {
    return make_layout(rp, rmax, cap, nqp).total;
}

template <int NQP>
static cudaError_t launch_step_t(const StepParams &p, int n_units, size_t smem,
                                 cudaStream_t stream) {
    auto kern = rkv_step_kernel<NQP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (p.cs > 8) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * p.cs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(p.cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_step(const StepParams &p, int n_units, int nqp, size_t smem,
                        cudaStream_t stream) {
    switch (nqp) {
        case 16: return launch_step_t<16>(p, n_units, smem, stream);
        case 32: return launch_step_t<32>(p, n_units, smem, stream);
        case 48: return launch_step_t<48>(p, n_units, smem, stream);
        case 64: return launch_step_t<64>(p, n_units, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rkv
