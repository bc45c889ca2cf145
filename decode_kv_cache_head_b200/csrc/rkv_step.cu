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
// Work decomposition.  One cluster of `cs` CTAs (256 threads each) handles one
// unit of N cached rows; CTA c owns rows [c*R, c*R + R) with R = ceil16(N/cs).
//   1. TMA loads the CTA's K rows and the unit's G*w query rows into shared
//      memory (128-byte swizzle); one bulk copy brings the CTA's V rows.  These
//      are the only reads of K and V, and they finish before barrier 1.
//   2. One thread issues tcgen05 UMMAs: logits[rows, G*w] = K_rows . Q^T into
//      TMEM (M = 128 key rows per tile, N = G*w padded to 16, K = 128).
//   3. Meanwhile all threads compute ||k_i||^2, 1/max(||k_i||, 1e-12) and the
//      CTA's part of S = sum_i khat_i (for the mean-redundancy row sum).
//   4. TMEM epilogue: per-query-column max and sum of exp over the CTA's
//      visible keys.  Every exchange is a push: each CTA stores its partials
//      straight into its slot in every peer's shared memory, so that after a
//      cluster barrier all reads are local (barrier 1).
//   5. Per row: p = softmax probabilities, mean over the window, max over the
//      group -> Ihat_i; r_i = (khat_i . S - khat_i . khat_i) / (N - 1) (MEAN)
//      or r from the similarity kernel (MAX).  (Ihat_i, r_i) and the partial
//      sum Ihat / max r / sum exp(r - max) are pushed to every CTA (barrier 2).
//   6. Every CTA forms Z = lambda Ihat/sum - (1-lambda) exp(r - rmax)/rsum for
//      all candidates and runs the same deterministic radix select (the k-th
//      largest key, ties to the lower index), so all CTAs agree on the kept
//      set without another exchange.
//   7. Each CTA writes its kept rows that move: K from its swizzled tile, V
//      from its staging copy.  Since every read of the unit's K and V finished
//      before barrier 1, these in-place writes cannot clobber a row that some
//      CTA still has to read.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_post.cuh"
#include "rkv_ptx.cuh"

namespace cg = cooperative_groups;

namespace rkv {

// ----------------------------------------------------------------------------
// Plan: clear the status words; which sequences are due; snapshot their length;
// set cur_len = budget; optionally order the sequences by decreasing length.  One
// CTA, so the clearing precedes every flag it records.
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rkv_plan_kernel(int batch, const int32_t *__restrict__ budgets,
                                                       int32_t budget_cfg, int32_t buffer, int32_t window,
                                                       int32_t cap, int32_t *__restrict__ cur_len,
                                                       int32_t *__restrict__ n_eff,
                                                       uint32_t *__restrict__ status, int update,
                                                       RaggedLayout rg, int32_t *__restrict__ order) {
    // the kernel that follows may be scheduled now; it waits for this one to finish
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int i = threadIdx.x; i < static_cast<int>(kStatusBytes / 4); i += blockDim.x) status[i] = 0u;
    __syncthreads();
    for (int b = threadIdx.x; b < batch; b += blockDim.x) {
        const int32_t bud = budgets ? budgets[b] : budget_cfg;
        const int32_t n = cur_len[b];
        // Compression is active only when budget and buffer are both positive.
        bool due = bud > 0 && buffer > 0 && n >= bud + buffer;
        // the sequence's capacity: its own block of a ragged pool, else the uniform one
        int32_t c = cap;
        bool bad_block = false;
        if (due && rg.seq_row) {
            c = rg.seq_cap[b];
            const int64_t r0 = rg.seq_row[b];
            bad_block = c < 2 || c > cap || r0 < 0 ||
                        r0 + static_cast<int64_t>(rg.n_kv) * c > rg.pool_rows;
        }
        if (due && (bud < window || n > c || bad_block)) {
            record_flag(status, kDevFlagBadSeq);
            due = false;
        }
        n_eff[b] = due ? n : 0;
        if (due && update) cur_len[b] = bud;
    }
    if (order == nullptr) return;
    // The sequences by decreasing tile count (ceil(N / 128), 0 when not due): a launch
    // that takes its units in this order starts the longest first and ends on the
    // shortest.  A counting sort over the tile counts; the order inside one count is
    // whichever the atomics give, which changes no result (units are independent).
    constexpr int kBins = 64;
    __shared__ uint32_t cnt[kBins];
    for (int i = threadIdx.x; i < kBins; i += blockDim.x) cnt[i] = 0u;
    __syncthreads();   // also: every n_eff above is written
    auto bin_of = [&](int b) {
        const int n = n_eff[b];
        return n > 0 ? min((n + 127) / 128, kBins - 1) : 0;
    };
    for (int b = threadIdx.x; b < batch; b += blockDim.x) atomicAdd(&cnt[bin_of(b)], 1u);
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;   // start of each bin, the highest bin first
        for (int i = kBins - 1; i >= 0; --i) {
            const uint32_t c = cnt[i];
            cnt[i] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int b = threadIdx.x; b < batch; b += blockDim.x)
        order[atomicAdd(&cnt[bin_of(b)], 1u)] = b;
}

cudaError_t launch_plan(int batch, const int32_t *budgets, int32_t budget_cfg, int32_t buffer,
                        int32_t window, int32_t cap, int32_t *cur_len, int32_t *n_eff,
                        uint32_t *status, cudaStream_t stream, bool update,
                        const RaggedLayout &rg, int32_t *order) {
    return launch_kernel(rkv_plan_kernel, dim3(1), dim3(256), 0, stream, batch, budgets, budget_cfg,
                         buffer, window, cap, cur_len, n_eff, status, update ? 1 : 0, rg, order);
}

// ----------------------------------------------------------------------------
// The fused per-unit kernel.
// ----------------------------------------------------------------------------
// NQP: query columns G*w rounded up to 16.  WC: the window size when it is
// known at compile time (the common w = 8), 0 for a runtime window.
template <int NQP, int WC>
__global__ void __launch_bounds__(kStepThreads, 2) rkv_step_kernel(const __grid_constant__ StepParams p) {
    constexpr int NT = kStepThreads;
    constexpr int NW = NT / 32;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    cg::cluster_group cluster = cg::this_cluster();
    const int cs = p.cs;
    const int rank = static_cast<int>(cluster.block_rank());
    const int unit = blockIdx.x / cs;
    const int h = unit % p.n_kv;
    const int b = (unit / p.n_kv) % p.batch;
    const int l = unit / (p.n_kv * p.batch);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int N = p.n_tokens_fixed > 0 ? p.n_tokens_fixed : p.n_eff[b];
    if (N <= 0) return;  // not due: the whole cluster leaves before any exchange

    const int w = WC > 0 ? WC : p.window;
    const int G = p.group;
    const int NQ = G * w;
    const int M = N - w;
    const int budget = p.budgets ? p.budgets[b] : p.budget_cfg;
    const float lam = p.lambdas ? p.lambdas[b] : p.lambda_cfg;
    const int kk = budget - w;
    const bool do_imp = (p.flags & kFlagImportance) != 0;
    const bool do_sel = (p.flags & kFlagSelect) != 0;
    const bool red_max = p.red_mode == RKV_RED_MAX;
    const bool pool_max = p.gqa_pool == RKV_GQA_MAX;

    const int R = ((N + cs - 1) / cs + 15) / 16 * 16;
    const int row0 = rank * R;
    const int nrows = max(0, min(R, N - row0));
    const int nbox = (nrows + 15) / 16;
    const int nrows_pad = nbox * 16;
    const int ntiles = (nrows_pad + 127) / 128;
    const int64_t krow0 = (static_cast<int64_t>(b) * p.n_kv + h) * p.cap;   // row in the layer's 2D view
    const int64_t unit_g = (static_cast<int64_t>(p.layer_base + l) * p.batch + b) * p.n_kv + h;

    const SmemLayout L = make_layout(p.rp, p.rmax, p.cap, NQP, cs);
    uint8_t *sK = base + L.k;
    uint8_t *sQ = base + L.q;                                     // until the UMMAs complete
    uint8_t *sV = base + L.v;
    float2 *xIR = reinterpret_cast<float2 *>(base + L.x);         // after barrier 1
    uint32_t *sKeys = reinterpret_cast<uint32_t *>(base + L.x);   // key of candidate j at [2j]
    float *sScratch = reinterpret_cast<float *>(base + L.scratch);  // before barrier 1 only
    float *sInv = reinterpret_cast<float *>(base + L.inv);
    float *sSS = reinterpret_cast<float *>(base + L.ss);
    float *sIhat = reinterpret_cast<float *>(base + L.ihat);
    float *sRr = reinterpret_cast<float *>(base + L.rr);
    int32_t *sDst = reinterpret_cast<int32_t *>(base + L.dst);
    float *xStatM = reinterpret_cast<float *>(base + L.xstatm);
    float *xStatL = reinterpret_cast<float *>(base + L.xstatl);
    float4 *xS = reinterpret_cast<float4 *>(base + L.xs);
    float *sGS = reinterpret_cast<float *>(base + L.gs);
    float *sSpart = reinterpret_cast<float *>(base + L.spart);
    float *sGM = reinterpret_cast<float *>(base + L.gm);
    float *sGLinv = reinterpret_cast<float *>(base + L.glinv);
    uint64_t *sVis = reinterpret_cast<uint64_t *>(base + L.vis);
    uint32_t *sHist = reinterpret_cast<uint32_t *>(base + L.hist);
    float *sRed = reinterpret_cast<float *>(base + L.red);
    uint32_t *sRedU = reinterpret_cast<uint32_t *>(base + L.red);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + L.bars);
    uint64_t *bar_tma = bars + 0, *bar_mma = bars + 1;
    uint32_t *sTmem = reinterpret_cast<uint32_t *>(bars + 4);

    // Query columns q = g * w + j.  colmask: columns that exist; lastmask: the
    // last window query of each head (where the window mean is complete).
    uint64_t colmask, lastmask;
    {
        const int j0 = lane % w, j1 = (lane + 32) % w;
        colmask = static_cast<uint64_t>(__ballot_sync(kFull, lane < NQ)) |
                  (static_cast<uint64_t>(__ballot_sync(kFull, lane + 32 < NQ)) << 32);
        lastmask = static_cast<uint64_t>(__ballot_sync(kFull, lane < NQ && j0 == w - 1)) |
                   (static_cast<uint64_t>(__ballot_sync(kFull, lane + 32 < NQ && j1 == w - 1)) << 32);
        // key M + d (a window key) is seen by query j only when j >= d (causal)
        if (warp == 0) {
            for (int d = 0; d < w; ++d) {
                const uint64_t m = static_cast<uint64_t>(__ballot_sync(kFull, lane < NQ && j0 >= d)) |
                                   (static_cast<uint64_t>(__ballot_sync(kFull, lane + 32 < NQ && j1 >= d)) << 32);
                if (lane == 0) sVis[d] = m;
            }
        }
    }

    bool ok = true;  // false after a timed-out wait: keep joining barriers, skip the writes

    // ---- set-up: TMEM, barriers, loads (K and Q by TMA, this CTA's V rows by one bulk copy)
    if (do_imp && warp == 0) {
        tmem_alloc(sTmem, static_cast<uint32_t>(p.tmem_cols));
        tmem_relinquish();
    }
    // warp 1 starts the loads while warp 0 allocates TMEM
    if (tid == 32) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (tid == 32 && nrows > 0) {
        const CUtensorMap *mk = &p.tmap_k[l];
        const uint32_t bytes = static_cast<uint32_t>(nbox) * 4096u +
                               (do_imp ? static_cast<uint32_t>(NQP) * 256u : 0u) +
                               (do_sel ? static_cast<uint32_t>(nrows) * 256u : 0u);
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
        if (do_sel)
            bulk_g2s(sV, p.v[l] + (krow0 + row0) * kHeadDim, static_cast<uint32_t>(nrows) * 256u,
                     bar_tma);
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = do_imp ? *sTmem : 0u;

    if (nrows > 0 && !mbar_wait(bar_tma, 0)) {
        ok = false;
        record_flag(p.status, kDevFlagTimeout);
    }

    // ---- UMMA: logits of every row against the G*w window queries
    auto tile_start = [&](int t) { return t < ntiles - 1 ? t * 128 : max(0, nrows_pad - 128); };
    if (do_imp && nrows > 0 && tid == kStepThreads - 32) {
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

    // Rows: thread tid takes tiles t = tid/128, tid/128 + 2, ..., row tile_start(t) + tid%128,
    // which is also the TMEM lane its warp reads.
    const int t_first = tid >> 7, lane_row = tid & 127;
    const uint32_t tmem_warp = tmem_base + ((32u * static_cast<uint32_t>(warp & 3)) << 16);

    // ---- norms while the tensor cores work
    for (int t = t_first; t < ntiles; t += 2) {
        const int row = tile_start(t) + lane_row;
        if (row < t * 128 || row >= nrows) continue;
        float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int c = 0; c < 16; ++c) {
            const uint4 raw = *reinterpret_cast<const uint4 *>(sK + (c >> 3) * p.rp * 128 +
                                                               sw128_offset(row, c & 7));
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                ss2 = __ffma2_rn(f, f, ss2);
            }
        }
        const float ss = ss2.x + ss2.y;
        sSS[row] = ss;
        sInv[row] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
    __syncthreads();

    // ---- this CTA's part of S = sum_i khat_i, pushed into every CTA's slot `rank`
    if (!red_max) {
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
        const int half = lane >> 4, cc = (lane & 15) >> 1, sub = lane & 1;
        for (int row = warp; row < nrows; row += NW) {
            const uint2 raw = *reinterpret_cast<const uint2 *>(sK + half * p.rp * 128 +
                                                               sw128_offset(row, cc) + sub * 8);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
            const float iv = sInv[row];
            const float2 iv2 = make_float2(iv, iv);
            acc0 = __ffma2_rn(__bfloat1622float2(h2[0]), iv2, acc0);
            acc1 = __ffma2_rn(__bfloat1622float2(h2[1]), iv2, acc1);
        }
        const int col = half * 64 + (lane & 15) * 4;
        *reinterpret_cast<float4 *>(sScratch + warp * 128 + col) = make_float4(acc0.x, acc0.y, acc1.x, acc1.y);
        __syncthreads();
        if (tid < 128) {
            float s = sScratch[tid];
#pragma unroll
            for (int w2 = 1; w2 < NW; ++w2) s += sScratch[w2 * 128 + tid];
            sSpart[tid] = s;
        }
        __syncthreads();
        const float4 *sp4 = reinterpret_cast<const float4 *>(sSpart);
        for (int i = tid; i < cs * 32; i += NT)
            cluster.map_shared_rank(xS, i >> 5)[rank * 32 + (i & 31)] = sp4[i & 31];
    }

    // ---- softmax statistics of the CTA's visible keys for every query column
    const float sc = p.logit_scale_log2;
    if (do_imp) {
        if (nrows > 0) {
            if (!mbar_wait(bar_mma, 0)) {
                ok = false;
                record_flag(p.status, kDevFlagTimeout);
            }
            tc_fence_after();
        }
        float *sRedQ = sScratch + NW * 128;   // [NW][NQP]
        const bool nopad = (NQ == NQP);
        // pass 1: column max (log2 domain)
        {
            float cm[NQP];
#pragma unroll
            for (int q = 0; q < NQP; ++q) cm[q] = -INFINITY;
            for (int t = t_first; t < ntiles; t += 2) {
                const int row = tile_start(t) + lane_row;
                const int gi = row0 + row;
                const bool valid = row >= t * 128 && row < nrows;
                // warp-uniform fast path: every row a candidate, every column real
                const bool fast = nopad && __all_sync(kFull, valid && gi < M);
                const uint64_t rm = !valid ? 0ull : (gi < M ? colmask : sVis[gi - M]);
#pragma unroll
                for (int c0 = 0; c0 < NQP; c0 += 16) {
                    float v[16];
                    tmem_ld16(tmem_warp + t * NQP + c0, v);
                    if (fast) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) cm[c0 + i] = fmaxf(cm[c0 + i], v[i] * sc);
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            cm[c0 + i] = fmaxf(cm[c0 + i], ((rm >> (c0 + i)) & 1ull) ? v[i] * sc : -INFINITY);
                    }
                }
            }
#pragma unroll
            for (int c0 = 0; c0 < NQP; c0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = cm[c0 + i];
                warp_transpose_reduce16(v, OpMax());
                if (lane < 16) sRedQ[warp * NQP + c0 + lane] = v[0];
            }
        }
        __syncthreads();
        if (tid < NQP) {
            float m = sRedQ[tid];
#pragma unroll
            for (int w2 = 1; w2 < NW; ++w2) m = fmaxf(m, sRedQ[w2 * NQP + tid]);
            sGM[tid] = m;    // local column max (pushed to the cluster below)
        }
        __syncthreads();
        // pass 2: exp2(s - local max), written back to TMEM (zero where not visible),
        // and its column sums
        {
            float cl[NQP];
#pragma unroll
            for (int q = 0; q < NQP; ++q) cl[q] = 0.f;
            for (int t = t_first; t < ntiles; t += 2) {
                const int row = tile_start(t) + lane_row;
                const int gi = row0 + row;
                const bool valid = row >= t * 128 && row < nrows;
                const bool fast = nopad && __all_sync(kFull, valid && gi < M);
                const uint64_t rm = !valid ? 0ull : (gi < M ? colmask : sVis[gi - M]);
#pragma unroll
                for (int c0 = 0; c0 < NQP; c0 += 16) {
                    float v[16], mq[16];
                    tmem_ld16(tmem_warp + t * NQP + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i) mq[i] = sGM[c0 + i];
                    if (fast) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            v[i] = ex2_approx(fmaf(v[i], sc, -mq[i]));
                            cl[c0 + i] += v[i];
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float e = ex2_approx(fmaf(v[i], sc, -mq[i]));
                            v[i] = ((rm >> (c0 + i)) & 1ull) ? e : 0.f;
                            cl[c0 + i] += v[i];
                        }
                    }
                    tmem_st16(tmem_warp + t * NQP + c0, v);
                }
            }
#pragma unroll
            for (int c0 = 0; c0 < NQP; c0 += 16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = cl[c0 + i];
                warp_transpose_reduce16(v, OpSum());
                if (lane < 16) sRedQ[warp * NQP + c0 + lane] = v[0];
            }
            tmem_wait_st();
        }
        __syncthreads();
        for (int i = tid; i < cs * NQP; i += NT) {
            const int q = i % NQP;
            float s = sRedQ[q];
#pragma unroll
            for (int w2 = 1; w2 < NW; ++w2) s += sRedQ[w2 * NQP + q];
            const int peer = i / NQP;
            cluster.map_shared_rank(xStatM, peer)[rank * NQP + q] = sGM[q];
            cluster.map_shared_rank(xStatL, peer)[rank * NQP + q] = s;
        }
    }

    // ================= cluster barrier 1: column statistics and S partials delivered
    cluster.sync();

    // Cluster-wide column statistics and S: thread t takes CTA slot t % cs of
    // column t / cs and the cs slots are folded with shuffles inside groups of
    // cs lanes (same order in every CTA, so every CTA gets the same bits).
    {
        const int per = NT / cs;   // columns per pass
        const int c = tid % cs, col = tid / cs;
        if (do_imp) {
            for (int q0 = 0; q0 < NQP; q0 += per) {
                const int q = q0 + col;
                const float mc = (q < NQP) ? xStatM[c * NQP + q] : -INFINITY;
                float m = mc;
                for (int off = 1; off < cs; off <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
                float lsum = (mc != -INFINITY && q < NQP) ? xStatL[c * NQP + q] * ex2_approx(mc - m) : 0.f;
                for (int off = 1; off < cs; off <<= 1) lsum += __shfl_xor_sync(kFull, lsum, off);
                if (c == 0 && q < NQP) {
                    // probabilities = (stored exp relative to this CTA's max) * factor
                    const float mloc = xStatM[rank * NQP + q];
                    sGLinv[q] = (lsum > 0.f && mloc != -INFINITY) ? ex2_approx(mloc - m) / lsum : 0.f;
                }
            }
        }
        if (!red_max) {
            for (int d0 = 0; d0 < 32; d0 += per) {
                const int d4 = d0 + col;
                float4 v = (d4 < 32) ? xS[c * 32 + d4] : make_float4(0.f, 0.f, 0.f, 0.f);
                for (int off = 1; off < cs; off <<= 1) {
                    v.x += __shfl_xor_sync(kFull, v.x, off);
                    v.y += __shfl_xor_sync(kFull, v.y, off);
                    v.z += __shfl_xor_sync(kFull, v.z, off);
                    v.w += __shfl_xor_sync(kFull, v.w, off);
                }
                if (c == 0 && d4 < 32) reinterpret_cast<float4 *>(sGS)[d4] = v;
            }
        }
    }
    __syncthreads();

    // ---- per row: importance Ihat_i, redundancy r_i; pushed to every CTA
    const float inv_w = 1.0f / static_cast<float>(w);
    const float inv_nm1 = 1.0f / static_cast<float>(N - 1);
    for (int t = t_first; t < ntiles; t += 2) {
        const int row = tile_start(t) + lane_row;
        const bool valid = row >= t * 128 && row < nrows;
        const int gi = row0 + row;
        float ihat = 0.f;
        if (do_imp) {
            // warp-collective loads: every lane takes part, valid or not
            // TMEM now holds exp2(s - local max), zero where the key is not visible;
            // probability = that value * per-column factor
            float run = 0.f, best = pool_max ? -INFINITY : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < NQP; c0 += 16) {
                float v[16], fq[16];
                tmem_ld16(tmem_warp + t * NQP + c0, v);
#pragma unroll
                for (int i = 0; i < 16; ++i) fq[i] = sGLinv[c0 + i];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int q = c0 + i;
                    run = fmaf(v[i], fq[i], run);
                    if (WC > 0) {
                        if (q % (WC > 0 ? WC : 1) == WC - 1) {   // compile time: end of a head
                            const float a = run * inv_w;
                            best = pool_max ? fmaxf(best, a) : best + a;
                            run = 0.f;
                        }
                    } else {
                        const bool last = (lastmask >> q) & 1ull;
                        const float a = run * inv_w;
                        best = last ? (pool_max ? fmaxf(best, a) : best + a) : best;
                        run = last ? 0.f : run;
                    }
                }
            }
            ihat = pool_max ? best : best / static_cast<float>(G);
        }
        if (!valid || gi >= M) continue;
        float r;
        if (red_max) {
            r = p.r_ext[unit_g * p.cap + gi];
        } else {
            float2 dot2 = make_float2(0.f, 0.f);
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(sK + (c >> 3) * p.rp * 128 +
                                                                   sw128_offset(row, c & 7));
                const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
                const float4 s0 = *reinterpret_cast<const float4 *>(sGS + c * 8);
                const float4 s1 = *reinterpret_cast<const float4 *>(sGS + c * 8 + 4);
                dot2 = __ffma2_rn(__bfloat1622float2(h2[0]), make_float2(s0.x, s0.y), dot2);
                dot2 = __ffma2_rn(__bfloat1622float2(h2[1]), make_float2(s0.z, s0.w), dot2);
                dot2 = __ffma2_rn(__bfloat1622float2(h2[2]), make_float2(s1.x, s1.y), dot2);
                dot2 = __ffma2_rn(__bfloat1622float2(h2[3]), make_float2(s1.z, s1.w), dot2);
            }
            const float dot = dot2.x + dot2.y;
            const float iv = sInv[row];
            r = (iv * dot - iv * iv * sSS[row]) * inv_nm1;
        }
        sIhat[row] = ihat;
        sRr[row] = r;
        const float2 ir = make_float2(ihat, r);
        for (int c = 0; c < cs; ++c) cluster.map_shared_rank(xIR, c)[gi] = ir;
    }
    // ================= cluster barrier 2: every candidate's (Ihat, r) delivered.
    // No CTA reads another's shared memory after this point, and every read of
    // this unit's K and V in global memory finished before barrier 1.
    cluster.sync();

    // Normalisers and keys from the local copies of every candidate's (Ihat, r):
    // identical data and order in every CTA, hence identical bits everywhere.
    float inv_sumI, rmax_g, inv_rsum;
    uint32_t T = 0xffffffffu;
    int n_gt = 0;
    {
        const bool sel = do_sel && nrows > 0;
        post_scores_any<NT, 2>([&](int j) { return xIR[j]; }, sKeys, sHist, sRed, M, kk, lam, sel,
                               inv_sumI, rmax_g, inv_rsum, T, n_gt);
    }

    if (p.flags & kFlagOutScores) {
        // per-head entry points: write this CTA's rows
        for (int t = t_first; t < ntiles; t += 2) {
            const int row = tile_start(t) + lane_row;
            const int gi = row0 + row;
            if (row < t * 128 || row >= nrows) continue;
            if (p.out_inv) p.out_inv[static_cast<int64_t>(h) * N + gi] = sInv[row];
            if (gi < M) {
                const int64_t o = static_cast<int64_t>(h) * M + gi;
                if (p.out_I) p.out_I[o] = sIhat[row] * inv_sumI;
                if (p.out_r) p.out_r[o] = sRr[row];
                if (p.out_R) p.out_R[o] = ex2_approx((sRr[row] - rmax_g) * kLog2e) * inv_rsum;
            }
        }
    }

    if (do_sel && nrows > 0) {
        const int need_eq = (kk > 0) ? kk - n_gt : 0;

        // counts of candidates above / tied with the threshold before this CTA's rows
        const int lim = min(row0, M);
        uint32_t packed = 0;
        if (kk > 0)
            for (int j = tid; j < lim; j += NT) {
                const uint32_t key = sKeys[2 * j];
                packed += (key > T ? 1u : 0u) + (key == T ? 65536u : 0u);
            }
        packed = block_sum_u32<NT>(packed, sRedU);
        uint32_t g_run = (packed & 0xffffu) + static_cast<uint32_t>(max(0, row0 - M));
        uint32_t e_run = packed >> 16;

        // kept flag and destination of each row: G_i = rows above the threshold or
        // in the window before i, E_i = tied candidates before i;
        // kept = above || window || (tied && E_i < need_eq), dst = G_i + min(E_i, need_eq)
        for (int c0 = 0; c0 < nrows; c0 += NT) {
            const int row = c0 + tid;
            const int gi = row0 + row;
            const bool in = row < nrows;
            const bool cand = in && gi < M;
            const uint32_t key = cand ? sKeys[2 * gi] : 0u;
            const bool eq = cand && kk > 0 && key == T;
            const bool gw = in && (!cand || (kk > 0 && key > T));
            uint32_t tot2;
            const uint32_t ex = block_excl_scan_u32<NT>((eq ? 65536u : 0u) + (gw ? 1u : 0u), sRedU, tot2);
            const uint32_t Ei = e_run + (ex >> 16), Gi = g_run + (ex & 0xffffu);
            const bool kept = gw || (eq && Ei < static_cast<uint32_t>(need_eq));
            if (in) sDst[row] = kept ? static_cast<int32_t>(Gi + min(Ei, static_cast<uint32_t>(need_eq))) : -1;
            e_run += tot2 >> 16;
            g_run += tot2 & 0xffffu;
        }
        __syncthreads();

        // optional outputs
        if (p.kept_out || p.scores_out) {
            for (int row = tid; row < nrows; row += NT) {
                const int gi = row0 + row;
                const int d = sDst[row];
                if (p.kept_out && d >= 0) p.kept_out[unit_g * p.cap + d] = gi;
                if (p.scores_out && gi < M) {
                    float *so = p.scores_out + unit_g * 4 * p.cap;
                    const float I = sIhat[row] * inv_sumI;
                    const float Rv = ex2_approx((sRr[row] - rmax_g) * kLog2e) * inv_rsum;
                    so[gi] = I;
                    so[p.cap + gi] = sRr[row];
                    so[2 * p.cap + gi] = Rv;
                    so[3 * p.cap + gi] = joint_score(lam, I, Rv);
                }
            }
        }

        // ---- compaction: kept rows that move, K from its swizzled tile, V from its staging
        ok = __syncthreads_and(ok);
        if (ok) {
            uint16_t *kdst = p.k[l] + krow0 * kHeadDim;
            uint16_t *vdst = p.v[l] + krow0 * kHeadDim;
            for (int idx = tid; idx < nrows * 16; idx += NT) {
                const int row = idx >> 4, c = idx & 15;
                const int d = sDst[row];
                if (d < 0 || d == row0 + row) continue;
                const uint4 kx = *reinterpret_cast<const uint4 *>(sK + (c >> 3) * p.rp * 128 +
                                                                  sw128_offset(row, c & 7));
                const uint4 vx = *reinterpret_cast<const uint4 *>(sV + row * 256 + c * 16);
                __stcs(reinterpret_cast<uint4 *>(kdst + static_cast<int64_t>(d) * kHeadDim + c * 8), kx);
                __stcs(reinterpret_cast<uint4 *>(vdst + static_cast<int64_t>(d) * kHeadDim + c * 8), vx);
            }
        }
    }

    __syncthreads();
    if (do_imp && warp == 0) {
        tc_fence_before();
        tmem_dealloc(tmem_base, static_cast<uint32_t>(p.tmem_cols));
    }
}

size_t step_smem_bytes(int rp, int rmax, int cap, int nqp, int cs) {
    return make_layout(rp, rmax, cap, nqp, cs).total;
}

template <int NQP, int WC>
static cudaError_t launch_step_t(const StepParams &p, int n_units, size_t smem,
                                 cudaStream_t stream) {
    auto kern = rkv_step_kernel<NQP, WC>;
    static std::atomic<int> granted{0};
    static std::atomic<bool> nonportable{false};
    cudaError_t e = ensure_smem_attr(kern, smem, granted);
    if (e != cudaSuccess) return e;
    if (p.cs > 8 && !nonportable.load()) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        nonportable.store(true);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * p.cs), 1, 1);
    cfg.blockDim = dim3(kStepThreads, 1, 1);
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
    if (p.window == 8) {   // the window of every R-KV configuration on the pages
        switch (nqp) {
            case 16: return launch_step_t<16, 8>(p, n_units, smem, stream);
            case 32: return launch_step_t<32, 8>(p, n_units, smem, stream);
            case 48: return launch_step_t<48, 8>(p, n_units, smem, stream);
            case 64: return launch_step_t<64, 8>(p, n_units, smem, stream);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (nqp) {
        case 16: return launch_step_t<16, 0>(p, n_units, smem, stream);
        case 32: return launch_step_t<32, 0>(p, n_units, smem, stream);
        case 48: return launch_step_t<48, 0>(p, n_units, smem, stream);
        case 64: return launch_step_t<64, 0>(p, n_units, smem, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rkv
