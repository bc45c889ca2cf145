// rkv_gram.cu -- MAX-mode redundancy on the tensor cores:
//   r_i = max_{j < N, j != i} khat_i . khat_j,  khat = k / max(||k||, 1e-12),
// for every candidate i < M of every due unit.  Redundancy is the cosine
// similarity of key vectors ("R-KV: Redundancy-aware KV Cache Compression for
// Reasoning Models", atlas.scime.ai summary, "Approach"); the max over the
// other keys is the near-duplicate reading of "cosine similarity to identify
// and prune near-duplicates" (sourcepulse summary, "How It Works").
//
// One CTA per (unit, block of 128 candidate rows).  The Gram tiles
// K_I . K_J^T are computed by tcgen05 UMMA (bf16 in, fp32 accumulate) into
// TMEM and folded to row maxima on chip; the N x N matrix never reaches HBM.
// A first pass (rkv_inv_norm_kernel) writes 1 / max(||k_j||, 1e-12) of every
// row once, so the row blocks of a unit do not each recompute the norms of
// every column tile.
// Warp roles (320 threads):
//   warps 0-7  epilogue: per row max_j acc_ij * inv_j from TMEM; warps w and
//              w + 4 read the same 32 TMEM lanes (rows) and split the tile's
//              128 columns;
//   warp 8     producer: TMA of the row block once, then 128-row column tiles
//              into a two-stage ring;
//   warp 9     MMA issuer: 8 UMMAs (K = 128) per column tile into one of two
//              TMEM accumulators (128 columns each).
// Hand-offs are mbarriers; every wait is bounded and a timeout is recorded in
// the status word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace rkv {

namespace {

constexpr int kGramThreads = 320;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = 128u * 256u;      // 128 rows x 128 bf16
constexpr uint32_t kTmemCols = 256;               // two 128-column accumulators

struct GramSmem {
    uint8_t a[kTileBytes];                 // row block (two 64-column halves)
    uint8_t b[kStages][kTileBytes];        // column tiles
    float inv_b[2][128];                   // inverse norms of the column tile in each accumulator
    float inv_a[128];
    float part[128];                       // row maxima of the second column half
    uint64_t bar_a;
    uint64_t full[kStages], empty[kStages];
    uint64_t tfull[2], tempty[2];
    uint32_t tmem;
};

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max(best, c[0..31]) as a tree of three-input maxima.
__device__ __forceinline__ float max_of_32(float best, const float (&c)[32]) {
    float t[11];
#pragma unroll
    for (int q = 0; q < 10; ++q) t[q] = fmax3(c[3 * q], c[3 * q + 1], c[3 * q + 2]);
    t[10] = fmaxf(c[30], c[31]);
    const float u0 = fmax3(t[0], t[1], t[2]), u1 = fmax3(t[3], t[4], t[5]);
    const float u2 = fmax3(t[6], t[7], t[8]), u3 = fmax3(t[9], t[10], best);
    return fmax3(u0, u1, fmaxf(u2, u3));
}

__device__ __forceinline__ void named_sync_epilogue() {
    asm volatile("bar.sync 1, 256;" ::: "memory");
}

}  // namespace

__global__ void __launch_bounds__(kGramThreads, 1) rkv_gram_max_kernel(const __grid_constant__ GramParams p) {
    extern __shared__ uint8_t smem_raw[];
    GramSmem &S = *reinterpret_cast<GramSmem *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    // a programmatic dependent of the inverse-norm pass: wait for it before reading
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x / p.nblk, bi = blockIdx.x % p.nblk;
    const int h = unit % p.n_kv;
    const int b = (unit / p.n_kv) % p.batch;
    const int l = unit / (p.n_kv * p.batch);
    const int N = p.n_tokens_fixed > 0 ? p.n_tokens_fixed : p.n_eff[b];
    const int M = N - p.window;
    const int i0 = bi * 128;
    if (N <= 0 || i0 >= M) return;
    const int n_tiles = (N + 127) / 128;
    const int64_t krow0 = (static_cast<int64_t>(b) * p.n_kv + h) * p.cap;
    const int64_t unit_g = (static_cast<int64_t>(p.layer_base + l) * p.batch + b) * p.n_kv + h;
    const CUtensorMap *map = &p.tmap[l];

    if (warp == 0) {
        tmem_alloc(&S.tmem, kTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&S.bar_a, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1);
            mbar_init(&S.empty[s], 1);   // the MMA is done reading the tile
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&S.tfull[t], 1);
            mbar_init(&S.tempty[t], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = S.tmem;
    bool ok = true;

    if (warp == 8) {
        // ---------------- producer
        if (lane == 0) {
            mbar_arrive_expect_tx(&S.bar_a, kTileBytes);
            tma_load_2d(S.a, map, &S.bar_a, 0, static_cast<int32_t>(krow0 + i0));
            tma_load_2d(S.a + 16384, map, &S.bar_a, 64, static_cast<int32_t>(krow0 + i0));
            for (int jt = 0; jt < n_tiles && ok; ++jt) {
                const int s = jt % kStages;
                if (jt >= kStages && !mbar_wait(&S.empty[s], ((jt / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&S.full[s], kTileBytes);
                const int32_t y = static_cast<int32_t>(krow0 + jt * 128);
                tma_load_2d(S.b[s], map, &S.full[s], 0, y);
                tma_load_2d(S.b[s] + 16384, map, &S.full[s], 64, y);
            }
        }
    } else if (warp == 9) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(128, 128);
            if (!mbar_wait(&S.bar_a, 0)) ok = false;
            tc_fence_after();
            const uint32_t a_base = smem_u32(S.a);
            for (int jt = 0; jt < n_tiles && ok; ++jt) {
                const int s = jt % kStages, t = jt & 1;
                if (!mbar_wait(&S.full[s], (jt / kStages) & 1)) { ok = false; break; }
                if (jt >= 2 && !mbar_wait(&S.tempty[t], ((jt >> 1) - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t b_base = smem_u32(S.b[s]);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384u + (ks & 3) * 32u;
                    umma_bf16(tmem_base + t * 128u, desc_kmajor_sw128(a_base + off),
                              desc_kmajor_sw128(b_base + off), idesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&S.tfull[t]);
                umma_commit(&S.empty[s]);
            }
        }
    } else {
        // ---------------- epilogue warps 0-7: row i0 + (tid & 127), column half tid >> 7
        const int lrow = tid & 127, chalf = tid >> 7;
        const int i = i0 + lrow;
        const float *inv_g = p.inv + unit_g * p.cap;
        if (tid < 128) {
            S.inv_a[tid] = (i0 + tid < N) ? inv_g[i0 + tid] : 0.f;
            S.inv_b[0][tid] = (tid < N) ? inv_g[tid] : 0.f;
        }
        named_sync_epilogue();
        float best = -INFINITY;
        for (int jt = 0; jt < n_tiles; ++jt) {
            const int t = jt & 1;
            // the next tile's inverse norms: loaded now, stored after this tile's epilogue
            float nxt = 0.f;
            if (tid < 128 && jt + 1 < n_tiles && (jt + 1) * 128 + tid < N) nxt = inv_g[(jt + 1) * 128 + tid];
            if (ok && !mbar_wait(&S.tfull[t], (jt >> 1) & 1)) ok = false;
            tc_fence_after();
            const int j0 = jt * 128 + chalf * 64;
            const bool clean = (jt * 128 + 128 <= N) && (jt != bi);
            const uint32_t taddr = tmem_base + ((32u * (warp & 3)) << 16) + t * 128u + chalf * 64u;
            const float *invt = &S.inv_b[t][chalf * 64];
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                // 32 columns in flight per wait
                uint32_t r0[16], r1[16];
                tmem_ld16_nowait(taddr + c0, r0);
                tmem_ld16_nowait(taddr + c0 + 16, r1);
                tmem_wait_ld();
                reg_tie16(r0);
                reg_tie16(r1);
                float c[32];
                const float4 *iv4 = reinterpret_cast<const float4 *>(invt + c0);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 iv = iv4[q];
                    const uint32_t *rr = q < 4 ? &r0[4 * q] : &r1[4 * (q - 4)];
                    const float2 a = __fmul2_rn(make_float2(__uint_as_float(rr[0]), __uint_as_float(rr[1])),
                                                make_float2(iv.x, iv.y));
                    const float2 bb = __fmul2_rn(make_float2(__uint_as_float(rr[2]), __uint_as_float(rr[3])),
                                                 make_float2(iv.z, iv.w));
                    c[4 * q] = a.x; c[4 * q + 1] = a.y; c[4 * q + 2] = bb.x; c[4 * q + 3] = bb.y;
                }
                if (clean) {
                    best = max_of_32(best, c);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int j = j0 + c0 + e;
                        best = (j < N && j != i) ? fmaxf(best, c[e]) : best;
                    }
                }
            }
            if (tid < 128 && jt + 1 < n_tiles) S.inv_b[t ^ 1][tid] = nxt;   // read last in tile jt - 1
            tc_fence_before();
            named_sync_epilogue();
            if (tid == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&S.tempty[t])) : "memory");
        }
        if (chalf == 1) S.part[lrow] = best;
        named_sync_epilogue();
        if (chalf == 0 && i < M) p.r_out[unit_g * p.cap + i] = fmaxf(best, S.part[lrow]) * S.inv_a[lrow];
    }
    if (!ok) record_flag(p.status, kDevFlagTimeout);
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// 1 / max(||k_j||, 1e-12) of every row of every due unit: half a warp per row
// (16 lanes x 8 columns), 64 rows per CTA.
__global__ void __launch_bounds__(256) rkv_inv_norm_kernel(const __grid_constant__ GramParams p,
                                                           int nchunk) {
    // a programmatic dependent of the plan kernel: wait for it before reading
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int unit = blockIdx.x / nchunk, chunk = blockIdx.x % nchunk;
    const int h = unit % p.n_kv;
    const int b = (unit / p.n_kv) % p.batch;
    const int l = unit / (p.n_kv * p.batch);
    const int N = p.n_tokens_fixed > 0 ? p.n_tokens_fixed : p.n_eff[b];
    if (N <= 0 || chunk * 64 >= N) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, half = lane >> 4, sub = lane & 15;
    const int64_t krow0 = (static_cast<int64_t>(b) * p.n_kv + h) * p.cap;
    const int64_t unit_g = (static_cast<int64_t>(p.layer_base + l) * p.batch + b) * p.n_kv + h;
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int row = chunk * 64 + warp * 8 + it * 2 + half;
        float2 ss2 = make_float2(0.f, 0.f);
        if (row < N) {
            const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(p.k[l] + (krow0 + row) * kHeadDim) + sub);
            const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(h2[e]);
                ss2 = __ffma2_rn(f, f, ss2);
            }
        }
        float ss = ss2.x + ss2.y;
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) ss += __shfl_xor_sync(kFull, ss, off);
        if (row < N && sub == 0) p.inv[unit_g * p.cap + row] = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
    }
}

size_t gram_smem_bytes() { return sizeof(GramSmem) + 1024; }

cudaError_t launch_gram_max(const GramParams &p, int n_units, cudaStream_t stream,
                            cudaEvent_t before_gram, cudaEvent_t after_gram) {
    const size_t smem = gram_smem_bytes();
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem_attr(rkv_gram_max_kernel, smem, granted);
    if (e != cudaSuccess) return e;
    const int nchunk = (p.cap + 63) / 64;
    // both launched as programmatic dependents of the kernel before them: their CTAs may
    // be scheduled while it finishes, and wait for it on the device
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * nchunk), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, rkv_inv_norm_kernel, p, nchunk);
    if (e == cudaSuccess && before_gram) e = cudaEventRecord(before_gram, stream);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * p.nblk), 1, 1);
    cfg.blockDim = dim3(kGramThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&cfg, rkv_gram_max_kernel, p);
    if (e == cudaSuccess && after_gram) e = cudaEventRecord(after_gram, stream);
    return e;
}

}  // namespace rkv
