// rkv_shared.cu -- shared selection: every KV head of a (sequence, layer)
// keeps the same tokens, chosen by the sum over the heads of their joint
// scores.  With the heads split over tensor-parallel ranks, each rank sums
// its own heads, an all-reduce (sum) over the ranks completes the score and
// every rank then evicts the identical set (the hysenlabs write-up of
// "R-KV: Redundancy-aware KV Cache Compression for Reasoning Models",
// decode-time section: the vLLM port's cross-rank eviction-score all-reduce).
//
// Two kernels around the per-head scoring (rkv_unit_kernel in scores-only
// mode writes Z of every head):
//   rkv_head_sum_kernel            z_sum[l][b][i] = sum_h Z[l][b][h][i], h ascending
//   rkv_shared_compact_kernel      one CTA per (layer, sequence, head): the top
//                                  budget - w candidates of z_sum by (score desc,
//                                  index asc) plus the window -- the same select
//                                  in every CTA of a (layer, sequence), so the
//                                  destinations never leave shared memory -- then
//                                  the head's in-place compaction in ascending
//                                  chunks of 128 rows
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace rkv {

namespace {
constexpr int kSelThreads = 256;
constexpr int kChunkRows = 128;
}

// Every entry of z_sum is written: the head sum for candidates of due
// sequences, 0 elsewhere (so that an all-reduce over ranks sees defined data).
__global__ void __launch_bounds__(256) rkv_head_sum_kernel(const SharedParams p) {
    // a programmatic dependent of the scoring kernel: wait for it before reading
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int nch = (p.cap + 255) / 256;
    const int lb = blockIdx.x / nch;                 // layer * batch + sequence
    const int b = lb % p.batch;
    const int N = p.n_eff[b];
    const int M = N - p.window;
    const int i = (blockIdx.x % nch) * blockDim.x + threadIdx.x;
    if (i >= p.cap) return;
    float s = 0.f;
    if (N > 0 && i < M) {
        const float *z = p.z_heads + static_cast<int64_t>(lb) * p.n_kv * p.cap + i;
        s = z[0];
        for (int h = 1; h < p.n_kv; ++h) s += z[static_cast<int64_t>(h) * p.cap];
    }
    p.z_sum[static_cast<int64_t>(lb) * p.cap + i] = s;
}

// Keys of z_sum, the radix select and the destination of every row (sDst).
template <int KPT>
__device__ __forceinline__ void shared_select_body(const SharedParams &p, int lb, int N, int M,
                                                   int kk, bool write_kept, uint32_t *sKeys,
                                                   int32_t *sDst, uint32_t *sHist,
                                                   uint32_t *sRedU) {
    constexpr int NT = kSelThreads;
    const int tid = threadIdx.x;
    const float *z = p.z_sum + static_cast<int64_t>(lb) * p.cap;
    uint32_t kr[KPT];
    bool kv[KPT];
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        const int j = tid + k * NT;
        kv[k] = j < M;
        kr[k] = kv[k] ? ordered_key(z[j]) : 0u;
        if (kv[k]) sKeys[j] = kr[k];
    }
    for (int i = tid; i < 256; i += NT) sHist[i] = 0;
    __syncthreads();
    uint32_t T = 0xffffffffu;
    int n_gt = 0;
    if (kk > 0) block_select_kth_fast<NT, KPT>(kr, kv, kk, sHist, T, n_gt);
    const int need_eq = (kk > 0) ? kk - n_gt : 0;
    uint32_t g_run = 0, e_run = 0;
    for (int c0 = 0; c0 < N; c0 += NT) {
        const int row = c0 + tid;
        const bool in = row < N;
        const bool cand = row < M;
        const uint32_t key = cand ? sKeys[row] : 0u;
        const bool eq = cand && kk > 0 && key == T;
        const bool gw = in && (!cand || (kk > 0 && key > T));
        uint32_t tot2;
        const uint32_t ex = block_excl_scan_u32<NT>((eq ? 65536u : 0u) + (gw ? 1u : 0u), sRedU, tot2);
        const uint32_t Ei = e_run + (ex >> 16), Gi = g_run + (ex & 0xffffu);
        const bool kept = gw || (eq && Ei < static_cast<uint32_t>(need_eq));
        if (in) {
            const int32_t d = kept ? static_cast<int32_t>(Gi + min(Ei, static_cast<uint32_t>(need_eq))) : -1;
            sDst[row] = d;
            if (write_kept && p.kept_out && d >= 0) p.kept_out[static_cast<int64_t>(lb) * p.cap + d] = row;
        }
        e_run += tot2 >> 16;
        g_run += tot2 & 0xffffu;
    }
    __syncthreads();
}

// One CTA per (layer, sequence, head): the select of its (layer, sequence),
// then the head's compaction.  In place: every source row of a chunk is read
// before any row of the chunk is written, and later chunks read only rows
// above it (destinations never exceed their source).
__global__ void __launch_bounds__(kSelThreads) rkv_shared_compact_kernel(const SharedParams p) {
    constexpr int NT = kSelThreads;
    // a programmatic dependent of the kernel before it: wait for it before reading
    asm volatile("griddepcontrol.wait;" ::: "memory");
    extern __shared__ uint32_t sel_smem[];
    const int unit = blockIdx.x;                 // (layer, sequence, head)
    const int h = unit % p.n_kv;
    const int lb = unit / p.n_kv;
    const int b = lb % p.batch;
    const int l = lb / p.batch;
    const int N = p.n_eff[b];
    if (N <= 0) return;
    const int M = N - p.window;
    const int budget = p.budgets ? p.budgets[b] : p.budget_cfg;
    const int kk = budget - p.window;
    uint32_t *sHist = sel_smem;                  // 4 x 256
    uint32_t *sRedU = sel_smem + 1024;           // 64
    uint32_t *sKeys = sel_smem + 1024 + 64;      // cap
    int32_t *sDst = reinterpret_cast<int32_t *>(sKeys + p.cap);   // cap
    const bool wk = h == 0;                      // one CTA writes kept_out
    if (M <= 5 * NT) shared_select_body<5>(p, lb, N, M, kk, wk, sKeys, sDst, sHist, sRedU);
    else if (M <= 9 * NT) shared_select_body<9>(p, lb, N, M, kk, wk, sKeys, sDst, sHist, sRedU);
    else if (M <= 16 * NT) shared_select_body<16>(p, lb, N, M, kk, wk, sKeys, sDst, sHist, sRedU);
    else shared_select_body<32>(p, lb, N, M, kk, wk, sKeys, sDst, sHist, sRedU);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t first = static_cast<uint32_t>(N);
    for (int row = tid; row < N; row += NT)
        if (sDst[row] != row) {
            first = static_cast<uint32_t>(row);
            break;
        }
    first = __reduce_min_sync(kFull, first);
    if (lane == 0) sRedU[warp] = first;
    __syncthreads();
    first = sRedU[0];
#pragma unroll
    for (int k = 1; k < NT / 32; ++k) first = min(first, sRedU[k]);
    const int64_t krow0 = (static_cast<int64_t>(b) * p.n_kv + h) * p.cap;
    uint16_t *kb = p.k[l] + krow0 * kHeadDim;
    uint16_t *vb = p.v[l] + krow0 * kHeadDim;
    constexpr int PER = kChunkRows * 16 / NT;
    for (int c0 = static_cast<int>(first); c0 < N; c0 += kChunkRows) {
        uint4 kx[PER], vx[PER];
        int dd[PER];
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            const int idx = tid + k * NT;
            const int row = c0 + (idx >> 4), pc = idx & 15;
            const int d = row < N ? sDst[row] : -1;
            dd[k] = (d >= 0 && d != row) ? d : -1;
            if (dd[k] >= 0) {
                kx[k] = __ldcg(reinterpret_cast<const uint4 *>(kb + static_cast<int64_t>(row) * kHeadDim) + pc);
                vx[k] = __ldcg(reinterpret_cast<const uint4 *>(vb + static_cast<int64_t>(row) * kHeadDim) + pc);
            }
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < PER; ++k) {
            if (dd[k] >= 0) {
                const int pc = (tid + k * NT) & 15;
                __stcs(reinterpret_cast<uint4 *>(kb + static_cast<int64_t>(dd[k]) * kHeadDim) + pc, kx[k]);
                __stcs(reinterpret_cast<uint4 *>(vb + static_cast<int64_t>(dd[k]) * kHeadDim) + pc, vx[k]);
            }
        }
    }
}

// Launches `kern` as a programmatic dependent of the kernel before it on `stream`: its
// CTAs may be scheduled while that kernel finishes, and wait for it on the device.
template <class Kern>
static cudaError_t launch_dependent(Kern kern, unsigned blocks, unsigned threads, size_t smem,
                                    cudaStream_t stream, const SharedParams &p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks, 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

cudaError_t launch_head_sum(const SharedParams &p, int n_lb, cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>(n_lb) * static_cast<unsigned>((p.cap + 255) / 256);
    return launch_dependent(rkv_head_sum_kernel, blocks, 256u, 0, stream, p);
}

size_t shared_select_smem(int cap) { return (1024u + 64u + 2u * static_cast<size_t>(cap)) * 4u; }

cudaError_t launch_shared_compact(const SharedParams &p, int n_units, cudaStream_t stream) {
    const size_t smem = shared_select_smem(p.cap);
    static std::atomic<int> granted{0};
    const cudaError_t e = ensure_smem_attr(rkv_shared_compact_kernel, smem, granted);
    if (e != cudaSuccess) return e;
    return launch_dependent(rkv_shared_compact_kernel, static_cast<unsigned>(n_units),
                            static_cast<unsigned>(kSelThreads), smem, stream, p);
}

}  // namespace rkv
