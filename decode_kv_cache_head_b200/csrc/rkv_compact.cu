// rkv_compact.cu -- physical compaction of one (sequence, layer):
// k_dst[h][t] = k_src[h][kept[h][t]] and the same for V, bit for bit.
// R-KV evicts physically rather than masking (hysenlabs write-up "R-KV:
// decoding-time KV cache compression for reasoning models", section "How
// this differs from attention-sink and heavy-hitter eviction"; its SGLang port
// uses a two-phase compaction, decode-time section).
//
// Out of place: a plain vectorised gather, 16 bytes per thread.
// In place: one thread-block cluster per head.  CTA c owns destinations
// [c*Rb, (c+1)*Rb); it bulk-copies their source rows of K and V into shared
// memory, the cluster waits until every CTA has its rows (so no source row of
// the head can be overwritten before it is read), then each CTA writes its
// destinations.  This is the two-phase scheme with the staging buffer spread
// over the cluster's shared memory instead of global memory.
#include <cooperative_groups.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace cg = cooperative_groups;

namespace rkv {

constexpr int kCompactMaxStageBytes = 200 * 1024;
constexpr int kThreads = 128;

__global__ void __launch_bounds__(256) rkv_gather_kernel(
    const uint16_t *__restrict__ k_src, const uint16_t *__restrict__ v_src,
    const int32_t *__restrict__ kept, uint16_t *__restrict__ k_dst, uint16_t *__restrict__ v_dst,
    int64_t head_stride, int budget, int n_tokens, uint32_t *status) {
    const int h = blockIdx.y;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(budget) * 16) return;
    const int t = static_cast<int>(idx >> 4), c = static_cast<int>(idx & 15);
    const int s = kept[static_cast<int64_t>(h) * budget + t];
    if (s < 0 || s >= n_tokens) {
        record_flag(status, kDevFlagBadIndex);
        return;
    }
    const int64_t so = h * head_stride + static_cast<int64_t>(s) * kHeadDim + c * 8;
    const int64_t d = h * head_stride + static_cast<int64_t>(t) * kHeadDim + c * 8;
    __stcs(reinterpret_cast<uint4 *>(k_dst + d), __ldg(reinterpret_cast<const uint4 *>(k_src + so)));
    __stcs(reinterpret_cast<uint4 *>(v_dst + d), __ldg(reinterpret_cast<const uint4 *>(v_src + so)));
}

__global__ void __launch_bounds__(kThreads, 1) rkv_compact_inplace_kernel(
    uint16_t *k, uint16_t *v, const int32_t *__restrict__ kept, int64_t head_stride, int budget,
    int n_tokens, uint32_t *status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stage = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
    __shared__ uint64_t bar;
    __shared__ float s_red[kThreads / 32];
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = static_cast<int>(cluster.num_blocks());
    const int rank = static_cast<int>(cluster.block_rank());
    const int h = blockIdx.x / cs;
    const int tid = threadIdx.x;
    const int rb = (budget + cs - 1) / cs;
    const int t0 = rank * rb;
    const int nt = max(0, min(rb, budget - t0));
    uint16_t *kh = k + h * head_stride;
    uint16_t *vh = v + h * head_stride;
    const int32_t *kp = kept + static_cast<int64_t>(h) * budget;
    if (tid == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    int moved = 0;
    for (int i = tid; i < nt; i += kThreads) {
        const int t = t0 + i;
        const int s = kp[t];
        if (s < 0 || s >= n_tokens) {
            record_flag(status, kDevFlagBadIndex);
            continue;
        }
        if (s == t) continue;
        bulk_g2s(stage + i * 512, kh + static_cast<int64_t>(s) * kHeadDim, 256u, &bar);
        bulk_g2s(stage + i * 512 + 256, vh + static_cast<int64_t>(s) * kHeadDim, 256u, &bar);
        ++moved;
    }
    moved = static_cast<int>(block_allreduce<kThreads>(static_cast<float>(moved), OpSum(), s_red));
    if (tid == 0) mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(moved) * 512u);
    bool ok = mbar_wait(&bar, 0);
    if (!ok) record_flag(status, kDevFlagTimeout);
    ok = __syncthreads_and(ok);
    cluster.sync();   // every source row of this head is now staged somewhere in the cluster
    if (!ok) return;
    for (int idx = tid; idx < nt * 32; idx += kThreads) {
        const int i = idx >> 5, c = idx & 31;
        const int t = t0 + i;
        const int s = kp[t];
        if (s < 0 || s >= n_tokens || s == t) continue;
        const uint4 x = *reinterpret_cast<const uint4 *>(stage + i * 512 + c * 16);
        uint16_t *dst = (c < 16 ? kh : vh) + static_cast<int64_t>(t) * kHeadDim + (c & 15) * 8;
        __stcs(reinterpret_cast<uint4 *>(dst), x);
    }
}

int compact_in_place_cluster(int budget) {
    for (int cs : {4, 8, 16}) {
        const int rb = (budget + cs - 1) / cs;
        if (rb * 512 + 256 <= kCompactMaxStageBytes) return cs;
    }
    return 0;
}

cudaError_t launch_compact(const uint16_t *k_src, const uint16_t *v_src, const int32_t *kept,
                           uint16_t *k_dst, uint16_t *v_dst, int64_t head_stride, int n_kv,
                           int budget, int n_tokens, bool in_place, int cs, uint32_t *status,
                           cudaStream_t stream) {
    if (!in_place) {
        const int64_t items = static_cast<int64_t>(budget) * 16;
        dim3 grid(static_cast<unsigned>((items + 255) / 256), static_cast<unsigned>(n_kv));
        return launch_kernel(rkv_gather_kernel, grid, dim3(256), 0, stream, k_src, v_src, kept, k_dst,
                             v_dst, head_stride, budget, n_tokens, status);
    }
    const int rb = (budget + cs - 1) / cs;
    const size_t smem = static_cast<size_t>(rb) * 512u + 128u;
    static std::atomic<int> granted{0};
    static std::atomic<bool> nonportable{false};
    cudaError_t e = ensure_smem_attr(rkv_compact_inplace_kernel, smem, granted);
    if (e != cudaSuccess) return e;
    if (cs > 8 && !nonportable.load()) {
        e = cudaFuncSetAttribute(rkv_compact_inplace_kernel,
                                 cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        nonportable.store(true);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_kv * cs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rkv_compact_inplace_kernel, k_dst, v_dst, kept, head_stride,
                              budget, n_tokens, status);
}

}  // namespace rkv
