// rkv_select.cu -- joint score and top-k selection for one (sequence, layer),
// one CTA per KV head: Z = lambda I - (1 - lambda) R ("Approach" of the
// atlas.scime.ai summary of "R-KV: Redundancy-aware KV Cache Compression for
// Reasoning Models"), the budget - window candidates with the largest Z
// (ties to the lower index) plus the protected window, in ascending order
// (sourcepulse summary, "How It Works"; hysenlabs write-up, decode-time
// section on window_size).
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace rkv {

__global__ void __launch_bounds__(kThreads) rkv_select_kernel(
    const float *__restrict__ I, const float *__restrict__ R, int M, int N, int budget,
    float lambda, int32_t *__restrict__ kept, float *__restrict__ Z_out) {
    extern __shared__ uint32_t sk_keys[];   // [M]
    __shared__ uint32_t s_hist[256];
    __shared__ int s_int[8];
    const int h = blockIdx.x, tid = threadIdx.x;
    const int w = N - M, kk = budget - w;
    const float *Ih = I + static_cast<int64_t>(h) * M;
    const float *Rh = R + static_cast<int64_t>(h) * M;
    for (int j = tid; j < M; j += kThreads) {
        const float z = joint_score(lambda, Ih[j], Rh[j]);
        if (Z_out) Z_out[static_cast<int64_t>(h) * M + j] = z;
        sk_keys[j] = ordered_key(z);
    }
    __syncthreads();
    uint32_t T = 0xffffffffu;
    int n_gt = 0;
    if (kk > 0) block_select_kth(sk_keys, M, kk, s_hist, s_int, T, n_gt);
    const int need_eq = kk > 0 ? kk - n_gt : 0;
    int32_t *out = kept + static_cast<int64_t>(h) * budget;
    int eq_run = 0, kept_run = 0;
    for (int c0 = 0; c0 < M; c0 += kThreads) {
        const int j = c0 + tid;
        const bool in = j < M;
        const uint32_t key = in ? sk_keys[j] : 0u;
        const bool eq = in && kk > 0 && key == T;
        int eq_tot, kept_tot;
        const int eq_rank = eq_run + block_excl_scan_flag(eq, s_int + 4, eq_tot);
        const bool k = in && kk > 0 && (key > T || (eq && eq_rank < need_eq));
        const int dst = kept_run + block_excl_scan_flag(k, s_int + 4, kept_tot);
        if (k) out[dst] = j;
        eq_run += eq_tot;
        kept_run += kept_tot;
    }
    for (int t = tid; t < w; t += kThreads) out[kk + t] = M + t;
}

cudaError_t launch_select(const float *I, const float *R, int n_kv, int M, int N, int budget,
                          float lambda, int32_t *kept, float *Z, uint32_t * /*status*/,
                          cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(M) * 4u;
    cudaError_t e = cudaFuncSetAttribute(rkv_select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    rkv_select_kernel<<<n_kv, kThreads, smem, stream>>>(I, R, M, N, budget, lambda, kept, Z);
    return cudaGetLastError();
}

}  // namespace rkv
