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

constexpr int kSelThreads = 128;

__global__ void __launch_bounds__(kSelThreads) rkv_select_kernel(
    const float *__restrict__ I, const float *__restrict__ R, int M, int N, int budget,
    float lambda, int32_t *__restrict__ kept, float *__restrict__ Z_out) {
    constexpr int NT = kSelThreads;
    extern __shared__ uint32_t sk_keys[];   // [M]
    __shared__ uint32_t s_hist[(NT / 32) * 256];
    __shared__ uint32_t s_int[NT / 32 + 4];
    __shared__ uint32_t s_red[NT / 32];
    const int h = blockIdx.x, tid = threadIdx.x;
    const int w = N - M, kk = budget - w;
    const float *Ih = I + static_cast<int64_t>(h) * M;
    const float *Rh = R + static_cast<int64_t>(h) * M;
    for (int j = tid; j < M; j += NT) {
        const float z = joint_score(lambda, Ih[j], Rh[j]);
        if (Z_out) Z_out[static_cast<int64_t>(h) * M + j] = z;
        sk_keys[j] = ordered_key(z);
    }
    __syncthreads();
    uint32_t T = 0xffffffffu;
    int n_gt = 0;
    if (kk > 0) block_select_kth_small<NT>(sk_keys, M, kk, s_hist, s_int, T, n_gt);
    const uint32_t need_eq = kk > 0 ? static_cast<uint32_t>(kk - n_gt) : 0u;
    int32_t *out = kept + static_cast<int64_t>(h) * budget;
    uint32_t e_run = 0, g_run = 0;
    for (int c0 = 0; c0 < M; c0 += NT) {
        const int j = c0 + tid;
        const bool in = j < M;
        const uint32_t key = in ? sk_keys[j] : 0u;
        const bool eq = in && kk > 0 && key == T;
        const bool gt = in && kk > 0 && key > T;
        uint32_t tot;
        const uint32_t ex = block_excl_scan_u32<NT>((eq ? 65536u : 0u) + (gt ? 1u : 0u), s_red, tot);
        const uint32_t Ei = e_run + (ex >> 16), Gi = g_run + (ex & 0xffffu);
        if (gt || (eq && Ei < need_eq)) out[Gi + min(Ei, need_eq)] = j;
        e_run += tot >> 16;
        g_run += tot & 0xffffu;
    }
    for (int t = tid; t < w; t += NT) out[kk + t] = M + t;
}

cudaError_t launch_select(const float *I, const float *R, int n_kv, int M, int N, int budget,
                          float lambda, int32_t *kept, float *Z, uint32_t * /*status*/,
                          cudaStream_t stream) {
    const size_t smem = static_cast<size_t>(M) * 4u;
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem_attr(rkv_select_kernel, smem, granted);
    if (e != cudaSuccess) return e;
    return launch_kernel(rkv_select_kernel, dim3(n_kv), dim3(kSelThreads), smem, stream, I, R, M, N,
                         budget, lambda, kept, Z);
}

}  // namespace rkv
