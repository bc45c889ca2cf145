// rkv_post.cuh -- the part of the step that follows scoring, shared by the
// cluster kernel and the one-CTA-per-unit kernel: from every candidate's
// (Ihat_i, r_i) the normalisers sum Ihat, max r and sum exp(r - max r), then
// each candidate's joint score Z_i = lambda I_i - (1 - lambda) R_i as an
// order-preserving key and the radix select of the k-th largest key.
//
// "R-KV: Redundancy-aware KV Cache Compression for Reasoning Models"
// (atlas.scime.ai summary, "Approach": Z = lambda I - (1 - lambda) R and the
// top-k within the budget; sourcepulse summary, "How It Works").
#pragma once

#include <cstdint>

#include "rkv_block.cuh"
#include "rkv_ptx.cuh"

namespace rkv {

// All NT threads call.  load(j) returns (Ihat_j, r_j) for candidate j < M;
// thread tid takes candidates tid + k * NT (k < KPT, needs M <= KPT * NT).
// Outputs: 1 / sum Ihat, max r, 1 / sum exp(r - max r); if `select`, the key
// of candidate j is stored at sKeys[KSTRIDE * j] and T / n_gt are the k-th
// largest key and the number of keys above it (kk > 0).  sHist: 4 x 256
// uint32 (zeroed here); sRed: 4 * NT/32 floats.  Ends with the block in sync.
template <int NT, int KPT, int KSTRIDE, class Load>
__device__ __forceinline__ void post_scores(Load load, uint32_t *sKeys, uint32_t *sHist,
                                            float *sRed, int M, int kk, float lam, bool select,
                                            float &inv_sumI, float &rmax_g, float &inv_rsum,
                                            uint32_t &T, int &n_gt) {
    constexpr int NW = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float ih[KPT], rr[KPT];
    bool kv[KPT];
    float sI = 0.f, mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        const int j = tid + k * NT;
        kv[k] = j < M;
        const float2 v = kv[k] ? load(j) : make_float2(0.f, -INFINITY);
        ih[k] = v.x;
        rr[k] = v.y;
        sI += v.x;
        mx = fmaxf(mx, v.y);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        sI += __shfl_xor_sync(kFull, sI, off);
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
    }
    if (lane == 0) {
        sRed[2 * warp] = sI;
        sRed[2 * warp + 1] = mx;
    }
    for (int i = tid; i < 256; i += NT) sHist[i] = 0;   // first histogram of the select
    __syncthreads();
    sI = sRed[0];
    mx = sRed[1];
#pragma unroll
    for (int w = 1; w < NW; ++w) {
        sI += sRed[2 * w];
        mx = fmaxf(mx, sRed[2 * w + 1]);
    }
    float e[KPT];
    float rs = 0.f;
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        e[k] = kv[k] ? ex2_approx((rr[k] - mx) * kLog2e) : 0.f;
        rs += e[k];
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) rs += __shfl_xor_sync(kFull, rs, off);
    if (lane == 0) sRed[2 * NW + warp] = rs;
    __syncthreads();
    rs = sRed[2 * NW];
#pragma unroll
    for (int w = 1; w < NW; ++w) rs += sRed[2 * NW + w];
    inv_sumI = 1.0f / sI;
    rmax_g = mx;
    inv_rsum = 1.0f / rs;
    if (!select) return;
    uint32_t kr[KPT];
#pragma unroll
    for (int k = 0; k < KPT; ++k) {
        kr[k] = ordered_key(joint_score(lam, ih[k] * inv_sumI, e[k] * inv_rsum));
        if (kv[k]) sKeys[KSTRIDE * (tid + k * NT)] = kr[k];
    }
    if (kk > 0) block_select_kth_fast<NT, KPT>(kr, kv, kk, sHist, T, n_gt);
    else __syncthreads();
}

// Dispatches post_scores on the number of candidates per thread.
template <int NT, int KSTRIDE, class Load>
__device__ __forceinline__ void post_scores_any(Load load, uint32_t *sKeys, uint32_t *sHist,
                                                float *sRed, int M, int kk, float lam,
                                                bool select, float &inv_sumI, float &rmax_g,
                                                float &inv_rsum, uint32_t &T, int &n_gt) {
    if (M <= 5 * NT)
        post_scores<NT, 5, KSTRIDE>(load, sKeys, sHist, sRed, M, kk, lam, select, inv_sumI, rmax_g,
                                    inv_rsum, T, n_gt);
    else if (M <= 7 * NT)
        post_scores<NT, 7, KSTRIDE>(load, sKeys, sHist, sRed, M, kk, lam, select, inv_sumI, rmax_g,
                                    inv_rsum, T, n_gt);
    else if (M <= 9 * NT)
        post_scores<NT, 9, KSTRIDE>(load, sKeys, sHist, sRed, M, kk, lam, select, inv_sumI, rmax_g,
                                    inv_rsum, T, n_gt);
    else if (M <= 16 * NT)
        post_scores<NT, 16, KSTRIDE>(load, sKeys, sHist, sRed, M, kk, lam, select, inv_sumI,
                                     rmax_g, inv_rsum, T, n_gt);
    else
        post_scores<NT, 32, KSTRIDE>(load, sKeys, sHist, sRed, M, kk, lam, select, inv_sumI,
                                     rmax_g, inv_rsum, T, n_gt);
}

}  // namespace rkv
