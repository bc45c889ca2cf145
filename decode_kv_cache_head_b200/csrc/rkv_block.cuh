// rkv_block.cuh -- block-level building blocks for 128-thread CTAs:
// deterministic reductions (fixed butterfly order, then warps 0..3 in order),
// 0/1 exclusive scans, a warp "transpose-reduce" that folds 16 per-thread
// columns across the 32 lanes, the order-preserving key of a float, and a
// radix select of the k-th largest 32-bit key.
#pragma once

#include <cstdint>

namespace rkv {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xffffffffu;

struct OpSum {
    __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};
struct OpMax {
    __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};

template <class Op>
__device__ __forceinline__ float warp_allreduce(float x, Op op) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) x = op(x, __shfl_xor_sync(kFull, x, off));
    return x;
}

// Every thread gets the same value: butterfly inside each warp, then the four
// warp results combined in warp order.  `red` needs kWarps floats.
template <class Op>
__device__ __forceinline__ float block_allreduce(float x, Op op, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    x = warp_allreduce(x, op);
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) r = op(r, red[w]);
    __syncthreads();
    return r;
}

// Exclusive prefix count of a 0/1 flag across the block in thread order;
// `total` receives the block-wide count.  `sw` needs kWarps ints.
__device__ __forceinline__ int block_excl_scan_flag(bool f, int *sw, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned m = __ballot_sync(kFull, f);
    const int lane_pre = __popc(m & ((1u << lane) - 1u));
    if (lane == 0) sw[warp] = __popc(m);
    __syncthreads();
    int pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int c = sw[w];
        pre += (w < warp) ? c : 0;
        tot += c;
    }
    __syncthreads();
    total = tot;
    return pre + lane_pre;
}

__device__ __forceinline__ int block_count(bool f, int *sw) {
    int total;
    block_excl_scan_flag(f, sw, total);
    return total;
}

// Folds v[0..15] (16 columns held by every lane) across the warp: afterwards
// v[0] of lane L holds op over all 32 lanes of column (L & 15).  16 shuffles.
template <class Op>
__device__ __forceinline__ void warp_transpose_reduce16(float (&v)[16], Op op) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 8; off >= 1; off >>= 1) {
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
            const float send = up ? v[i] : v[i + off];
            const float keep = up ? v[i + off] : v[i];
            v[i] = op(keep, __shfl_xor_sync(kFull, send, off));
        }
    }
    v[0] = op(v[0], __shfl_xor_sync(kFull, v[0], 16));
}

// Order-preserving map float -> uint32 (larger float, larger key); -0 is
// folded onto +0 first so that the two zeros tie.
__device__ __forceinline__ uint32_t ordered_key(float z) {
    const uint32_t u = __float_as_uint(z + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Joint score Z = lambda I - (1 - lambda) R rounded as fp32 mul, mul, sub in
// that order (never contracted into an FMA), so that every place computing Z
// from the same I and R gets the same bits.
__device__ __forceinline__ float joint_score(float lambda, float I, float R) {
    return __fsub_rn(__fmul_rn(lambda, I), __fmul_rn(__fsub_rn(1.0f, lambda), R));
}

// Radix select over keys[0..n) in shared memory (all threads call): T = the
// kk-th largest key (1 <= kk <= n) and n_gt = the number of keys > T.
// hist: 256 uint32, sh: 2 ints of shared scratch.
__device__ __forceinline__ void block_select_kth(const uint32_t *keys, int n, int kk,
                                                 uint32_t *hist, int *sh, uint32_t &T,
                                                 int &n_gt) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
    int remaining = kk, above_total = 0;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int j = tid; j < n; j += kThreads) {
            const uint32_t key = keys[j];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (warp == 0) {
            uint32_t c[8];
            uint32_t s = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                c[i] = hist[8 * lane + i];
                s += c[i];
            }
            uint32_t suf = s;  // inclusive suffix sum over lanes (higher lanes = higher bins)
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t o = __shfl_down_sync(kFull, suf, off);
                if (lane + off < 32) suf += o;
            }
            uint32_t above = suf - s;
#pragma unroll
            for (int i = 7; i >= 0; --i) {
                if (above < static_cast<uint32_t>(remaining) &&
                    above + c[i] >= static_cast<uint32_t>(remaining)) {
                    sh[0] = 8 * lane + i;
                    sh[1] = static_cast<int>(above);
                }
                above += c[i];
            }
        }
        __syncthreads();
        const uint32_t d = static_cast<uint32_t>(sh[0]);
        const int above = sh[1];
        __syncthreads();
        prefix |= d << shift;
        mask |= 255u << shift;
        remaining -= above;
        above_total += above;
    }
    T = prefix;
    n_gt = above_total;
}

}  // namespace rkv
