// rkv_block.cuh -- block-level building blocks, templated on the CTA's thread
// count NT (a multiple of 32): deterministic reductions (fixed butterfly order,
// then the warps in warp order), packed exclusive scans, a warp
// "transpose-reduce" that folds 16 per-thread columns across the 32 lanes, the
// order-preserving key of a float, the joint score, and radix selects of the
// k-th largest 32-bit key.
#pragma once

#include <cstdint>

namespace rkv {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

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

// Every thread gets the same value.  `red` needs NT/32 floats.
template <int NT, class Op>
__device__ __forceinline__ float block_allreduce(float x, Op op, float *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    x = warp_allreduce(x, op);
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) r = op(r, red[w]);
    __syncthreads();
    return r;
}

template <int NT>
__device__ __forceinline__ uint32_t block_sum_u32(uint32_t x, uint32_t *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    x = __reduce_add_sync(kFull, x);
    if (lane == 0) red[warp] = x;
    __syncthreads();
    uint32_t r = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) r += red[w];
    __syncthreads();
    return r;
}

// Exclusive prefix sum of small packed counters across the block in thread
// order; `total` receives the block-wide sum.  `sw` needs NT/32 uint32.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan_u32(uint32_t v, uint32_t *sw, uint32_t &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(kFull, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) sw[warp] = inc;
    __syncthreads();
    uint32_t pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const uint32_t c = sw[w];
        pre += (w < warp) ? c : 0u;
        tot += c;
    }
    __syncthreads();
    total = tot;
    return pre + inc - v;
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

// Radix select with the keys already in registers (thread tid holds keys
// tid + k * NT, k < KPT; kv[k] false where there is no key) and one block
// barrier per round: every warp adds into the round's shared 256-bin histogram
// (one atomic per warp when all its lanes share the digit), zeroes the next
// round's histogram, and after the barrier every warp scans the whole
// histogram itself, so that no result needs to be written back.
// hist: 4 * 256 uint32, whose first 256 entries must be zero on entry; the
// call ends with all threads synchronised.  T = the kk-th largest key
// (1 <= kk <= number of keys); n_gt = the number of keys above T.
template <int NT, int KPT>
__device__ __forceinline__ void block_select_kth_fast(const uint32_t (&kr)[KPT],
                                                      const bool (&kv)[KPT], int kk,
                                                      uint32_t *hist, uint32_t &T, int &n_gt) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t prefix = 0, mask = 0;
    int remaining = kk, above_total = 0;
#pragma unroll 1
    for (int round = 0; round < 4; ++round) {
        const int shift = 24 - 8 * round;
        uint32_t *H = hist + 256 * round;
#pragma unroll
        for (int k = 0; k < KPT; ++k) {
            const bool part = kv[k] && ((kr[k] & mask) == prefix);
            const uint32_t digit = (kr[k] >> shift) & 255u;
            const unsigned act = __ballot_sync(kFull, part);
            if (act != 0) {
                const uint32_t d0 = __shfl_sync(kFull, digit, __ffs(act) - 1);
                if (__all_sync(kFull, !part || digit == d0)) {
                    if (lane == 0) atomicAdd(&H[d0], static_cast<uint32_t>(__popc(act)));
                } else if (part) {
                    atomicAdd(&H[digit], 1u);
                }
            }
        }
        if (round < 3)
            for (int i = tid; i < 256; i += NT) H[256 + i] = 0;
        __syncthreads();
        // every warp: lane l holds bins 8l .. 8l + 7; suffix sums from the top bin down
        const uint4 a = *reinterpret_cast<const uint4 *>(H + 8 * lane);
        const uint4 b = *reinterpret_cast<const uint4 *>(H + 8 * lane + 4);
        const uint32_t c[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) s += c[i];
        uint32_t suf = s;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_down_sync(kFull, suf, off);
            if (lane + off < 32) suf += o;
        }
        uint32_t above = suf - s, found_bin = 0, found_above = 0;
        bool found = false;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            if (!found && above < static_cast<uint32_t>(remaining) &&
                above + c[i] >= static_cast<uint32_t>(remaining)) {
                found = true;
                found_bin = 8 * lane + i;
                found_above = above;
            }
            above += c[i];
        }
        const int src = __ffs(__ballot_sync(kFull, found)) - 1;
        const uint32_t d = __shfl_sync(kFull, found_bin, src);
        const int ab = static_cast<int>(__shfl_sync(kFull, found_above, src));
        prefix |= d << shift;
        mask |= 255u << shift;
        remaining -= ab;
        above_total += ab;
    }
    T = prefix;
    n_gt = above_total;
    __syncthreads();   // the histograms may be reused by the caller
}

// The same select for 128-thread CTAs (two bins per thread).
template <int NT>
__device__ __forceinline__ void block_select_kth_small(const uint32_t *keys, int n, int kk,
                                                       uint32_t *hist, uint32_t *scan,
                                                       uint32_t &T, int &n_gt) {
    constexpr int NW = NT / 32;
    static_assert(NT == 128, "two bins per thread");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t *my = hist + warp * 256;
    uint32_t prefix = 0, mask = 0;
    int remaining = kk, above_total = 0;
#pragma unroll 1
    for (int round = 0; round < 4; ++round) {
        const int shift = 24 - 8 * round;
#pragma unroll
        for (int i = lane; i < 256; i += 32) my[i] = 0;
        __syncwarp();
        for (int base = 0; base < n; base += NT) {
            const int j = base + tid;
            const uint32_t key = (j < n) ? keys[j] : 0u;
            const bool part = (j < n) && ((key & mask) == prefix);
            const uint32_t digit = (key >> shift) & 255u;
            const unsigned act = __ballot_sync(kFull, part);
            if (act == 0) continue;
            const uint32_t d0 = __shfl_sync(kFull, digit, __ffs(act) - 1);
            if (__all_sync(kFull, !part || digit == d0)) {
                if (lane == 0) my[d0] += static_cast<uint32_t>(__popc(act));
            } else if (part) {
                atomicAdd(&my[digit], 1u);
            }
            __syncwarp();
        }
        __syncthreads();
        // thread t owns bins 255 - 2t and 254 - 2t (descending)
        const int b0 = 255 - 2 * tid, b1 = 254 - 2 * tid;
        uint32_t c0 = 0, c1 = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            c0 += hist[w * 256 + b0];
            c1 += hist[w * 256 + b1];
        }
        const uint32_t cnt = c0 + c1;
        uint32_t inc = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(kFull, inc, off);
            if (lane >= off) inc += o;
        }
        if (lane == 31) scan[warp] = inc;
        __syncthreads();
        uint32_t above = inc - cnt;
#pragma unroll
        for (int w = 0; w < NW; ++w) above += (w < warp) ? scan[w] : 0u;
        const uint32_t rem = static_cast<uint32_t>(remaining);
        if (above < rem && above + c0 >= rem) {
            scan[NW + 0] = static_cast<uint32_t>(b0);
            scan[NW + 1] = above;
        } else if (above + c0 < rem && above + cnt >= rem) {
            scan[NW + 0] = static_cast<uint32_t>(b1);
            scan[NW + 1] = above + c0;
        }
        __syncthreads();
        const uint32_t d = scan[NW + 0];
        const int ab = static_cast<int>(scan[NW + 1]);
        prefix |= d << shift;
        mask |= 255u << shift;
        remaining -= ab;
        above_total += ab;
        __syncthreads();
    }
    T = prefix;
    n_gt = above_total;
}

}  // namespace rkv
