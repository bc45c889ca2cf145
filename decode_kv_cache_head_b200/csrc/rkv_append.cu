// rkv_append.cu -- the decode side of the R-KV loop: new tokens' keys and
// values are appended to each sequence's cache at its current length, and the
// length grows, until the buffer of new tokens is full and the compression
// step runs ("applied periodically during decoding with a fixed buffer",
// atlas.scime.ai summary of "R-KV: Redundancy-aware KV Cache Compression for
// Reasoning Models", "Approach"; divide_length new tokens between steps,
// hysenlabs write-up, decode-time section).
//
// Two launches: the copy reads cur_len, then one thread per sequence adds the
// chunk length, so that no copy ever sees a half-updated length.
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_internal.h"
#include "rkv_ptx.cuh"

namespace rkv {

// Grid: nchunk blocks of 256 threads per (layer, sequence, head), each thread
// one 16-byte piece of one of the n_new rows.
__global__ void __launch_bounds__(256) rkv_append_kernel(const __grid_constant__ AppendParams p,
                                                         int nchunk) {
    const int u = blockIdx.x / nchunk;
    const int h = u % p.n_kv;
    const int b = (u / p.n_kv) % p.batch;
    const int l = u / (p.n_kv * p.batch);
    const int64_t idx = static_cast<int64_t>(blockIdx.x % nchunk) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(p.n_new) * 16) return;
    const int len = p.cur_len[b];
    if (len < 0 || len + p.n_new > p.cap) {
        if (idx == 0) record_flag(p.status, kDevFlagBadSeq);
        return;
    }
    const int t = static_cast<int>(idx >> 4), c = static_cast<int>(idx & 15);
    const int64_t head = static_cast<int64_t>(b) * p.n_kv + h;
    const int64_t src = (head * p.n_new + t) * kHeadDim + c * 8;
    const int64_t dst = (head * p.cap + len + t) * kHeadDim + c * 8;
    *reinterpret_cast<uint4 *>(p.k[l] + dst) = *reinterpret_cast<const uint4 *>(p.k_new[l] + src);
    *reinterpret_cast<uint4 *>(p.v[l] + dst) = *reinterpret_cast<const uint4 *>(p.v_new[l] + src);
}

__global__ void rkv_bump_len_kernel(int batch, int n_new, int cap, int32_t *cur_len) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    const int len = cur_len[b];
    if (len >= 0 && len + n_new <= cap) cur_len[b] = len + n_new;
}

cudaError_t launch_append(const AppendParams &p, int n_layers, cudaStream_t stream) {
    const int nchunk = static_cast<int>((static_cast<int64_t>(p.n_new) * 16 + 255) / 256);
    const unsigned blocks = static_cast<unsigned>(n_layers * p.batch * p.n_kv) * nchunk;
    return launch_kernel(rkv_append_kernel, dim3(blocks), dim3(256), 0, stream, p, nchunk);
}

cudaError_t launch_bump(int batch, int n_new, int cap, int32_t *cur_len, cudaStream_t stream) {
    return launch_kernel(rkv_bump_len_kernel, dim3((batch + 127) / 128), dim3(128), 0, stream, batch,
                         n_new, cap, cur_len);
}

}  // namespace rkv
