// rkv_noalloc.cu -- rkv_compress_step_noalloc: the whole compression step for
// callers that cannot allocate device memory themselves.
//
// Some hosts own every byte of the GPU: a serving engine that reserves the
// device's memory up front for its own pool and hands plugins no allocator, or
// a latency-critical decode loop where a cudaMalloc (which may synchronise the
// device) is not acceptable.  Such callers still own their K/V caches, query
// windows and cur_len, but cannot provide the step's small scratch buffer.
// This entry point gives them one: a fixed array in the library's own device
// memory, holding the status header and the per-sequence length snapshot that
// rkv_compress_step keeps in its workspace.  The array is part of the loaded
// module, so every GPU on which the library is used holds it until the process
// exits.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "../../include/rkv.h"

namespace rkv {
// The part of a step's workspace the call cannot run without (rkv_abi.cu).
size_t workspace_required_bytes(const rkv_config *cfg, int32_t n_layers, int32_t batch,
                                int32_t cap);
}  // namespace rkv

namespace {

constexpr size_t kScratchBytes = RKV_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per
// device (with that device current) and cached for the life of the process.
rkv_status scratch_address(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RKV_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return RKV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return RKV_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return RKV_OK;
}

}  // namespace

extern "C" rkv_status rkv_compress_step_noalloc(const rkv_config *cfg, int32_t n_layers,
                                                int32_t batch, int32_t cap,
                                                rkv_bf16 *const *k_layers,
                                                rkv_bf16 *const *v_layers,
                                                const rkv_bf16 *const *q_layers,
                                                const int32_t *budgets, const float *lambdas,
                                                int32_t *cur_len, const rkv_step_options *opts,
                                                rkv_stream_t stream) {
    if (!cfg) return RKV_ERR_NULL;
    if (n_layers < 1 || batch < 1 || cap < 2) return RKV_ERR_INVALID;
    const size_t need = rkv::workspace_required_bytes(cfg, n_layers, batch, cap);
    if (need == 0)   // invalid config: let the step report exactly what is wrong
        return rkv_compress_step(cfg, n_layers, batch, cap, k_layers, v_layers, q_layers, budgets,
                                 lambdas, cur_len, opts, nullptr, 0, stream);
    // MAX redundancy keeps r of every unit in the workspace: far beyond the scratch
    if (cfg->redundancy_mode == RKV_RED_MAX) return RKV_ERR_UNSUPPORTED;
    if (batch > RKV_NOALLOC_MAX_BATCH || need > kScratchBytes) return RKV_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    const rkv_status st = scratch_address(&scratch);
    if (st != RKV_OK) return st;
    return rkv_compress_step(cfg, n_layers, batch, cap, k_layers, v_layers, q_layers, budgets,
                             lambdas, cur_len, opts, scratch, kScratchBytes, stream);
}

extern "C" rkv_status rkv_noalloc_status(rkv_stream_t stream) {
    void *scratch = nullptr;
    const rkv_status st = scratch_address(&scratch);
    if (st != RKV_OK) return st;
    // the status word sits at the start of the scratch, as in a workspace
    return rkv_workspace_status(scratch, stream);
}
