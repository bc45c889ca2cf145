// rkv_paged.cu -- the page-return side of the step on paged caches: after a
// sequence is compacted from N to `budget` rows, its pages
// ceil(budget / P) .. ceil(N / P) - 1 hold nothing it needs, and their ids are
// handed back for the caller's allocator (physical eviction returning freed
// blocks, the vLLM port's FREE_BLOCKS path: hysenlabs write-up of "R-KV:
// Redundancy-aware KV Cache Compression for Reasoning Models", decode-time
// section).
#include <cuda_runtime.h>

#include <cstdint>

#include "rkv_internal.h"

namespace rkv {

__global__ void rkv_freed_pages_kernel(int batch, const int32_t *__restrict__ budgets,
                                       int32_t budget_cfg, const int32_t *__restrict__ n_eff,
                                       const int32_t *__restrict__ block_table, int max_blocks,
                                       int page_rows, int32_t *__restrict__ freed,
                                       int32_t *__restrict__ n_freed) {
    // a programmatic dependent of the step kernel: wait for it before reading or writing
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= batch) return;
    const int N = n_eff[b];
    int count = 0;
    if (N > 0) {
        const int budget = budgets ? budgets[b] : budget_cfg;
        const int keep = (budget + page_rows - 1) / page_rows;
        const int used = (N + page_rows - 1) / page_rows;
        count = used - keep;
        const int64_t row = static_cast<int64_t>(b) * max_blocks;
        for (int j = 0; j < count; ++j) freed[row + j] = block_table[row + keep + j];
    }
    n_freed[b] = count;
}

cudaError_t launch_freed_pages(int batch, const int32_t *budgets, int32_t budget_cfg,
                               const int32_t *n_eff, const int32_t *block_table, int max_blocks,
                               int page_rows, int32_t *freed, int32_t *n_freed,
                               cudaStream_t stream) {
    // launched as a programmatic dependent of the kernel before it: its CTAs may be
    // scheduled while that kernel finishes, and wait for it on the device
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((batch + 127) / 128), 1, 1);
    cfg.blockDim = dim3(128, 1, 1);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, rkv_freed_pages_kernel, batch, budgets, budget_cfg, n_eff,
                              block_table, max_blocks, page_rows, freed, n_freed);
}

}  // namespace rkv
