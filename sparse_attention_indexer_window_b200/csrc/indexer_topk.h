// Launch interface of the block-selection kernel (indexer_topk.cu).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sai {

// Largest block count per row the selection kernel keeps in shared memory.
constexpr int kTopkMaxP = 32768;
size_t indexer_topk_smem_bytes(int P);
cudaError_t launch_indexer_topk(const float *scores, const int32_t *doc_start, int B, int S, int cr, int K,
                                int32_t *idx, float *sel, uint8_t *valid, cudaStream_t stream);

}  // namespace sai
