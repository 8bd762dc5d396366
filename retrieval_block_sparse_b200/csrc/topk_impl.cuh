// Top-k internals shared by the selector and the fused decode step.
#pragma once

#include "rba_internal.cuh"

namespace rba {

// Rows of at most kSmallN scores are selected by one CTA in shared memory
// (5 bytes a score: the values and a flag, 80 KB at the limit).
constexpr int kSmallN = 16384;
// Largest k the radix path handles (its final sort holds k positions in smem).
constexpr int kLargeMaxK = 16384;

size_t topk_large_workspace(int rows, int n, int k);
rba_status launch_topk_large(const float* scores, int rows, int n, int k, int index_base,
                             int32_t* idx, void* ws, cudaStream_t stream);
// pdl: launched as a programmatic dependent of the previous kernel on the
// stream (it waits for that kernel's completion before reading scores)
rba_status launch_topk(const float* scores, int rows, int n, int k, int index_base, int32_t* idx,
                       void* ws, size_t ws_bytes, cudaStream_t stream, bool pdl);
size_t topk_workspace(int rows, int n, int k);
// CTAs the selector of `rows` rows of n scores runs while a dependent kernel
// starts (0: the multi-CTA path)
int topk_ctas(int rows, int n);

}  // namespace rba
