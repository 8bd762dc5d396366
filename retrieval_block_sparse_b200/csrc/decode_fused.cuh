// Decode step: the persistent attention kernel that follows the score and
// top-k kernels as a programmatic dependent (host-side entry points).
#pragma once

#include "rba_internal.cuh"

namespace rba {

bool fused_eligible(const rba_store* st, const Geometry& g, int k);
int fused_grid(const rba_store* st, const Geometry& g, int k);
// zeroed synchronisation words (per-head merge tickets)
size_t fused_sync_bytes(const rba_store* st);
// partial-state slots
size_t fused_slot_bytes(const rba_store* st, const Geometry& g, int k, int* ms);
// CTAs of the attention kernel per SM for this store's types (0: none, <0: CUDA error)
int fused_occupancy(const rba_store* st);
// whether the persistent kernel of this store is the whole-block tensor-core one
bool fused_whole_blocks(const rba_store* st);
// pdl: launched as a programmatic dependent of the top-k kernel (its stager
// waits for that kernel before reading idx)
rba_status launch_fused(const rba_store* st, const void* q, int k, const Geometry& g, float scale,
                        const int32_t* idx, float* out, float* lse, void* sync, float* slots,
                        bool pdl, cudaStream_t stream);

}  // namespace rba
