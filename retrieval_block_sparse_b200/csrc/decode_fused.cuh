// Fused decode step (one persistent launch): host-side entry points.
#pragma once

#include "rba_internal.cuh"

namespace rba {

bool fused_eligible(const rba_store* st, const Geometry& g, int k);
int fused_grid(const rba_store* st, const Geometry& g, int k);
// zeroed synchronisation words (tickets, ready flags, score counters)
size_t fused_sync_bytes(const rba_store* st);
// partial-state slots
size_t fused_slot_bytes(const rba_store* st, const Geometry& g, int k, int* ms);
// CTAs of the fused kernel per SM for this store's types (0: none, <0: CUDA error)
int fused_occupancy(const rba_store* st);
rba_status launch_fused(const rba_store* st, const void* q, int k, const Geometry& g, float scale,
                        float* scores, int32_t* idx, float* out, float* lse, void* sync,
                        float* slots, cudaStream_t stream);

}  // namespace rba
