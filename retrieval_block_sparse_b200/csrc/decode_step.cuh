// The whole decode step in one cooperative launch (host-side entry points).
#pragma once

#include "rba_internal.cuh"

namespace rba {

// Whether the one-launch decode step covers this problem: bf16 store whose
// blocks are whole 64-row tiles, head dim 64 or 128, GQA group of 1, 2 or 4,
// dot-mode representations with at most 8 keys, 1 <= k <= 256, at most 4096
// candidates per (batch, kv head), and at most half as many (batch, kv head)
// units as SMs.  Queries the device (occupancy).
bool step_eligible(const rba_store* st, const Geometry& g, int k);
// zeroed synchronisation words (two per (batch, kv head)); every call leaves them zero
size_t step_sync_bytes(const rba_store* st);
// partial-state slots (one per CTA)
size_t step_slot_bytes(const rba_store* st);
rba_status launch_step(const rba_store* st, const void* q, int k, const Geometry& g, float scale,
                       float* scores, int32_t* idx, float* out, float* lse, void* sync,
                       float* slots, cudaStream_t stream);

}  // namespace rba
