// Internal interface of the slot scan (used by moe_dispatch).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace moe {

// Bytes of look-back state the scan needs for T tokens and E experts.
size_t dispatch_scan_state_bytes(int64_t T, int32_t E);

// Clears `state_mem` (stream-ordered), fills token_of_slot with -1 and launches
// the scan.  `state_mem` must hold dispatch_scan_state_bytes(T, E) bytes.
// Expert parallelism: rank_base (E) != NULL starts expert e's slots at
// rank_base[e] (the assignments of lower ranks), used/overflow are then not
// written (they depend on every rank), token_of_slot (may be NULL) records
// token_base + t.
int dispatch_scan_launch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C, int64_t* slot,
                         uint8_t* kept, int32_t* used, int32_t* overflow, int32_t* drops, int32_t* token_of_slot,
                         void* state_mem, int32_t* status, cudaStream_t stream, const int32_t* rank_base = nullptr,
                         int64_t token_base = 0);

// Host-side validation shared by the dispatch entry points.
int dispatch_check_args(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C, const void* x,
                        moe_dtype dtype, int64_t D, int64_t ldx, const int64_t* slot, const uint8_t* kept,
                        const int32_t* used, const int32_t* overflow, const int32_t* drops,
                        const int32_t* token_of_slot, const void* xbuf);

}  // namespace moe
