// Sample (segment) tables from position_ids, shared by forward and backward.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/ulysses.h"

namespace uly {

// For every token t of every batch row: segstart[t] = first token of t's
// sample, segend[t] = one past its last token.  A sample starts at t == 0
// and wherever position_ids[t] == 0 (blog "Ulysses Sequence Parallelism:
// Training with Million-Token Contexts", position_ids paragraph: causal
// masking comes from position_ids, which restart per packed sample).
cudaError_t launch_segments(const int64_t* position_ids, int32_t* segstart, int32_t* segend, int64_t b,
                            int64_t n, cudaStream_t s);

// Bytes of the workspace prefix both attention calls use (status word plus
// the two tables).
size_t seg_workspace_bytes(int64_t b, int64_t n);

// Argument checks shared by the attention entry points.
uly_status validate_attn(const void* q, const void* k, const void* v, const int64_t* pos, const uly_shape* s,
                         int32_t rank, const void* ws, size_t ws_bytes, size_t need);

}  // namespace uly
