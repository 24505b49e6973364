// Host-side helpers shared by the entry points: argument checks, status
// mapping, tensor-map encoding through the driver entry point.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/ulysses.h"

namespace uly {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

inline size_t dtype_size(uly_dtype t) { return t == ULY_F32 ? 4 : 2; }
inline bool dtype_ok(uly_dtype t) { return t == ULY_BF16 || t == ULY_F32; }

// Product of non-negative sizes, false on overflow past 2^62.
inline bool checked_mul(int64_t a, int64_t b, int64_t* out) {
  if (a < 0 || b < 0) return false;
  if (a != 0 && b > (int64_t(1) << 62) / a) return false;
  *out = a * b;
  return true;
}

inline bool elems(int64_t b, int64_t n, int64_t H, int64_t d, int64_t* out) {
  int64_t t;
  return checked_mul(b, n, &t) && checked_mul(t, H, &t) && checked_mul(t, d, out);
}

// The divisibility rules of the pages: n and the query head count divisible
// by P; H_q a multiple of H_kv.  The kv head count is divisible by P, or
// (fewer kv heads than ranks) divides P: then each rank holds one replicated
// kv head (ulysses_kv_seq_to_head).
inline uly_status check_shape(const uly_shape* s) {
  if (!s) return ULY_ERR_INVALID_ARG;
  if (s->P < 1 || s->b < 1 || s->n < 1 || s->h_q < 1 || s->h_kv < 1 || s->d < 1) return ULY_ERR_INVALID_ARG;
  if (s->n % s->P || s->h_q % s->P || s->h_q % s->h_kv) return ULY_ERR_INVALID_ARG;
  if (s->h_kv % s->P && (s->h_kv > s->P || s->P % s->h_kv)) return ULY_ERR_INVALID_ARG;
  if (s->n > (int64_t(1) << 31) - 256) return ULY_ERR_UNSUPPORTED;   // TMA coordinates are int32
  int64_t e;
  if (!elems(s->b, s->n, s->h_q, s->d, &e)) return ULY_ERR_INVALID_ARG;
  return ULY_OK;
}

// kv heads one rank holds in the head layout: H_kv / P, or one replicated
// head when H_kv < P.  Query heads per local kv head follow.
inline int64_t kv_heads_per_rank(const uly_shape& s) { return s.h_kv >= s.P ? s.h_kv / s.P : 1; }
inline int64_t group_per_rank(const uly_shape& s) { return (s.h_q / s.P) / kv_heads_per_rank(s); }

inline uly_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ULY_OK : ULY_ERR_CUDA; }

// fp16 copies of up to four bf16 tensors (f16copy.cu): tensor t's elements
// [off[t], off[t] + cnt[t]) (multiples of 8) of src[t] go, scaled by 2^-s_t,
// to the same elements of dst[t]; s_t puts the tensor's largest magnitude in
// [2^target[t], 2^(target[t]+1)).  amax (count words) receives the largest
// magnitudes as bf16 bits and shifts (count words) the s_t; both device memory.
struct F16Copies {
  const uint16_t* src[4];
  uint16_t* dst[4];
  int64_t off[4], cnt[4];
  int32_t target[4];
  int32_t count;
};
cudaError_t launch_f16_copies(const F16Copies& a, uint32_t* amax, int32_t* shifts, cudaStream_t s);

// 2^e for a shift e in [-120, 120] (a normal float: built from its exponent field).
__host__ __device__ __forceinline__ float pow2i(int e) {
#ifdef __CUDA_ARCH__
  return __int_as_float((e + 127) << 23);
#else
  union { uint32_t u; float f; } x;
  x.u = uint32_t(e + 127) << 23;
  return x.f;
#endif
}

// The global sequence rows the attention buffers hold: Q (and O, LSE, dO,
// dQ) rows [q_base, q_base + q_rows), K (and V, dK, dV) rows
// [k_base, k_base + k_rows).  The head-layout calls pass the whole sequence;
// the block calls (ring attention) one block of queries and one of keys.
struct RowBlocks {
  int64_t q_base, q_rows, k_base, k_rows;
};
inline RowBlocks whole_rows(int64_t n) { return RowBlocks{0, n, 0, n}; }
// Blocks inside [0, n), starting on tile boundaries (multiples of `tile`).
inline bool rows_ok(const RowBlocks& r, int64_t n, int64_t tile) {
  return r.q_base >= 0 && r.q_rows >= 1 && r.q_base + r.q_rows <= n && r.q_base % tile == 0 && r.k_base >= 0 &&
         r.k_rows >= 1 && r.k_base + r.k_rows <= n && r.k_base % tile == 0;
}

typedef CUresult (*TensorMapEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                      const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                      CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda).  Looked up once; the lookup result is immutable.
TensorMapEncodeFn tensor_map_encoder();

// 4-D bf16 tensor map over a head-layout tensor [P*b][n][h][d] viewed as
// dims {d, h, n, P*b}; box {64, 1, rows, 1}, 128-byte swizzle.
bool make_head_map(CUtensorMap* map, const void* base, int64_t Pb, int64_t n, int64_t h, int64_t d,
                   uint32_t box_rows);

}  // namespace uly
