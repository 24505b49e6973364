// seq <-> head re-layouts: the two all-to-alls of Ulysses sequence
// parallelism, done among P virtual ranks in one GPU's memory.
//
// Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
// "How Ulysses works", steps 3 and 5; Transformers docs "Ulysses sequence
// parallelism", figure (seq-sharded -> head-sharded -> seq-sharded).
//
// Both directions move whole runs of h*d contiguous elements (h = H/P heads
// of one token): in the seq-sharded buffer a run is a slice of one token's
// row, in the head-sharded buffer consecutive tokens' runs are adjacent.  A
// CTA takes T consecutive tokens of one source rank s and one destination
// rank r: on the head side that is one contiguous block of T*h*d elements, on
// the seq side T runs at a fixed row pitch.  So every load and store is a
// fully coalesced 16-byte vector; no shared-memory staging is needed to
// coalesce, and each thread keeps several independent loads in flight.
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace uly {
namespace {

struct RelayoutArgs {
  int64_t b, m, n;        // batch rows, tokens per rank (n/P), tokens
  int64_t vrow;           // vectors per seq-layout token row (H*d*esize / vsize)
  int64_t vpr;            // vectors per run (h*d*esize / vsize)
  int32_t vpr_shift;      // log2(vpr) when vpr is a power of two, else -1
  int32_t tile_tokens;    // T
  int32_t tiles_per_rank; // ceil(m / T)
};

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

template <typename V, bool kToHead, bool kPow2>
__global__ void __launch_bounds__(kThreads) relayout_kernel(const V* __restrict__ src, V* __restrict__ dst,
                                                            RelayoutArgs a) {
  const int64_t tile = blockIdx.x;
  const int64_t r = blockIdx.y;                       // head-sharded rank
  const int64_t per_s = a.b * a.tiles_per_rank;
  const int64_t s = tile / per_s;                     // seq-sharded rank
  const int64_t rem = tile - s * per_s;
  const int64_t bb = rem / a.tiles_per_rank;
  const int64_t u0 = (rem - bb * a.tiles_per_rank) * a.tile_tokens;
  const int64_t rows = (a.m - u0 < a.tile_tokens) ? (a.m - u0) : int64_t(a.tile_tokens);
  const int64_t total = rows * a.vpr;

  const int64_t seq_base = ((s * a.b + bb) * a.m + u0) * a.vrow + r * a.vpr;
  const int64_t head_base = ((r * a.b + bb) * a.n + s * a.m + u0) * a.vpr;

  for (int64_t i0 = threadIdx.x; i0 < total; i0 += int64_t(kThreads) * kUnroll) {
    V val[kUnroll];
    int64_t seq_idx[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * kThreads;
      int64_t row, col;
      if (kPow2) {
        row = i >> a.vpr_shift;
        col = i & (a.vpr - 1);
      } else {
        row = i / a.vpr;
        col = i - row * a.vpr;
      }
      seq_idx[u] = seq_base + row * a.vrow + col;
      if (i < total) val[u] = kToHead ? src[seq_idx[u]] : src[head_base + i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * kThreads;
      if (i < total) {
        if (kToHead)
          dst[head_base + i] = val[u];
        else
          dst[seq_idx[u]] = val[u];
      }
    }
  }
}

template <typename V, bool kToHead>
cudaError_t launch_typed(const void* src, void* dst, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                         size_t esize, cudaStream_t stream) {
  RelayoutArgs a;
  const int64_t h = H / P;
  a.b = b;
  a.m = n / P;
  a.n = n;
  a.vrow = H * d * int64_t(esize) / int64_t(sizeof(V));
  a.vpr = h * d * int64_t(esize) / int64_t(sizeof(V));
  a.vpr_shift = -1;
  for (int sh = 0; sh < 62; ++sh)
    if ((int64_t(1) << sh) == a.vpr) a.vpr_shift = sh;
  // ~64 KB of payload per CTA: enough work per block, many blocks per SM.
  const int64_t target_vectors = (64 * 1024) / int64_t(sizeof(V));
  int64_t T = target_vectors / a.vpr;
  if (T < 1) T = 1;
  if (T > a.m) T = a.m;
  a.tile_tokens = int32_t(T);
  a.tiles_per_rank = int32_t((a.m + T - 1) / T);
  const int64_t gx = int64_t(P) * b * a.tiles_per_rank;
  if (gx > 0x7FFFFFFF || P > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid{unsigned(gx), unsigned(P), 1u};
  const V* s = static_cast<const V*>(src);
  V* o = static_cast<V*>(dst);
  if (a.vpr_shift >= 0)
    relayout_kernel<V, kToHead, true><<<grid, kThreads, 0, stream>>>(s, o, a);
  else
    relayout_kernel<V, kToHead, false><<<grid, kThreads, 0, stream>>>(s, o, a);
  return cudaGetLastError();
}

template <bool kToHead>
uly_status relayout(const void* src, void* dst, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                    uly_dtype dt, void* stream) {
  if (!src || !dst || !dtype_ok(dt)) return ULY_ERR_INVALID_ARG;
  if (P < 1 || b < 1 || n < 1 || H < 1 || d < 1) return ULY_ERR_INVALID_ARG;
  if (n % P || H % P) return ULY_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16)) return ULY_ERR_INVALID_ARG;
  int64_t e;
  if (!elems(b, n, H, d, &e)) return ULY_ERR_INVALID_ARG;
  const size_t esize = dtype_size(dt);
  const size_t bytes = size_t(e) * esize;
  if (overlaps(src, bytes, dst, bytes)) return ULY_ERR_INVALID_ARG;
  if (n / P > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t run_bytes = (H / P) * d * int64_t(esize);
  cudaError_t err;
  if (run_bytes % 16 == 0)
    err = launch_typed<uint4, kToHead>(src, dst, b, n, H, d, P, esize, s);
  else if (run_bytes % 8 == 0)
    err = launch_typed<uint2, kToHead>(src, dst, b, n, H, d, P, esize, s);
  else if (run_bytes % 4 == 0)
    err = launch_typed<uint32_t, kToHead>(src, dst, b, n, H, d, P, esize, s);
  else
    err = launch_typed<uint16_t, kToHead>(src, dst, b, n, H, d, P, esize, s);
  return cuda_status(err);
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_seq_to_head(const void* x_seq, void* x_head, int64_t b, int64_t n, int64_t H,
                                          int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::relayout<true>(x_seq, x_head, b, n, H, d, P, dt, stream);
}

extern "C" uly_status ulysses_head_to_seq(const void* x_head, void* x_seq, int64_t b, int64_t n, int64_t H,
                                          int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::relayout<false>(x_head, x_seq, b, n, H, d, P, dt, stream);
}
