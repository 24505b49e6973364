// position_ids -> per-token sample start / end tables.
//
// One CTA per batch row walks the row in chunks of 8192 tokens: a max-scan of
// "t if a sample starts at t" gives the sample start of every token, and a
// min-scan (from the end) of "t+1 if a sample starts at t+1" gives the sample
// end.  O(n) work and memory; no n x n mask anywhere.
#include <cuda_runtime.h>
#include <cstdint>

#include "segments.cuh"

namespace uly {
namespace {

constexpr int kThreads = 1024;
constexpr int kItems = 8;

// Exclusive block scan (max or min) of one value per thread; *total gets the
// whole block's aggregate.  Thread 0 gets `identity`.
template <bool kMax>
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t x, int32_t* warp_tot, int32_t identity,
                                                        int32_t* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  auto op = [](int32_t a, int32_t b) { return kMax ? max(a, b) : min(a, b); };
  int32_t incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl = op(incl, y);
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    int32_t t = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, t, off);
      if (lane >= off) t = op(t, y);
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  int32_t excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = identity;
  const int32_t before = w > 0 ? warp_tot[w - 1] : identity;
  *total = warp_tot[kThreads / 32 - 1];
  __syncthreads();
  return op(before, excl);
}

__global__ void __launch_bounds__(kThreads) segments_kernel(const int64_t* __restrict__ pos,
                                                            int32_t* __restrict__ segstart,
                                                            int32_t* __restrict__ segend, int64_t n) {
  __shared__ int32_t warp_tot[kThreads / 32];
  const int64_t* row = pos + int64_t(blockIdx.x) * n;
  int32_t* st = segstart + int64_t(blockIdx.x) * n;
  int32_t* en = segend + int64_t(blockIdx.x) * n;
  constexpr int64_t kChunk = int64_t(kThreads) * kItems;
  const int32_t n32 = int32_t(n);

  // Sample start: running max of the positions where a sample starts.
  int32_t carry = -1;
  for (int64_t base = 0; base < n; base += kChunk) {
    int32_t v[kItems];
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int64_t t = base + int64_t(threadIdx.x) * kItems + k;
      const int32_t x = (t < n && (t == 0 || row[t] == 0)) ? int32_t(t) : -1;
      v[k] = k > 0 ? max(v[k - 1], x) : x;
    }
    int32_t total;
    const int32_t before = max(carry, block_exclusive_scan<true>(v[kItems - 1], warp_tot, -1, &total));
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int64_t t = base + int64_t(threadIdx.x) * kItems + k;
      if (t < n) st[t] = max(before, v[k]);
    }
    carry = max(carry, total);
  }

  // Sample end: walking from the end, running min of the next sample start.
  carry = n32;
  for (int64_t base = 0; base < n; base += kChunk) {
    int32_t v[kItems];
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int64_t i = base + int64_t(threadIdx.x) * kItems + k;   // i-th token from the end
      const int64_t t = n - 1 - i;
      const int32_t x = (i < n && t + 1 < n && row[t + 1] == 0) ? int32_t(t + 1) : n32;
      v[k] = k > 0 ? min(v[k - 1], x) : x;
    }
    int32_t total;
    const int32_t before = min(carry, block_exclusive_scan<false>(v[kItems - 1], warp_tot, n32, &total));
#pragma unroll
    for (int k = 0; k < kItems; ++k) {
      const int64_t i = base + int64_t(threadIdx.x) * kItems + k;
      if (i < n) en[n - 1 - i] = min(before, v[k]);
    }
    carry = min(carry, total);
  }
}

}  // namespace

cudaError_t launch_segments(const int64_t* position_ids, int32_t* segstart, int32_t* segend, int64_t b,
                            int64_t n, cudaStream_t s) {
  if (b > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  segments_kernel<<<unsigned(b), kThreads, 0, s>>>(position_ids, segstart, segend, n);
  return cudaGetLastError();
}

}  // namespace uly
