// Weighted loss aggregation across the P sequence-parallel ranks.
//
// Accelerate concept guide "Sequence parallelism", custom training loop:
// every rank's loss is weighted by its number of labels that take part in
// the loss (shift_labels other than the ignore index, -100 there); ranks with
// no such label are left out of the sum, so a NaN loss on such a rank cannot
// reach the result; the sum is divided by max(total count, 1).  The blog
// "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
// "Loss aggregation", gives the reason: ranks can hold very different numbers
// of valid tokens.  The gradient with respect to each rank's loss is
// good_r / max(G, 1) for a rank with valid tokens and 0 otherwise.
//
// Two launches:
//  * sp_count_kernel: one CTA per rank counts its valid labels (HBM-bound
//    read of b*n/P int64; 8-byte loads, four in flight per thread).
//  * sp_combine_kernel: one CTA combines the P counts and losses in double
//    precision with a fixed reduction tree (bitwise reproducible).
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace uly {
namespace {

constexpr int kCountThreads = 1024;
constexpr int kMaxRanks = 1024;

__device__ __forceinline__ long long block_sum_ll(long long v, long long* red) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < int(blockDim.x >> 5) ? red[lane] : 0;
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  }
  return v;   // valid in thread 0
}

__global__ void __launch_bounds__(kCountThreads) sp_count_kernel(const int64_t* __restrict__ labels, int64_t per_rank,
                                                                 int64_t ignore_index, int64_t* __restrict__ good) {
  __shared__ long long red[32];
  const int r = blockIdx.x;
  const int64_t* lab = labels + int64_t(r) * per_rank;
  long long c = 0;
  int64_t i = threadIdx.x;
  for (; i + 3 * kCountThreads < per_rank; i += 4 * kCountThreads) {
    const int64_t a0 = lab[i], a1 = lab[i + kCountThreads], a2 = lab[i + 2 * kCountThreads],
                  a3 = lab[i + 3 * kCountThreads];
    c += (a0 != ignore_index) + (a1 != ignore_index) + (a2 != ignore_index) + (a3 != ignore_index);
  }
  for (; i < per_rank; i += kCountThreads) c += lab[i] != ignore_index;
  c = block_sum_ll(c, red);
  if (threadIdx.x == 0) good[r] = c;
}

__global__ void __launch_bounds__(kMaxRanks) sp_combine_kernel(const float* __restrict__ losses,
                                                               int64_t* __restrict__ good, int P,
                                                               float* __restrict__ loss, float* __restrict__ dlosses) {
  __shared__ double tot[kMaxRanks];
  __shared__ long long cnt[kMaxRanks];
  const int r = threadIdx.x;
  long long g = 0;
  double t = 0.0;
  if (r < P) {
    g = good[r];
    // a rank without valid labels is skipped, not multiplied by zero
    t = g > 0 ? double(losses[r]) * double(g) : 0.0;
  }
  tot[r] = t;
  cnt[r] = g;
  __syncthreads();
  for (int half = blockDim.x / 2; half > 0; half >>= 1) {
    if (r < half) {
      tot[r] += tot[r + half];
      cnt[r] += cnt[r + half];
    }
    __syncthreads();
  }
  const double denom = double(cnt[0] > 1 ? cnt[0] : 1);
  if (r == 0) *loss = float(tot[0] / denom);
  if (r < P) dlosses[r] = g > 0 ? float(double(g) / denom) : 0.f;
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_sp_loss_aggregate(const float* losses, const int64_t* shift_labels, int64_t b,
                                                int64_t n, int32_t P, int64_t ignore_index, float* loss,
                                                int64_t* good, float* dlosses, void* stream) {
  using namespace uly;
  if (!losses || !shift_labels || !loss || !good || !dlosses) return ULY_ERR_INVALID_ARG;
  if (P < 1 || P > kMaxRanks || b < 1 || n < 1 || n % P) return ULY_ERR_INVALID_ARG;
  int64_t per_rank;
  if (!checked_mul(b, n / P, &per_rank)) return ULY_ERR_INVALID_ARG;
  if (!aligned(losses, 4) || !aligned(shift_labels, 8) || !aligned(loss, 4) || !aligned(good, 8) ||
      !aligned(dlosses, 4))
    return ULY_ERR_INVALID_ARG;
  const size_t lab_bytes = size_t(per_rank) * size_t(P) * 8;
  const void* ins[2] = {losses, shift_labels};
  const size_t insz[2] = {size_t(P) * 4, lab_bytes};
  void* outs[3] = {loss, good, dlosses};
  const size_t outsz[3] = {4, size_t(P) * 8, size_t(P) * 4};
  for (int a = 0; a < 3; ++a) {
    for (int i = 0; i < 2; ++i)
      if (overlaps(outs[a], outsz[a], ins[i], insz[i])) return ULY_ERR_INVALID_ARG;
    for (int c = a + 1; c < 3; ++c)
      if (overlaps(outs[a], outsz[a], outs[c], outsz[c])) return ULY_ERR_INVALID_ARG;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  sp_count_kernel<<<unsigned(P), kCountThreads, 0, cs>>>(shift_labels, per_rank, ignore_index, good);
  if (cudaGetLastError() != cudaSuccess) return ULY_ERR_CUDA;
  int threads = 32;
  while (threads < P) threads <<= 1;
  sp_combine_kernel<<<1, unsigned(threads), 0, cs>>>(losses, good, int(P), loss, dlosses);
  return cuda_status(cudaGetLastError());
}
