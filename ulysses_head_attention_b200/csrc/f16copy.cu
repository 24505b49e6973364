// fp16 copies of bf16 tensors, each scaled by a power of two chosen from its
// largest magnitude (the attention kernels' 16-bit operands, see attn_bwd.cu
// and attn_fwd.cu).
//
// Two launches: the largest magnitude of each tensor (bf16 bit patterns with
// the sign cleared compare like the values; NaN patterns sort above
// infinity), then the copies x' = x 2^-s with s chosen so that the largest
// magnitude lands in [2^T, 2^(T+1)) for the tensor's target T.  Scaling by a
// power of two is exact; the users fold 2^s back into their results.
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace uly {
namespace {

// Tensor t's fields, selected without indexing the parameter arrays at run time.
template <typename T>
__device__ __forceinline__ T pick(const T (&x)[4], int t) { return t == 0 ? x[0] : t == 1 ? x[1] : t == 2 ? x[2] : x[3]; }

__global__ void __launch_bounds__(256) absmax_kernel(const F16Copies a, uint32_t* __restrict__ amax) {
  const int t = blockIdx.y;
  const uint4* src = reinterpret_cast<const uint4*>(pick(a.src, t) + pick(a.off, t));
  const int64_t nvec = pick(a.cnt, t) / 8;
  uint32_t m = 0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += int64_t(gridDim.x) * blockDim.x) {
    const uint4 v = src[i];
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                             __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
  }
  m = max(m & 0xFFFFu, m >> 16);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0 && m != 0) atomicMax(amax + t, m);
}

// Shift s of a tensor whose largest magnitude has bf16 bits `bits`: the
// scaled maximum 2^(ilogb(max) - s) is 2^T.  All-zero and non-finite
// tensors keep s = 0; s is clamped so 2^-s stays a normal float.
__device__ __forceinline__ int scale_shift(uint32_t bits, int target) {
  if (bits == 0 || bits >= 0x7F80u) return 0;
  const int e = int(bits >> 7);
  const int ilog = e > 0 ? e - 127 : (31 - __clz(int(bits & 0x7Fu))) - 133;
  const int sh = ilog - target;
  return sh < -120 ? -120 : (sh > 120 ? 120 : sh);
}

__global__ void __launch_bounds__(256) to_f16_kernel(const F16Copies a, const uint32_t* __restrict__ amax,
                                                     int32_t* __restrict__ shifts) {
  const int t = blockIdx.y;
  const int sh = scale_shift(amax[t], pick(a.target, t));
  if (blockIdx.x == 0 && threadIdx.x == 0) shifts[t] = sh;
  const float f = __int_as_float((127 - sh) << 23);   // 2^-sh
  const uint4* src = reinterpret_cast<const uint4*>(pick(a.src, t) + pick(a.off, t));
  uint4* dst = reinterpret_cast<uint4*>(pick(a.dst, t) + pick(a.off, t));
  const int64_t nvec = pick(a.cnt, t) / 8;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += int64_t(gridDim.x) * blockDim.x) {
    const uint4 v = src[i];
    uint4 o;
    o.x = pack_f16x2(__uint_as_float(v.x << 16) * f, __uint_as_float(v.x & 0xFFFF0000u) * f);
    o.y = pack_f16x2(__uint_as_float(v.y << 16) * f, __uint_as_float(v.y & 0xFFFF0000u) * f);
    o.z = pack_f16x2(__uint_as_float(v.z << 16) * f, __uint_as_float(v.z & 0xFFFF0000u) * f);
    o.w = pack_f16x2(__uint_as_float(v.w << 16) * f, __uint_as_float(v.w & 0xFFFF0000u) * f);
    dst[i] = o;
  }
}

}  // namespace

cudaError_t launch_f16_copies(const F16Copies& a, uint32_t* amax, int32_t* shifts, cudaStream_t cs) {
  if (a.count < 1 || a.count > 4) return cudaErrorInvalidValue;
  int64_t most = 0;
  for (int t = 0; t < a.count; ++t) most = a.cnt[t] > most ? a.cnt[t] : most;
  // a few waves of 256-thread blocks per tensor; each thread strides over 16-byte vectors
  const int64_t want = (most / 8 + 255) / 256;
  const unsigned gx = unsigned(want < 4 * 148 ? (want > 0 ? want : 1) : 4 * 148);
  cudaError_t e = cudaMemsetAsync(amax, 0, size_t(a.count) * sizeof(uint32_t), cs);
  if (e != cudaSuccess) return e;
  absmax_kernel<<<dim3(gx, unsigned(a.count)), 256, 0, cs>>>(a, amax);
  to_f16_kernel<<<dim3(gx, unsigned(a.count)), 256, 0, cs>>>(a, amax, shifts);
  return cudaGetLastError();
}

}  // namespace uly
