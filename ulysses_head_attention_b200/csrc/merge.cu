// Log-sum-exp merge of the partial attention results of several key blocks.
//
// Ring attention and the Ulysses + ring hybrid (Accelerate concept guide
// "Sequence parallelism", "How Ulysses SP differs from FSDP CP"; blog
// "Ulysses Sequence Parallelism: Training with Million-Token Contexts") shard
// the sequence and pass key/value blocks between ranks; each rank computes
// its queries' attention over one block at a time (ulysses_attn_fwd_kv_range)
// and combines the partial results:
//   LSE = log sum_b exp(LSE_b),   O = sum_b exp(LSE_b - LSE) O_b,
// with rows that saw no key in any block left at O = 0, LSE = -inf.
//
// One warp per output row (rank, batch row, token, head): lanes 0..B-1 read
// the B partial LSEs (warp max and sum by shuffles), then every lane combines
// d/32 consecutive elements of the B partial rows.  HBM-bound: B+1 fp32 rows
// read, one row written, per output row.
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace uly {
namespace {

constexpr int kMergeWarps = 8;
constexpr int kMaxParts = 32;

template <int D, bool kOutF32>
__global__ void __launch_bounds__(32 * kMergeWarps) lse_merge_kernel(const float* __restrict__ o_parts,
                                                                     const float* __restrict__ lse_parts, int nparts,
                                                                     int64_t rows, int64_t n, int64_t h,
                                                                     void* __restrict__ o, float* __restrict__ lse) {
  constexpr int E = D / 32;   // elements per lane
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  // row = (rb * n + t) * h + j in the O layout; LSE layout is [rb][h][n]
  const int64_t j = row % h, t = (row / h) % n, rb = row / (h * n);
  const int64_t lidx = (rb * h + j) * n + t;
  const int64_t part_rows = rows;   // rows per part, for both layouts
  float lb = -INFINITY;
  if (lane < nparts) lb = lse_parts[int64_t(lane) * part_rows + lidx];
  float m = lb;
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  const bool any = m != -INFINITY;
  float w = (any && lb != -INFINITY) ? expf(lb - m) : 0.f;
  float s = w;
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float inv_s = any ? 1.f / s : 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int b = 0; b < nparts; ++b) {
    const float wb = __shfl_sync(0xffffffffu, w, b) * inv_s;
    if (wb == 0.f) continue;   // uniform across the warp
    const float* src = o_parts + (int64_t(b) * part_rows + row) * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = fmaf(wb, src[e], acc[e]);
  }
  if (kOutF32) {
    float* dst = static_cast<float*>(o) + row * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) dst[e] = acc[e];
  } else {
    uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(o) + row * D + lane * E);
#pragma unroll
    for (int e = 0; e < E; e += 2) dst[e / 2] = pack_bf16x2(acc[e], acc[e + 1]);
  }
  if (lane == 0) lse[lidx] = any ? m + logf(s) : -INFINITY;
}

template <int D, bool kOutF32>
cudaError_t launch_merge(const float* o_parts, const float* lse_parts, int nparts, int64_t rows, int64_t n, int64_t h,
                         void* o, float* lse, cudaStream_t cs) {
  const int64_t blocks = (rows + kMergeWarps - 1) / kMergeWarps;
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  lse_merge_kernel<D, kOutF32><<<unsigned(blocks), 32 * kMergeWarps, 0, cs>>>(o_parts, lse_parts, nparts, rows, n,
                                                                              h, o, lse);
  return cudaGetLastError();
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_attn_lse_merge(const float* o_parts, const float* lse_parts, int32_t nparts,
                                             const uly_shape* shape, void* o_head, uly_dtype o_dtype, float* lse,
                                             void* stream) {
  using namespace uly;
  if (!o_parts || !lse_parts || !o_head || !lse || !shape || !dtype_ok(o_dtype)) return ULY_ERR_INVALID_ARG;
  const uly_status st = check_shape(shape);
  if (st != ULY_OK) return st;
  if (nparts < 1 || nparts > kMaxParts) return ULY_ERR_INVALID_ARG;
  if (shape->d != 64 && shape->d != 128) return ULY_ERR_UNSUPPORTED;
  if (!aligned(o_parts, 16) || !aligned(lse_parts, 16) || !aligned(o_head, 16) || !aligned(lse, 16))
    return ULY_ERR_INVALID_ARG;
  const uly_shape& s = *shape;
  const int64_t h = s.h_q / s.P;
  int64_t rows;
  if (!checked_mul(int64_t(s.P) * s.b, s.n * h, &rows)) return ULY_ERR_INVALID_ARG;
  const size_t part_o = size_t(rows) * size_t(s.d) * 4, part_l = size_t(rows) * 4;
  const size_t out_o = size_t(rows) * size_t(s.d) * dtype_size(o_dtype);
  if (overlaps(o_head, out_o, o_parts, part_o * size_t(nparts)) ||
      overlaps(o_head, out_o, lse_parts, part_l * size_t(nparts)) ||
      overlaps(lse, part_l, o_parts, part_o * size_t(nparts)) ||
      overlaps(lse, part_l, lse_parts, part_l * size_t(nparts)) || overlaps(o_head, out_o, lse, part_l))
    return ULY_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const bool f32 = o_dtype == ULY_F32;
  if (s.d == 128)
    e = f32 ? launch_merge<128, true>(o_parts, lse_parts, nparts, rows, s.n, h, o_head, lse, cs)
            : launch_merge<128, false>(o_parts, lse_parts, nparts, rows, s.n, h, o_head, lse, cs);
  else
    e = f32 ? launch_merge<64, true>(o_parts, lse_parts, nparts, rows, s.n, h, o_head, lse, cs)
            : launch_merge<64, false>(o_parts, lse_parts, nparts, rows, s.n, h, o_head, lse, cs);
  return cuda_status(e);
}

// ---------------------------------------------------------------------------
// ulysses_accumulate: dst += src over float32 elements (the ring passes' sums
// of per-block dQ shares and of the dK / dV that travel with a key block).
// 16-byte vectors, grid-stride; HBM-bound (two reads, one write per element).
// ---------------------------------------------------------------------------
namespace uly {
namespace {

__global__ void __launch_bounds__(256) accumulate_kernel(float4* __restrict__ dst, const float4* __restrict__ src,
                                                         int64_t nvec) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += int64_t(gridDim.x) * blockDim.x) {
    float4 a = dst[i];
    const float4 b = src[i];
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    dst[i] = a;
  }
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_accumulate(float* dst, const float* src, int64_t count, void* stream) {
  using namespace uly;
  if (!dst || !src || count < 1 || count % 4 || !aligned(dst, 16) || !aligned(src, 16)) return ULY_ERR_INVALID_ARG;
  if (overlaps(dst, size_t(count) * 4, src, size_t(count) * 4) && dst != src) return ULY_ERR_INVALID_ARG;
  const int64_t nvec = count / 4;
  const int64_t want = (nvec + 255) / 256;
  const unsigned grid = unsigned(want < 8 * 148 ? want : 8 * 148);
  accumulate_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<float4*>(dst),
                                                                          reinterpret_cast<const float4*>(src), nvec);
  return cuda_status(cudaGetLastError());
}

