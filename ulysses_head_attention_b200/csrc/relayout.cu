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
#include "sm100.cuh"

namespace uly {
namespace {

#ifdef ULY_DEBUG_BOUNDS
// The debug build's record of a re-layout index outside its buffer (read and
// cleared by ulysses_debug_status).
__device__ int g_relayout_bounds;
#define ULY_RELAYOUT_STATUS (&g_relayout_bounds)
#else
#define ULY_RELAYOUT_STATUS nullptr
#endif

struct RelayoutArgs {
  int64_t b, m, n;        // batch rows, tokens per rank (n/P), tokens
  int64_t vrow;           // vectors per seq-layout token row (H*d*esize / vsize)
  int64_t vpr;            // vectors per run (h*d*esize / vsize)
  int32_t vpr_shift;      // log2(vpr) when vpr is a power of two, else -1
  int32_t tile_tokens;    // T
  int32_t tiles_per_rank; // ceil(m / T)
  int64_t total_vecs;     // vectors in either buffer (debug build checks)
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
      if (i < total && in_bounds(seq_idx[u] < a.total_vecs && head_base + i < a.total_vecs, ULY_RELAYOUT_STATUS))
        val[u] = kToHead ? src[seq_idx[u]] : src[head_base + i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * kThreads;
      if (i < total && in_bounds(seq_idx[u] < a.total_vecs && head_base + i < a.total_vecs, ULY_RELAYOUT_STATUS)) {
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
  a.total_vecs = b * n * H * d * int64_t(esize) / int64_t(sizeof(V));
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

// ---------------------------------------------------------------------------
// K/V with fewer kv heads than ranks (H_kv < P, P a multiple of H_kv): every
// rank r gets a copy of kv head g(r) = r*H_kv/P, the one its query heads
// read (the pages are silent on this case; this is the plain reading).  The
// gradient of the copies is the sum over the P/H_kv ranks holding a head.
// Both are HBM-bound: 16-byte vectors, one CTA per (rank, batch row, tile of
// tokens).
// ---------------------------------------------------------------------------
struct KvArgs {
  int64_t b, m, n, H, P;   // batch rows, tokens per rank, tokens, kv heads, ranks
  int64_t vrow;            // 16-byte vectors per head row (d * esize / 16)
  int32_t tile_tokens;
  int32_t tiles;           // tiles per (rank, batch row)
};

// x_head[r][bb][t][0][:] = x_seq[t / m][bb][t % m][g(r)][:]
__global__ void __launch_bounds__(kThreads) kv_replicate_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                                KvArgs a) {
  const int64_t tile = blockIdx.x % a.tiles;
  const int64_t rb = blockIdx.x / a.tiles;            // r * b + bb
  const int64_t r = rb / a.b, bb = rb % a.b;
  const int64_t g = r * a.H / a.P;
  const int64_t t0 = tile * a.tile_tokens;
  const int64_t t1 = t0 + a.tile_tokens < a.n ? t0 + a.tile_tokens : a.n;
  const int64_t total = (t1 - t0) * a.vrow;
  uint4* out = dst + (rb * a.n + t0) * a.vrow;
  for (int64_t k = threadIdx.x; k < total; k += kThreads) {
    const int64_t t = t0 + k / a.vrow, c = k % a.vrow;
    const int64_t s = t / a.m, u = t % a.m;
    out[k] = src[(((s * a.b + bb) * a.m + u) * a.H + g) * a.vrow + c];
  }
}

template <typename T>
__device__ __forceinline__ void add8(float (&acc)[8], const uint4* p);
template <>
__device__ __forceinline__ void add8<uint16_t>(float (&acc)[8], const uint4* p) {
  const uint4 v = *p;
  acc[0] += __uint_as_float(v.x << 16); acc[1] += __uint_as_float(v.x & 0xFFFF0000u);
  acc[2] += __uint_as_float(v.y << 16); acc[3] += __uint_as_float(v.y & 0xFFFF0000u);
  acc[4] += __uint_as_float(v.z << 16); acc[5] += __uint_as_float(v.z & 0xFFFF0000u);
  acc[6] += __uint_as_float(v.w << 16); acc[7] += __uint_as_float(v.w & 0xFFFF0000u);
}
template <>
__device__ __forceinline__ void add8<float>(float (&acc)[8], const uint4* p) {
  const uint4 v0 = p[0], v1 = p[1];
  acc[0] += __uint_as_float(v0.x); acc[1] += __uint_as_float(v0.y);
  acc[2] += __uint_as_float(v0.z); acc[3] += __uint_as_float(v0.w);
  acc[4] += __uint_as_float(v1.x); acc[5] += __uint_as_float(v1.y);
  acc[6] += __uint_as_float(v1.z); acc[7] += __uint_as_float(v1.w);
}

__device__ __forceinline__ uint32_t bf16_rne(float x) {
  const uint32_t u = __float_as_uint(x);
  if ((u & 0x7F800000u) == 0x7F800000u) return (u >> 16) | ((u & 0xFFFFu) ? 0x40u : 0u);   // inf / nan
  return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// x_seq[s][bb][u][g][:] = sum over r in [g P/H, (g+1) P/H), ascending, of
// x_head[r][bb][s m + u][0][:]; fp32 sums.  One thread per 8 elements.
template <typename T>
__global__ void __launch_bounds__(kThreads) kv_reduce_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                             KvArgs a, int64_t d) {
  constexpr int kVec = sizeof(T) == 2 ? 1 : 2;        // 16-byte vectors per 8 elements
  const int64_t groups_per_row = d / 8;               // 8-element groups per head row
  const int64_t tile = blockIdx.x % a.tiles;
  const int64_t sb = blockIdx.x / a.tiles;            // s * b + bb (output rank, batch row)
  const int64_t s = sb / a.b, bb = sb % a.b;
  const int64_t u0 = tile * a.tile_tokens;
  const int64_t u1 = u0 + a.tile_tokens < a.m ? u0 + a.tile_tokens : a.m;
  const int64_t R = a.P / a.H;
  const int64_t total = (u1 - u0) * a.H * groups_per_row;
  for (int64_t k = threadIdx.x; k < total; k += kThreads) {
    const int64_t c = k % groups_per_row;
    const int64_t g = (k / groups_per_row) % a.H;
    const int64_t u = u0 + k / (groups_per_row * a.H);
    const int64_t t = s * a.m + u;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t r = g * R; r < (g + 1) * R; ++r)
      add8<T>(acc, src + ((r * a.b + bb) * a.n + t) * groups_per_row * kVec + c * kVec);
    uint4* o = dst + ((sb * a.m + u) * a.H + g) * groups_per_row * kVec + c * kVec;
    if (sizeof(T) == 2) {
      o[0] = make_uint4(bf16_rne(acc[0]) | (bf16_rne(acc[1]) << 16), bf16_rne(acc[2]) | (bf16_rne(acc[3]) << 16),
                        bf16_rne(acc[4]) | (bf16_rne(acc[5]) << 16), bf16_rne(acc[6]) | (bf16_rne(acc[7]) << 16));
    } else {
      o[0] = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                        __float_as_uint(acc[3]));
      o[kVec - 1] = make_uint4(__float_as_uint(acc[4]), __float_as_uint(acc[5]), __float_as_uint(acc[6]),
                               __float_as_uint(acc[7]));
    }
  }
}

// Validation shared by both directions; H < P, P % H == 0 here.  The seq
// buffer holds b*n*H*d elements, the head buffer b*n*P*d (one head per rank).
uly_status kv_check(const void* src, void* dst, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                    uly_dtype dt, bool to_head, KvArgs* a) {
  if (d % 8 || d * int64_t(dtype_size(dt)) % 16) return ULY_ERR_UNSUPPORTED;
  int64_t e_seq, e_head;
  if (!elems(b, n, H, d, &e_seq) || !elems(b, n, P, d, &e_head)) return ULY_ERR_INVALID_ARG;
  const size_t es = dtype_size(dt);
  const size_t src_bytes = size_t(to_head ? e_seq : e_head) * es, dst_bytes = size_t(to_head ? e_head : e_seq) * es;
  if (overlaps(src, src_bytes, dst, dst_bytes)) return ULY_ERR_INVALID_ARG;
  a->b = b;
  a->n = n;
  a->m = n / P;
  a->H = H;
  a->P = P;
  a->vrow = d * int64_t(es) / 16;
  return ULY_OK;
}

template <bool kToHead>
uly_status kv_relayout(const void* src, void* dst, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                       uly_dtype dt, void* stream) {
  if (!src || !dst || !dtype_ok(dt)) return ULY_ERR_INVALID_ARG;
  if (P < 1 || b < 1 || n < 1 || H < 1 || d < 1 || n % P) return ULY_ERR_INVALID_ARG;
  if (H % P == 0) return relayout<kToHead>(src, dst, b, n, H, d, P, dt, stream);
  if (P % H) return ULY_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16)) return ULY_ERR_INVALID_ARG;
  KvArgs a;
  const uly_status st = kv_check(src, dst, b, n, H, d, P, dt, kToHead, &a);
  if (st != ULY_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (kToHead) {
    a.tile_tokens = int32_t(4096 / a.vrow > 0 ? 4096 / a.vrow : 1);
    a.tiles = int32_t((n + a.tile_tokens - 1) / a.tile_tokens);
    const int64_t grid = int64_t(P) * b * a.tiles;
    if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    kv_replicate_kernel<<<unsigned(grid), kThreads, 0, cs>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), a);
  } else {
    const int64_t groups = H * (d / 8);                // 8-element groups per token of the output
    a.tile_tokens = int32_t(2048 / groups > 0 ? 2048 / groups : 1);
    a.tiles = int32_t((a.m + a.tile_tokens - 1) / a.tile_tokens);
    const int64_t grid = int64_t(P) * b * a.tiles;
    if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    if (dt == ULY_BF16)
      kv_reduce_kernel<uint16_t><<<unsigned(grid), kThreads, 0, cs>>>(static_cast<const uint4*>(src),
                                                                      static_cast<uint4*>(dst), a, d);
    else
      kv_reduce_kernel<float><<<unsigned(grid), kThreads, 0, cs>>>(static_cast<const uint4*>(src),
                                                                   static_cast<uint4*>(dst), a, d);
  }
  return cuda_status(cudaGetLastError());
}

// ---------------------------------------------------------------------------
// dst[j][i][:] = src[i][j][:] for runs of run_bytes: the local permutations
// around a real (multi-process) all-to-all.  One CTA per (j, tile of i): it
// writes one contiguous block of dst and reads T runs of src at pitch B runs.
// ---------------------------------------------------------------------------
template <typename V>
__global__ void __launch_bounds__(kThreads) transpose_runs_kernel(const V* __restrict__ src, V* __restrict__ dst,
                                                                  int64_t A, int64_t B, int64_t vrun, int64_t tile,
                                                                  int64_t tiles) {
  const int64_t j = blockIdx.x / tiles, i0 = (blockIdx.x % tiles) * tile;
  const int64_t i1 = i0 + tile < A ? i0 + tile : A;
  const int64_t total = (i1 - i0) * vrun;
  V* out = dst + (j * A + i0) * vrun;
  for (int64_t k = threadIdx.x; k < total; k += kThreads) {
    const int64_t i = i0 + k / vrun, c = k % vrun;
    out[k] = src[(i * B + j) * vrun + c];
  }
}

template <typename V>
cudaError_t launch_transpose(const void* src, void* dst, int64_t A, int64_t B, int64_t run_bytes, cudaStream_t cs) {
  const int64_t vrun = run_bytes / int64_t(sizeof(V));
  const int64_t tile = (65536 / run_bytes) > 0 ? (65536 / run_bytes) : 1;   // ~64 KB per CTA
  const int64_t tiles = (A + tile - 1) / tile;
  const int64_t grid = B * tiles;
  if (grid > 0x7FFFFFFF) return cudaErrorInvalidConfiguration;
  transpose_runs_kernel<V><<<unsigned(grid), kThreads, 0, cs>>>(static_cast<const V*>(src), static_cast<V*>(dst), A, B,
                                                               vrun, tile, tiles);
  return cudaGetLastError();
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_kv_seq_to_head(const void* x_seq, void* x_head, int64_t b, int64_t n, int64_t H_kv,
                                             int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::kv_relayout<true>(x_seq, x_head, b, n, H_kv, d, P, dt, stream);
}

extern "C" uly_status ulysses_kv_head_to_seq(const void* x_head, void* x_seq, int64_t b, int64_t n, int64_t H_kv,
                                             int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::kv_relayout<false>(x_head, x_seq, b, n, H_kv, d, P, dt, stream);
}

extern "C" uly_status ulysses_seq_to_head(const void* x_seq, void* x_head, int64_t b, int64_t n, int64_t H,
                                          int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::relayout<true>(x_seq, x_head, b, n, H, d, P, dt, stream);
}

extern "C" uly_status ulysses_head_to_seq(const void* x_head, void* x_seq, int64_t b, int64_t n, int64_t H,
                                          int64_t d, int32_t P, uly_dtype dt, void* stream) {
  return uly::relayout<false>(x_head, x_seq, b, n, H, d, P, dt, stream);
}

extern "C" uly_status ulysses_transpose_runs(const void* src, void* dst, int64_t A, int64_t B, int64_t run_bytes,
                                             void* stream) {
  using namespace uly;
  if (!src || !dst || A < 1 || B < 1 || run_bytes < 1) return ULY_ERR_INVALID_ARG;
  int64_t bytes;
  if (!checked_mul(A, B, &bytes) || !checked_mul(bytes, run_bytes, &bytes)) return ULY_ERR_INVALID_ARG;
  if (overlaps(src, size_t(bytes), dst, size_t(bytes))) return ULY_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const bool a16 = aligned(src, 16) && aligned(dst, 16), a8 = aligned(src, 8) && aligned(dst, 8),
             a4 = aligned(src, 4) && aligned(dst, 4), a2 = aligned(src, 2) && aligned(dst, 2);
  if (run_bytes % 16 == 0 && a16) e = launch_transpose<uint4>(src, dst, A, B, run_bytes, cs);
  else if (run_bytes % 8 == 0 && a8) e = launch_transpose<uint2>(src, dst, A, B, run_bytes, cs);
  else if (run_bytes % 4 == 0 && a4) e = launch_transpose<uint32_t>(src, dst, A, B, run_bytes, cs);
  else if (run_bytes % 2 == 0 && a2) e = launch_transpose<uint16_t>(src, dst, A, B, run_bytes, cs);
  else e = launch_transpose<uint8_t>(src, dst, A, B, run_bytes, cs);
  return cuda_status(e);
}

// Debug build: reads and clears the re-layout kernels' bounds record.  The
// release build compiles no checks and answers ULY_ERR_UNSUPPORTED.
extern "C" uly_status ulysses_debug_status(void* stream, int32_t* code) {
  if (!code) return ULY_ERR_INVALID_ARG;
#ifdef ULY_DEBUG_BOUNDS
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int word = 0;
  if (cudaMemcpyFromSymbolAsync(&word, uly::g_relayout_bounds, sizeof(int), 0, cudaMemcpyDeviceToHost, s) !=
      cudaSuccess)
    return ULY_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ULY_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbolAsync(uly::g_relayout_bounds, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return ULY_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ULY_ERR_CUDA;
  *code = word == 0 ? ULY_OK : ULY_ERR_BOUNDS;
  return ULY_OK;
#else
  (void)stream;
  *code = ULY_OK;
  return ULY_ERR_UNSUPPORTED;
#endif
}

