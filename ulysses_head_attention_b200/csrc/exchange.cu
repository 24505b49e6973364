// The two all-to-alls of Ulysses between GPUs, fused with the re-layout:
// each rank stores its chunks straight into its peers' buffers (plain
// stores through peer-mapped pointers over NVLink / NVSwitch), then releases
// one flag per destination; a consumer waits on its flags with a bounded
// spin before it reads.
//
// Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
// "How Ulysses works", steps 3 and 5 (the all-to-all from seq-sharded to
// head-sharded and back), "Communication complexity" (each rank sends
// (P-1)/P of its shard, one chunk per peer).
//
// seq -> head, source rank r, destination s (h = H/P, m = n/P):
//   dst_s[bb][r m + t][j] = x_seq[bb][t][s h + j]      t < m, j < h
// head -> seq, source rank r (it holds heads [r h, (r+1) h) of all tokens):
//   dst_s[bb][t][r h + j] = x_head[bb][s m + t][j]
// A CTA moves T tokens of one destination: on the head side one contiguous
// block, on the seq side T runs of h*d elements at the row pitch, so every
// load and store is a 16-byte vector and no staging is needed (the same
// access pattern as the one-GPU re-layout).
//
// Completion: after its stores every thread fences at system scope; the
// CTA's thread 0 then counts the CTA in a per-destination counter (in the
// caller's workspace, zeroed by the entry point before the launch); the CTA
// that completes a destination's count fences again and stores `epoch` into
// that destination's flag slot r with release semantics at system scope.
// The flags live in the destination's memory; ulysses_wait_flags polls them
// with acquire loads, bounded in time.  No TMA, no multicast: peers' memory
// is only ever touched by these plain stores.
#include <cuda_runtime.h>
#include <cstdint>
#include <cstring>

#include "common.cuh"
#include "sm100.cuh"

namespace uly {
namespace xchg {

constexpr int kMaxRanks = 64;
constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int64_t kTileBytes = 64 * 1024;   // bytes one CTA moves (about)

struct PushArgs {
  const uint4* src;                 // this rank's buffer
  uint4* dst[kMaxRanks];            // destination buffer of every rank
  uint32_t* flags[kMaxRanks];       // flag array of every rank ([P] slots)
  uint32_t* counters;               // [P], zeroed before the launch
  int64_t b, m, n;                  // batch rows, tokens per rank, tokens
  int64_t vrow;                     // 16-byte vectors per seq-layout token row (H d es / 16)
  int64_t vpr;                      // vectors per run (h d es / 16)
  int32_t tile_tokens, tiles_per_dst;   // T; CTAs per destination = b * ceil(m / T)
  int32_t rank, P;
  uint32_t epoch;
};

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <bool kToHead>
__global__ void __launch_bounds__(kThreads) push_kernel(const PushArgs a) {
  const int s = blockIdx.y;                               // destination rank
  const int64_t bb = blockIdx.x / ((a.m + a.tile_tokens - 1) / a.tile_tokens);
  const int64_t u0 = (blockIdx.x - bb * ((a.m + a.tile_tokens - 1) / a.tile_tokens)) * a.tile_tokens;
  const int64_t rows = (a.m - u0 < a.tile_tokens) ? (a.m - u0) : int64_t(a.tile_tokens);
  const int64_t total = rows * a.vpr;
  const int r = a.rank;
  uint4* dst = a.dst[s];
  // seq side: [b][m][H] runs; head side: [b][n][h] contiguous
  int64_t seq_base, head_base;
  if (kToHead) {
    seq_base = (bb * a.m + u0) * a.vrow + int64_t(s) * a.vpr;           // source, this rank's shard
    head_base = (bb * a.n + int64_t(r) * a.m + u0) * a.vpr;             // destination rows r m + u0 ...
  } else {
    head_base = (bb * a.n + int64_t(s) * a.m + u0) * a.vpr;             // source rows s m + u0 ...
    seq_base = (bb * a.m + u0) * a.vrow + int64_t(r) * a.vpr;           // destination heads r h ...
  }
  for (int64_t i0 = threadIdx.x; i0 < total; i0 += int64_t(kThreads) * kUnroll) {
    uint4 val[kUnroll];
    int64_t sidx[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * kThreads;
      const int64_t row = i / a.vpr, col = i - row * a.vpr;
      sidx[u] = seq_base + row * a.vrow + col;
      if (i < total) val[u] = kToHead ? a.src[sidx[u]] : a.src[head_base + i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * kThreads;
      if (i < total) {
        if (kToHead)
          dst[head_base + i] = val[u];
        else
          dst[sidx[u]] = val[u];
      }
    }
  }
  __threadfence_system();   // this thread's stores, before the CTA is counted
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t done = atomicAdd(a.counters + s, 1u) + 1u;
    if (done == uint32_t(a.b) * uint32_t(a.tiles_per_dst)) {   // the last CTA of destination s
      __threadfence_system();
      st_release_sys(a.flags[s] + r, a.epoch);
    }
  }
}

// One warp polls count flags until each holds `epoch` or a later one
// (epochs increase by one per exchange; compared modulo 2^32); gives up
// after limit_ns and records kDevTimeout in *status.
__global__ void __launch_bounds__(32) wait_flags_kernel(const uint32_t* __restrict__ flags, int count, uint32_t epoch,
                                                        uint64_t limit_ns, int* status) {
  const int lane = threadIdx.x;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    bool mine = true;
    for (int i = lane; i < count; i += 32) mine = mine && int32_t(ld_acquire_sys(flags + i) - epoch) >= 0;
    if (__all_sync(0xffffffffu, mine)) return;
    if ((it & 15u) == 15u && globaltimer_ns() - t0 > limit_ns) {
      if (lane == 0) atomicExch(status, kDevTimeout);
      return;
    }
    __nanosleep(200);
  }
}

struct ReleaseArgs {
  uint32_t* slots[kMaxRanks];
};

// Thread i stores epoch into slots[i] with release semantics at system scope,
// after a system-scope fence (everything this stream ran before is visible
// to whoever acquires the slot).
__global__ void release_flags_kernel(const ReleaseArgs a, int count, uint32_t epoch) {
  if (int(threadIdx.x) < count) {
    __threadfence_system();
    st_release_sys(a.slots[threadIdx.x], epoch);
  }
}

}  // namespace xchg
}  // namespace uly

using namespace uly;

static uly_status push_impl(bool to_head, const void* src, void* const* dst, uint32_t* const* flags, int32_t rank,
                            int64_t b, int64_t n, int64_t H, int64_t d, int32_t P, uly_dtype dt, uint32_t epoch,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!src || !dst || !flags) return ULY_ERR_INVALID_ARG;
  if (P < 1 || P > xchg::kMaxRanks || rank < 0 || rank >= P) return ULY_ERR_INVALID_ARG;
  if (b < 1 || n < 1 || H < 1 || d < 1 || n % P || H % P) return ULY_ERR_INVALID_ARG;
  if (!dtype_ok(dt)) return ULY_ERR_INVALID_ARG;
  if (epoch == 0) return ULY_ERR_INVALID_ARG;   // 0 is a flag's "nothing yet"
  const int64_t es = int64_t(dtype_size(dt)), h = H / P, m = n / P;
  if ((h * d * es) % 16) return ULY_ERR_UNSUPPORTED;
  int64_t e;
  if (!elems(b, n, H, d, &e)) return ULY_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256) || ws_bytes < size_t(P) * 4) return ULY_ERR_WORKSPACE;
  if (!aligned(src, 16)) return ULY_ERR_INVALID_ARG;
  xchg::PushArgs a;
  for (int s = 0; s < P; ++s) {
    if (!dst[s] || !flags[s] || !aligned(dst[s], 16) || !aligned(flags[s], 4)) return ULY_ERR_INVALID_ARG;
    a.dst[s] = static_cast<uint4*>(dst[s]);
    a.flags[s] = flags[s];
  }
  // the source shard must not overlap this rank's own destination buffer
  const size_t shard_bytes = size_t(b * m * H * d * es);
  if (overlaps(src, shard_bytes, dst[rank], shard_bytes)) return ULY_ERR_INVALID_ARG;
  a.src = static_cast<const uint4*>(src);
  a.counters = static_cast<uint32_t*>(ws);
  a.b = b;
  a.m = m;
  a.n = n;
  a.vrow = H * d * es / 16;
  a.vpr = h * d * es / 16;
  const int64_t run_bytes = h * d * es;
  int64_t T = xchg::kTileBytes / run_bytes;
  T = T < 1 ? 1 : (T > m ? m : T);
  a.tile_tokens = int32_t(T);
  a.tiles_per_dst = int32_t((m + T - 1) / T);
  a.rank = rank;
  a.P = P;
  a.epoch = epoch;
  const int64_t gx = b * a.tiles_per_dst;
  if (gx > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, size_t(P) * 4, cs) != cudaSuccess) return ULY_ERR_CUDA;
  if (to_head)
    xchg::push_kernel<true><<<dim3(unsigned(gx), unsigned(P)), xchg::kThreads, 0, cs>>>(a);
  else
    xchg::push_kernel<false><<<dim3(unsigned(gx), unsigned(P)), xchg::kThreads, 0, cs>>>(a);
  return cuda_status(cudaGetLastError());
}

extern "C" uly_status ulysses_seq_to_head_push(const void* x_seq, void* const* dst_heads, uint32_t* const* dst_flags,
                                               int32_t rank, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                                               uly_dtype dtype, uint32_t epoch, void* ws, size_t ws_bytes,
                                               void* stream) {
  return push_impl(true, x_seq, dst_heads, dst_flags, rank, b, n, H, d, P, dtype, epoch, ws, ws_bytes, stream);
}

extern "C" uly_status ulysses_head_to_seq_push(const void* x_head, void* const* dst_seqs, uint32_t* const* dst_flags,
                                               int32_t rank, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                                               uly_dtype dtype, uint32_t epoch, void* ws, size_t ws_bytes,
                                               void* stream) {
  return push_impl(false, x_head, dst_seqs, dst_flags, rank, b, n, H, d, P, dtype, epoch, ws, ws_bytes, stream);
}

extern "C" uly_status ulysses_wait_flags(const uint32_t* flags, int32_t count, uint32_t epoch, uint64_t limit_ns,
                                         void* ws, void* stream) {
  if (!flags || count < 1 || count > 1024 || epoch == 0 || !aligned(flags, 4)) return ULY_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 60000000000ull) return ULY_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 256)) return ULY_ERR_WORKSPACE;
  xchg::wait_flags_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(flags, count, epoch, limit_ns,
                                                                            static_cast<int*>(ws));
  return cuda_status(cudaGetLastError());
}

extern "C" uly_status ulysses_release_flags(uint32_t* const* slots, int32_t count, uint32_t epoch, void* stream) {
  if (!slots || count < 1 || count > xchg::kMaxRanks || epoch == 0) return ULY_ERR_INVALID_ARG;
  xchg::ReleaseArgs a;
  for (int i = 0; i < count; ++i) {
    if (!slots[i] || !aligned(slots[i], 4)) return ULY_ERR_INVALID_ARG;
    a.slots[i] = slots[i];
  }
  xchg::release_flags_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(a, count, epoch);
  return cuda_status(cudaGetLastError());
}

extern "C" uly_status ulysses_ipc_handle(const void* dev_ptr, void* handle_out /* 64 bytes */) {
  if (!dev_ptr || !handle_out) return ULY_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, const_cast<void*>(dev_ptr)) != cudaSuccess) return ULY_ERR_CUDA;
  static_assert(sizeof(h) == 64, "CUDA IPC handles are 64 bytes");
  memcpy(handle_out, &h, sizeof(h));
  return ULY_OK;
}

extern "C" uly_status ulysses_ipc_open(const void* handle /* 64 bytes */, void** dev_ptr_out) {
  if (!handle || !dev_ptr_out) return ULY_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle, sizeof(h));
  void* p = nullptr;
  if (cudaIpcOpenMemHandle(&p, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return ULY_ERR_CUDA;
  *dev_ptr_out = p;
  return ULY_OK;
}

extern "C" uly_status ulysses_ipc_close(void* dev_ptr) {
  if (!dev_ptr) return ULY_ERR_INVALID_ARG;
  return cuda_status(cudaIpcCloseMemHandle(dev_ptr));
}
