// Self-test of the failure path every attention kernel shares: a bounded
// mbarrier wait that runs out.
//
// The attention kernels wait on their own pipeline stages (TMA copies landing,
// tensor-core MMAs completing, softmax warps handing tiles back).  On valid
// input every wait completes; should one not, the wait gives up after its
// time limit, raises the CTA's abort flag and the workspace status word, the
// other roles see the flag and stop, the producer lets its copies in flight
// land, and the TMEM owner frees TMEM before the kernel returns.  This kernel
// runs exactly that sequence with the attention kernels' own helpers, on a
// barrier nothing ever arrives at, so the path can be checked on a GPU
// without a fault, a trap or an unbounded spin.
//
// One CTA of 384 threads, the attention kernels' shape:
//   warp 0 lane 0   starts one real bulk copy (1 KB of the workspace into
//                   shared memory), then waits on the dead barrier; on the
//                   way out it waits (bounded) for its copy to land
//   warp 1          allocates 512 TMEM columns; waits as a whole warp
//                   (mbar_wait_warp) on the dead barrier; frees TMEM
//   warps 4..11     wait one thread each (mbar_wait) on the dead barrier
// Whichever wait reaches the limit first records kDevTimeout; the rest
// return once they see the abort flag.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"
#include "sm100.cuh"

namespace uly {
namespace selftest {

constexpr int kThreads = 384;
constexpr uint32_t kCopyBytes = 1024;

struct Smem {
  alignas(128) uint8_t buf[kCopyBytes];
  uint64_t dead;        // no thread ever arrives here
  uint64_t copy_done;   // completes when the bulk copy lands
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
wait_timeout_kernel(const uint8_t* __restrict__ src, int* status, uint64_t limit_ns) {
  __shared__ Smem sm;
  volatile int* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sm.dead, 1);
    mbar_init(&sm.copy_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.copy_done, kCopyBytes);
      bulk_load(sm.buf, src, kCopyBytes, &sm.copy_done);
      mbar_wait(&sm.dead, 0, abort_flag, status, limit_ns);
      // error path: let the copy this thread started land before exit
      mbar_wait(&sm.copy_done, 0, nullptr, nullptr, limit_ns);
    }
  } else if (warp == 1) {
    mbar_wait_warp(&sm.dead, 0, abort_flag, status, limit_ns);
  } else if (warp >= 4) {
    mbar_wait(&sm.dead, 0, abort_flag, status, limit_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace selftest
}  // namespace uly

extern "C" uly_status ulysses_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
  using namespace uly;
  if (!ws || !aligned(ws, 256) || ws_bytes < 256 + selftest::kCopyBytes) return ULY_ERR_WORKSPACE;
  if (limit_ns < 1000 || limit_ns > 5000000000ull) return ULY_ERR_INVALID_ARG;
  const uint8_t* src = static_cast<const uint8_t*>(ws) + 256;
  selftest::wait_timeout_kernel<<<1, selftest::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      src, static_cast<int*>(ws), limit_ns);
  return cuda_status(cudaGetLastError());
}
