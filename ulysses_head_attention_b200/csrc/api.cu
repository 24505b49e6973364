// Entry points that are not kernels: status text, workspace status word,
// tensor-map encoding.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace uly {

TensorMapEncodeFn tensor_map_encoder() {
  static TensorMapEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<TensorMapEncodeFn>(p);
  });
  return fn;
}

bool make_head_map(CUtensorMap* map, const void* base, int64_t Pb, int64_t n, int64_t h, int64_t d,
                   uint32_t box_rows) {
  TensorMapEncodeFn enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(h), cuuint64_t(n), cuuint64_t(Pb)};
  const cuuint64_t strides[3] = {cuuint64_t(d * 2), cuuint64_t(h * d * 2), cuuint64_t(n * h * d * 2)};
  const cuuint32_t box[4] = {64, 1, box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace uly

extern "C" const char* ulysses_status_string(uly_status s) {
  switch (s) {
    case ULY_OK: return "ok";
    case ULY_ERR_INVALID_ARG: return "invalid argument";
    case ULY_ERR_UNSUPPORTED: return "unsupported size or type";
    case ULY_ERR_CUDA: return "CUDA error";
    case ULY_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case ULY_ERR_TIMEOUT: return "a kernel gave up waiting on its own pipeline";
    case ULY_ERR_BOUNDS: return "debug build: an index fell outside its buffer";
  }
  return "unknown status";
}

extern "C" uly_status ulysses_workspace_status(void* ws, void* stream, int32_t* code) {
  if (!ws || !code || !uly::aligned(ws, 256)) return ULY_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return ULY_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ULY_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(word), s) != cudaSuccess) return ULY_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ULY_ERR_CUDA;
  *code = word == 0                    ? ULY_OK
          : word == uly::kDevSmemAlign ? ULY_ERR_CUDA
          : word == uly::kDevBounds    ? ULY_ERR_BOUNDS
                                       : ULY_ERR_TIMEOUT;
  return ULY_OK;
}
