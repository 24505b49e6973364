// One Ulysses layer step from host memory: the seq-sharded inputs come from
// (pinned) host buffers and the seq-sharded outputs go back to host buffers,
// with the copies running on their own streams so they overlap attention.
//
// Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts",
// "How Ulysses works", steps 1-6, forward and backward: seq_to_head(q, k, v)
// -> attention -> head_to_seq(O); seq_to_head(dO) -> attention backward ->
// head_to_seq(dQ, dK, dV), here for P virtual ranks on one GPU.  Every step
// is one of this library's entry points; this file only orders them and the
// copies on three streams:
//   h2d      copies q, k, v (then dO) into device staging
//   compute  position_ids (1 copy, in order behind the previous call's
//            backward, which reads them), the re-layouts and the attention
//   d2h      copies O (while the backward runs) and dQ, dK, dV back
// and three caller-owned events carry the order from one call to the next
// (the device buffers are reused):
//   events[0]  the previous call's staged q, k, v and dO are consumed (its
//              last seq_to_head, of dO, ran): this call's host-to-device
//              copies wait for it, so they overlap the previous backward
//   events[1]  the previous call's O is copied out: this call's head_to_seq(O)
//              waits for it
//   events[2]  the previous call's gradients are copied out: this call's
//              head_to_seq of the gradients waits for it.  It is also the
//              call's own completion: every output is on the host once the
//              events[2] this call records has completed.
// Events that were never recorded count as complete, so the first call
// waits for nothing.
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"

namespace uly {
namespace {

struct LayerBuffers {
  size_t q, kv, o, lse, kvo, pos, ws_f, ws_b;   // bytes of each piece
  size_t total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

bool layer_buffers(const uly_shape* s, LayerBuffers* L) {
  if (check_shape(s) != ULY_OK) return false;
  const size_t bnd = size_t(s->b) * size_t(s->n) * size_t(s->d);
  const size_t hkv_r = size_t(kv_heads_per_rank(*s)) * size_t(s->P);   // kv heads in the head layout, all ranks
  L->q = up256(bnd * size_t(s->h_q) * 2);                    // q or dO, bf16, either layout
  L->kv = up256(bnd * size_t(s->h_kv) * 2);                  // k or v, seq layout
  L->kvo = up256(bnd * hkv_r * 2);                           // k or v, head layout
  L->o = up256(bnd * size_t(s->h_q) * 4);                    // O or dQ, fp32, either layout
  L->lse = up256(size_t(s->b) * size_t(s->h_q) * size_t(s->n) * 4);
  L->pos = up256(size_t(s->b) * size_t(s->n) * 8);
  L->ws_f = up256(ulysses_attn_fwd_workspace(s));
  L->ws_b = up256(ulysses_attn_bwd_workspace(s, ULY_F32));
  // seq: q, dO, k, v, pos; head: q, dO, k, v; O head, O seq, LSE; grads head
  // dQ (o-sized), dK, dV (kv head layout, fp32); grads seq dQ, dK, dV (fp32)
  const size_t kv_f32_head = up256(bnd * hkv_r * 4), kv_f32_seq = up256(bnd * size_t(s->h_kv) * 4);
  L->total = 2 * L->q + 2 * L->kv + L->pos + 2 * L->q + 2 * L->kvo + 2 * L->o + L->lse + L->o + 2 * kv_f32_head +
             L->o + 2 * kv_f32_seq + L->ws_f + L->ws_b;
  return true;
}

}  // namespace
}  // namespace uly

using namespace uly;

extern "C" size_t ulysses_layer_step_host_bytes(const uly_shape* s) {
  LayerBuffers L;
  return layer_buffers(s, &L) ? L.total : 0;
}

extern "C" uly_status ulysses_layer_step_host(const void* q_seq, const void* k_seq, const void* v_seq,
                                              const void* do_seq, const int64_t* position_ids, const uly_shape* shape,
                                              float softmax_scale, float* o_seq, float* dq_seq, float* dk_seq,
                                              float* dv_seq, void* dev, size_t dev_bytes, void* stream,
                                              void* h2d_stream, void* d2h_stream, void* const* events) {
  LayerBuffers L;
  if (!q_seq || !k_seq || !v_seq || !do_seq || !position_ids || !o_seq || !dq_seq || !dk_seq || !dv_seq || !events)
    return ULY_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (!events[i]) return ULY_ERR_INVALID_ARG;
  if (!shape) return ULY_ERR_INVALID_ARG;
  const uly_status sst = check_shape(shape);
  if (sst != ULY_OK) return sst;
  if (shape->d != 64 && shape->d != 128) return ULY_ERR_UNSUPPORTED;
  if (!layer_buffers(shape, &L)) return ULY_ERR_INVALID_ARG;
  if (!dev || !aligned(dev, 256) || dev_bytes < L.total) return ULY_ERR_WORKSPACE;
  const uly_shape& s = *shape;
  const int64_t hkv_r = kv_heads_per_rank(s);
  const size_t bnd = size_t(s.b) * size_t(s.n) * size_t(s.d);

  // carve the device buffer
  uint8_t* p = static_cast<uint8_t*>(dev);
  auto take = [&](size_t bytes) { uint8_t* r = p; p += bytes; return static_cast<void*>(r); };
  void* d_q = take(L.q); void* d_do = take(L.q); void* d_k = take(L.kv); void* d_v = take(L.kv);
  int64_t* d_pos = static_cast<int64_t*>(take(L.pos));
  void* h_q = take(L.q); void* h_do = take(L.q); void* h_k = take(L.kvo); void* h_v = take(L.kvo);
  float* o_head = static_cast<float*>(take(L.o));
  float* o_dev = static_cast<float*>(take(L.o));
  float* lse = static_cast<float*>(take(L.lse));
  float* g_q = static_cast<float*>(take(L.o));
  const size_t kvf_head = up256(bnd * size_t(hkv_r) * size_t(s.P) * 4), kvf_seq = up256(bnd * size_t(s.h_kv) * 4);
  float* g_k = static_cast<float*>(take(kvf_head)); float* g_v = static_cast<float*>(take(kvf_head));
  float* gs_q = static_cast<float*>(take(L.o));
  float* gs_k = static_cast<float*>(take(kvf_seq)); float* gs_v = static_cast<float*>(take(kvf_seq));
  void* ws_f = take(L.ws_f); void* ws_b = take(L.ws_b);

  cudaStream_t cs = static_cast<cudaStream_t>(stream), up = static_cast<cudaStream_t>(h2d_stream),
               down = static_cast<cudaStream_t>(d2h_stream);
  cudaEvent_t inputs_consumed = static_cast<cudaEvent_t>(events[0]), o_out = static_cast<cudaEvent_t>(events[1]),
              grads_out = static_cast<cudaEvent_t>(events[2]);
  cudaEvent_t e_qkv = nullptr, e_do = nullptr, e_o = nullptr, e_g = nullptr;
  uly_status st = ULY_OK;
  auto ok = [&](cudaError_t e) { if (e != cudaSuccess && st == ULY_OK) st = ULY_ERR_CUDA; return st == ULY_OK; };
  auto call = [&](uly_status r) { if (r != ULY_OK && st == ULY_OK) st = r; return st == ULY_OK; };
  const size_t qbytes = bnd * size_t(s.h_q) * 2, kvbytes = bnd * size_t(s.h_kv) * 2;
  do {
    if (!ok(cudaEventCreateWithFlags(&e_qkv, cudaEventDisableTiming)) ||
        !ok(cudaEventCreateWithFlags(&e_do, cudaEventDisableTiming)) ||
        !ok(cudaEventCreateWithFlags(&e_o, cudaEventDisableTiming)) ||
        !ok(cudaEventCreateWithFlags(&e_g, cudaEventDisableTiming)))
      break;
    // inputs in, once the previous call has consumed its own
    if (!ok(cudaStreamWaitEvent(up, inputs_consumed, 0))) break;
    if (!ok(cudaMemcpyAsync(d_q, q_seq, qbytes, cudaMemcpyHostToDevice, up)) ||
        !ok(cudaMemcpyAsync(d_k, k_seq, kvbytes, cudaMemcpyHostToDevice, up)) ||
        !ok(cudaMemcpyAsync(d_v, v_seq, kvbytes, cudaMemcpyHostToDevice, up)) ||
        !ok(cudaEventRecord(e_qkv, up)) ||
        !ok(cudaMemcpyAsync(d_do, do_seq, qbytes, cudaMemcpyHostToDevice, up)) || !ok(cudaEventRecord(e_do, up)))
      break;
    // forward; position_ids are read until the end of the backward, so they
    // are replaced in order on the compute stream
    if (!ok(cudaMemcpyAsync(d_pos, position_ids, size_t(s.b) * size_t(s.n) * 8, cudaMemcpyHostToDevice, cs)) ||
        !ok(cudaStreamWaitEvent(cs, e_qkv, 0)))
      break;
    if (!call(ulysses_seq_to_head(d_q, h_q, s.b, s.n, s.h_q, s.d, s.P, ULY_BF16, cs)) ||
        !call(ulysses_kv_seq_to_head(d_k, h_k, s.b, s.n, s.h_kv, s.d, s.P, ULY_BF16, cs)) ||
        !call(ulysses_kv_seq_to_head(d_v, h_v, s.b, s.n, s.h_kv, s.d, s.P, ULY_BF16, cs)) ||
        !call(ulysses_attn_fwd(h_q, h_k, h_v, d_pos, &s, -1, softmax_scale, o_head, ULY_F32, lse, ws_f, L.ws_f, cs)))
      break;
    if (!ok(cudaStreamWaitEvent(cs, o_out, 0))) break;
    if (!call(ulysses_head_to_seq(o_head, o_dev, s.b, s.n, s.h_q, s.d, s.P, ULY_F32, cs)) || !ok(cudaEventRecord(e_o, cs)))
      break;
    // O out while the backward runs
    if (!ok(cudaStreamWaitEvent(down, e_o, 0)) ||
        !ok(cudaMemcpyAsync(o_seq, o_dev, bnd * size_t(s.h_q) * 4, cudaMemcpyDeviceToHost, down)) ||
        !ok(cudaEventRecord(o_out, down)))
      break;
    // backward
    if (!ok(cudaStreamWaitEvent(cs, e_do, 0))) break;
    if (!call(ulysses_seq_to_head(d_do, h_do, s.b, s.n, s.h_q, s.d, s.P, ULY_BF16, cs)) ||
        !ok(cudaEventRecord(inputs_consumed, cs)) ||
        !call(ulysses_attn_bwd(h_q, h_k, h_v, o_head, ULY_F32, lse, h_do, d_pos, &s, -1, softmax_scale, g_q, g_k, g_v,
                               ULY_F32, ws_b, L.ws_b, cs)))
      break;
    if (!ok(cudaStreamWaitEvent(cs, grads_out, 0))) break;
    if (!call(ulysses_head_to_seq(g_q, gs_q, s.b, s.n, s.h_q, s.d, s.P, ULY_F32, cs)) ||
        !call(ulysses_kv_head_to_seq(g_k, gs_k, s.b, s.n, s.h_kv, s.d, s.P, ULY_F32, cs)) ||
        !call(ulysses_kv_head_to_seq(g_v, gs_v, s.b, s.n, s.h_kv, s.d, s.P, ULY_F32, cs)) ||
        !ok(cudaEventRecord(e_g, cs)))
      break;
    // gradients out
    if (!ok(cudaStreamWaitEvent(down, e_g, 0)) ||
        !ok(cudaMemcpyAsync(dq_seq, gs_q, bnd * size_t(s.h_q) * 4, cudaMemcpyDeviceToHost, down)) ||
        !ok(cudaMemcpyAsync(dk_seq, gs_k, bnd * size_t(s.h_kv) * 4, cudaMemcpyDeviceToHost, down)) ||
        !ok(cudaMemcpyAsync(dv_seq, gs_v, bnd * size_t(s.h_kv) * 4, cudaMemcpyDeviceToHost, down)) ||
        !ok(cudaEventRecord(grads_out, down)))
      break;
  } while (false);
  // the temporary events are released once their work completes
  for (cudaEvent_t e : {e_qkv, e_do, e_o, e_g})
    if (e) cudaEventDestroy(e);
  return st;
}

extern "C" uly_status ulysses_layer_status(void* dev, const uly_shape* shape, void* stream, int32_t* code) {
  // the status words of the two attention workspaces inside the layer buffer
  LayerBuffers L;
  if (!dev || !code || !shape || !layer_buffers(shape, &L)) return ULY_ERR_INVALID_ARG;
  uint8_t* ws_f = static_cast<uint8_t*>(dev) + (L.total - L.ws_b - L.ws_f);
  uint8_t* ws_b = ws_f + L.ws_f;
  int32_t a = 0, b = 0;
  uly_status st = ulysses_workspace_status(ws_f, stream, &a);
  if (st != ULY_OK) return st;
  st = ulysses_workspace_status(ws_b, stream, &b);
  if (st != ULY_OK) return st;
  *code = a != ULY_OK ? a : b;
  return ULY_OK;
}
