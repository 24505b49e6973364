// Local causal attention backward of every virtual rank on its head slice.
//
// Training through the Ulysses layer (Accelerate guide "Sequence
// parallelism", custom training loop: the loss is backpropagated through the
// attention); the gradient of the local attention of blog "Ulysses Sequence
// Parallelism: Training with Million-Token Contexts", "How Ulysses works",
// step 4, with the same position_ids causality as the forward.
//
//   D_i   = dO_i . O_i                       (bwd_pre kernel)
//   P_ij  = exp(scale q_i.k_j - LSE_i)        recomputed from the forward LSE
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dV_j  = sum_{group heads} sum_i P_ij dO_i
//   dK_j  = scale sum_{group heads} sum_i dS_ij q_i
//   dQ_i  = scale sum_j dS_ij k_j             (fp32 reductions across key tiles)
//
// Main kernel: one CTA per (rank, batch row, kv head, 128-key tile), heaviest
// (earliest) key tiles first.  It loops over the G query heads of the kv
// head and the 64-row query tiles that can see the key tile:
//   warp 0      TMA producer (K, V once; Q / dO tiles into a 2-stage ring)
//   warp 1      TMEM owner, single-thread tcgen05 MMA issuer
//   warps 4..7  thread = key row: P^T and dS^T from S^T, dP^T (TMEM) into
//               128B-swizzled shared memory; at the end dK, dV to global
//   warps 8..11 thread = head-dim index: dQ^T tile (TMEM) -> red.add into
//               an fp32 dQ accumulator
// MMAs per query tile (M = 128 always):
//   S^T  = K  Q^T   (A: K  K-major,  B: Q  K-major)        N = 64
//   dP^T = V  dO^T  (A: V  K-major,  B: dO K-major)        N = 64
//   dV  += P^T dO   (A: P^T K-major, B: dO MN-major)       N = D
//   dK  += dS^T Q   (A: dS^T K-major, B: Q MN-major)       N = D
//   dQ^T = K^T dS^T (A: K MN-major,  B: dS^T MN-major)     N = 64
// TMEM columns: dK [0,128) dV [128,256) S^T [256,320) dP^T [320,384)
// dQ^T [384,448).  For D = 64 the dQ^T product still runs with M = 128: its
// A operand's second 64-row half points at the V tile and those output
// lanes are ignored.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace uly {
namespace bwd {

constexpr int BKV = 128;   // keys per CTA
constexpr int BQ = 64;     // query rows per inner tile
constexpr int NS = 2;      // Q/dO stages
constexpr int kThreads = 384;

struct Params {
  const int32_t* segstart;
  const int32_t* segend;
  const float* lse;     // [P*b][hq][n]
  const float* delta;   // [P*b][hq][n]
  float* dq_acc;        // [P*b][n][hq][D] fp32, pre-zeroed
  void* dk;             // [P*b][n][hkv][D]
  void* dv;
  int* status;
  int64_t n;
  int32_t b, P_sel, rank0, hq, hkv, G, nkt;
  float scale, scale_log2;
  int32_t g_f32;
  uint64_t limit_ns;
};

template <int D>
struct Layout {
  static constexpr uint32_t kKVBytes = BKV * D * 2;      // K or V tile
  static constexpr uint32_t kQBytes = BQ * D * 2;        // Q or dO tile
  static constexpr uint32_t kPBytes = BKV * BQ * 2;      // P^T or dS^T tile
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kKVBytes;
  static constexpr uint32_t kQ = kV + kKVBytes;          // NS stages of Q
  static constexpr uint32_t kDO = kQ + NS * kQBytes;     // NS stages of dO
  static constexpr uint32_t kPt = kDO + NS * kQBytes;
  static constexpr uint32_t kDSt = kPt + kPBytes;
  static constexpr uint32_t kRowStats = kDSt + kPBytes;  // 2 x (LSE*log2e, D) x 64 floats
  static constexpr uint32_t kBar = kRowStats + 2 * 2 * BQ * 4;
  static constexpr uint32_t kBytes = kBar + 256;
  static constexpr uint32_t kDynamic = kBytes + 1024;
};

struct Bars {
  uint64_t kv_full;
  uint64_t q_full[NS], q_empty[NS];
  uint64_t sdp_full, sdp_free, p_ready, pds_free, dq_full, dq_free, mma_final;
  uint64_t stats_ready[2];
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mdo, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBar);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: earliest key tiles (most query rows) first
  const int per_tile = p.P_sel * p.b * p.hkv;
  const int kt = int(blockIdx.x / per_tile);
  int rem = int(blockIdx.x % per_tile);
  const int g = rem % p.hkv;
  rem /= p.hkv;
  const int bb = rem % p.b;
  const int r = p.rank0 + rem / p.b;
  const int rb = r * p.b + bb;
  const int64_t k0 = int64_t(kt) * BKV;
  const int64_t last_key = (k0 + BKV - 1 < p.n - 1) ? (k0 + BKV - 1) : (p.n - 1);
  const int32_t* se = p.segend + int64_t(bb) * p.n;
  const int64_t q_end = se[last_key];          // rows that see this tile: [k0, q_end)
  const int64_t seg_end_min = se[k0];
  const int qt_first = int(k0 / BQ);
  const int nqt = int((q_end + BQ - 1) / BQ) - qt_first;
  const int niter = nqt * p.G;                 // (head, query tile) pairs, head-major

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    mbar_init(&bars->sdp_full, 1);
    mbar_init(&bars->sdp_free, 128);
    mbar_init(&bars->p_ready, 128);
    mbar_init(&bars->pds_free, 1);
    mbar_init(&bars->dq_full, 1);
    mbar_init(&bars->dq_free, 128);
    mbar_init(&bars->mma_final, 1);
    mbar_init(&bars->stats_ready[0], 128);
    mbar_init(&bars->stats_ready[1], 128);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const uint32_t tDK = tmem, tDV = tmem + 128, tS = tmem + 256, tDP = tmem + 320, tDQ = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mdo);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kKVBytes);
      for (int dc = 0; dc < D / 64; ++dc) {
        tma_load_4d(&mk, &bars->kv_full, smem + L::kK + dc * BKV * 128, dc * 64, g, int(k0), rb);
        tma_load_4d(&mv, &bars->kv_full, smem + L::kV + dc * BKV * 128, dc * 64, g, int(k0), rb);
      }
      int issued = 0;
      for (int it = 0; it < niter; ++it) {
        const int st = it % NS, rnd = it / NS;
        const int h = g * p.G + it / nqt;
        const int q0 = (qt_first + it % nqt) * BQ;
        if (rnd > 0 && !mbar_wait(&bars->q_empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        mbar_arrive_expect_tx(&bars->q_full[st], 2 * L::kQBytes);
        for (int dc = 0; dc < D / 64; ++dc) {
          tma_load_4d(&mq, &bars->q_full[st], smem + L::kQ + st * L::kQBytes + dc * BQ * 128, dc * 64, h, q0, rb);
          tma_load_4d(&mdo, &bars->q_full[st], smem + L::kDO + st * L::kQBytes + dc * BQ * 128, dc * 64, h, q0, rb);
        }
        issued = it + 1;
      }
      if (*abort_flag) {   // error path: let started copies land before exit
        mbar_wait(&bars->kv_full, 0, nullptr, nullptr, p.limit_ns);
        for (int x = max(0, issued - NS); x < issued; ++x)
          mbar_wait(&bars->q_full[x % NS], (x / NS) & 1, nullptr, nullptr, p.limit_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_sdp = idesc_bf16(BKV, BQ, false, false);
      const uint32_t id_grad = idesc_bf16(BKV, D, false, true);
      const uint32_t id_dq = idesc_bf16(128, BQ, true, true);
      const uint32_t k_addr = smem_u32(smem + L::kK), v_addr = smem_u32(smem + L::kV);
      const uint32_t pt_addr = smem_u32(smem + L::kPt), ds_addr = smem_u32(smem + L::kDSt);
      // dQ^T A operand (K^T, MN-major): 64-row chunks of the head dim are the
      // K tile's 16 KB column chunks; for D = 64 the second chunk is the V tile.
      const uint32_t kt_lbo = (D == 128) ? uint32_t(BKV * 128) : (L::kV - L::kK);
      bool ok = mbar_wait(&bars->kv_full, 0, abort_flag, p.status, p.limit_ns);
      tc_fence_after();
      auto issue_grads = [&](int jt) -> bool {
        const int st = jt % NS;
        if (!mbar_wait(&bars->p_ready, jt & 1, abort_flag, p.status, p.limit_ns)) return false;
        if (jt >= 1 && !mbar_wait(&bars->dq_free, (jt - 1) & 1, abort_flag, p.status, p.limit_ns)) return false;
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQ + st * L::kQBytes);
        const uint32_t do_addr = smem_u32(smem + L::kDO + st * L::kQBytes);
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t acc = (jt > 0 || kk > 0) ? 1u : 0u;
          umma_ss(tDV, sdesc_sw128(pt_addr + kk * 32, 16, 1024), sdesc_sw128(do_addr + kk * 2048, BQ * 128, 1024),
                  id_grad, acc);
          umma_ss(tDK, sdesc_sw128(ds_addr + kk * 32, 16, 1024), sdesc_sw128(q_addr + kk * 2048, BQ * 128, 1024),
                  id_grad, acc);
        }
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk)
          umma_ss(tDQ, sdesc_sw128(k_addr + kk * 2048, kt_lbo, 1024), sdesc_sw128(ds_addr + kk * 2048, BQ * 128, 1024),
                  id_dq, kk > 0 ? 1u : 0u);
        umma_commit(&bars->dq_full);
        umma_commit(&bars->pds_free);
        umma_commit(&bars->q_empty[st]);
        return true;
      };
      for (int it = 0; ok && it < niter; ++it) {
        const int st = it % NS, rnd = it / NS;
        if (!mbar_wait(&bars->q_full[st], rnd & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        if (it >= 1 && !mbar_wait(&bars->sdp_free, (it - 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t q_addr = smem_u32(smem + L::kQ + st * L::kQBytes);
        const uint32_t do_addr = smem_u32(smem + L::kDO + st * L::kQBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ka = (kk >> 2) * (BKV * 128) + (kk & 3) * 32;   // K / V chunk offset
          const uint32_t qa = (kk >> 2) * (BQ * 128) + (kk & 3) * 32;    // Q / dO chunk offset
          umma_ss(tS, sdesc_sw128(k_addr + ka, 16, 1024), sdesc_sw128(q_addr + qa, 16, 1024), id_sdp, kk > 0 ? 1u : 0u);
          umma_ss(tDP, sdesc_sw128(v_addr + ka, 16, 1024), sdesc_sw128(do_addr + qa, 16, 1024), id_sdp, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->sdp_full);
        if (it >= 1 && !issue_grads(it - 1)) { ok = false; break; }
      }
      if (ok && niter > 0) issue_grads(niter - 1);
      umma_commit(&bars->mma_final);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ P^T / dS^T
    const int row = (warp - 4) * 32 + lane;        // key row within the tile
    const uint32_t lane_off = uint32_t((warp - 4) * 32) << 16;
    const int64_t kj = k0 + row;
    const int64_t kj_end = kj < p.n ? int64_t(se[kj]) : kj;   // rows i in [kj, kj_end) see key kj
    float* stats = reinterpret_cast<float*>(smem + L::kRowStats);
    uint8_t* pt = smem + L::kPt;
    uint8_t* ds = smem + L::kDSt;
    const int tid = threadIdx.x - 128;
    bool ok = true;
    for (int it = 0; it < niter; ++it) {
      const int h = g * p.G + it / nqt;
      const int64_t q0 = int64_t(qt_first + it % nqt) * BQ;
      // row statistics of this query tile: LSE*log2(e) and D
      float* st_l = stats + (it & 1) * 2 * BQ;
      float* st_d = st_l + BQ;
      if (tid < BQ) {
        const int64_t q = q0 + tid;
        const int64_t idx = (int64_t(rb) * p.hq + h) * p.n + q;
        st_l[tid] = q < p.n ? p.lse[idx] * 1.4426950408889634f : 0.f;
      } else {
        const int64_t q = q0 + tid - BQ;
        const int64_t idx = (int64_t(rb) * p.hq + h) * p.n + q;
        st_d[tid - BQ] = q < p.n ? p.delta[idx] : 0.f;
      }
      mbar_arrive(&bars->stats_ready[it & 1]);
      if (!mbar_wait(&bars->stats_ready[it & 1], (it >> 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
      if (!mbar_wait(&bars->sdp_full, it & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t s0[32], s1[32], d0[32], d1[32];
      tmem_ld32(tS + lane_off, s0);
      tmem_ld32(tS + lane_off + 32, s1);
      tmem_ld32(tDP + lane_off, d0);
      tmem_ld32(tDP + lane_off + 32, d1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->sdp_free);
      const bool need_mask = (q0 < k0 + BKV - 1) || (q0 + BQ > seg_end_min) || (q0 + BQ > p.n);
      uint32_t pw[32], dw[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        float pv[2], dsv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = 2 * c + e;
          const uint32_t sbits = col < 32 ? s0[col] : s1[col - 32];
          const uint32_t dbits = col < 32 ? d0[col] : d1[col - 32];
          float pr = ex2_approx(__uint_as_float(sbits) * p.scale_log2 - st_l[col]);
          if (need_mask) {
            const int64_t q = q0 + col;
            if (q < kj || q >= kj_end) pr = 0.f;
          }
          pv[e] = pr;
          dsv[e] = pr * (__uint_as_float(dbits) - st_d[col]);
        }
        pw[c] = pack_bf16x2(pv[0], pv[1]);
        dw[c] = pack_bf16x2(dsv[0], dsv[1]);
      }
      if (it >= 1 && !mbar_wait(&bars->pds_free, (it - 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
      // row `row` of the [128][64] bf16 tiles: 8 chunks of 16 B, 128B-swizzled
#pragma unroll
      for (int c16 = 0; c16 < 8; ++c16) {
        const uint32_t off = sw128_offset(row, c16 * 16);
        *reinterpret_cast<uint4*>(pt + off) = make_uint4(pw[4 * c16], pw[4 * c16 + 1], pw[4 * c16 + 2], pw[4 * c16 + 3]);
        *reinterpret_cast<uint4*>(ds + off) = make_uint4(dw[4 * c16], dw[4 * c16 + 1], dw[4 * c16 + 2], dw[4 * c16 + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars->p_ready);
    }
    // ---- epilogue: dK (scaled), dV
    if (mbar_wait(&bars->mma_final, 0, abort_flag, p.status, p.limit_ns) && ok && !*abort_flag) {
      tc_fence_after();
      const bool valid = kj < p.n;
      const int64_t orow = (int64_t(rb) * p.n + kj) * p.hkv + g;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t base = which == 0 ? tDK : tDV;
        const float mul = which == 0 ? p.scale : 1.f;
        void* out = which == 0 ? p.dk : p.dv;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(base + lane_off + c, o);
          tmem_ld_wait();
          if (valid) {
            if (p.g_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + orow * D + c);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * mul, __uint_as_float(o[4 * e + 1]) * mul,
                                     __uint_as_float(o[4 * e + 2]) * mul, __uint_as_float(o[4 * e + 3]) * mul);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + orow * D + c);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * e]) * mul, __uint_as_float(o[8 * e + 1]) * mul),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 2]) * mul, __uint_as_float(o[8 * e + 3]) * mul),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 4]) * mul, __uint_as_float(o[8 * e + 5]) * mul),
                                    pack_bf16x2(__uint_as_float(o[8 * e + 6]) * mul, __uint_as_float(o[8 * e + 7]) * mul));
            }
          }
        }
      }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dQ reduction
    const int dd = (warp - 8) * 32 + lane;          // head-dim index (TMEM lane)
    const uint32_t lane_off = uint32_t((warp - 8) * 32) << 16;
    for (int it = 0; it < niter; ++it) {
      const int h = g * p.G + it / nqt;
      const int64_t q0 = int64_t(qt_first + it % nqt) * BQ;
      if (!mbar_wait(&bars->dq_full, it & 1, abort_flag, p.status, p.limit_ns)) break;
      tc_fence_after();
      uint32_t a0[32], a1[32];
      tmem_ld32(tDQ + lane_off, a0);
      tmem_ld32(tDQ + lane_off + 32, a1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->dq_free);
      if (dd < D) {
        float* base = p.dq_acc + ((int64_t(rb) * p.n + q0) * p.hq + h) * D + dd;
        const int64_t stride = int64_t(p.hq) * D;
        const int nvalid = int(p.n - q0 < BQ ? p.n - q0 : BQ);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          if (c < nvalid) atomicAdd(base + c * stride, __uint_as_float(a0[c]) * p.scale);
          if (c + 32 < nvalid) atomicAdd(base + (c + 32) * stride, __uint_as_float(a1[c]) * p.scale);
        }
      }
    }
  }

  if (warp == 1 && lane == 0) mbar_wait(&bars->mma_final, 0, nullptr, nullptr, p.limit_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dO_i . O_i for every (rank, row, head) of the selected ranks, and the
// fp32 dQ accumulator rows zeroed.  One warp per (row, head).
template <int D, bool kOF32>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const void* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      float* __restrict__ delta, float* __restrict__ dq_acc,
                                                      int64_t rb0, int64_t rows_per_rb, int64_t total_rows, int64_t n,
                                                      int32_t hq) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= total_rows) return;
  const int64_t rb = rb0 + w / rows_per_rb;
  const int64_t rem = w % rows_per_rb;      // (token, head) with head fastest
  const int64_t i = rem / hq;
  const int64_t h = rem % hq;
  const int64_t row = rb * rows_per_rb + rem;   // [P*b][n][hq] flattened
  constexpr int E = D / 32;                      // elements per lane (2 or 4)
  float acc = 0.f;
  const uint16_t* dp = dO + row * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float dv = __uint_as_float(uint32_t(dp[e]) << 16);
    float ov;
    if (kOF32)
      ov = static_cast<const float*>(o)[row * D + lane * E + e];
    else
      ov = __uint_as_float(uint32_t(static_cast<const uint16_t*>(o)[row * D + lane * E + e]) << 16);
    acc = fmaf(dv, ov, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[(rb * hq + h) * n + i] = acc;
#pragma unroll
  for (int e = 0; e < E; ++e) dq_acc[row * D + lane * E + e] = 0.f;
}

// dQ (bf16) from the fp32 accumulator of the selected ranks.
__global__ void __launch_bounds__(256) bwd_post_kernel(const float4* __restrict__ acc, uint2* __restrict__ dq,
                                                       int64_t nvec) {
  for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec; v += int64_t(gridDim.x) * blockDim.x) {
    const float4 a = acc[v];
    dq[v] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
}

template <int D>
cudaError_t launch_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                        const Params& p, int64_t grid, cudaStream_t s) {
  auto kern = attn_bwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<D>::kDynamic);
  if (e != cudaSuccess) return e;
  kern<<<unsigned(grid), kThreads, Layout<D>::kDynamic, s>>>(mq, mk, mv, mdo, p);
  return cudaGetLastError();
}

}  // namespace bwd

// Backward workspace: the segment tables (as the forward), then D
// ([P][b][hq][n] fp32), then, for bf16 gradients, the fp32 dQ accumulator.
static size_t bwd_ws_delta_off(const uly_shape* s) { return seg_workspace_bytes(s->b, s->n); }
static size_t bwd_ws_delta_bytes(const uly_shape* s) {
  return (size_t(s->P) * size_t(s->b) * size_t(s->h_q / s->P) * size_t(s->n) * 4 + 255) & ~size_t(255);
}

}  // namespace uly

using namespace uly;

extern "C" size_t ulysses_attn_bwd_workspace(const uly_shape* s, uly_dtype g_dtype) {
  if (check_shape(s) != ULY_OK || !dtype_ok(g_dtype)) return 0;
  size_t need = bwd_ws_delta_off(s) + bwd_ws_delta_bytes(s);
  if (g_dtype == ULY_BF16) need += size_t(s->b) * size_t(s->n) * size_t(s->h_q) * size_t(s->d) * 4;
  return need;
}

extern "C" uly_status ulysses_attn_bwd(const void* q_head, const void* k_head, const void* v_head, const void* o_head,
                                       uly_dtype o_dtype, const float* lse, const void* do_head,
                                       const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                       float softmax_scale, void* dq_head, void* dk_head, void* dv_head,
                                       uly_dtype g_dtype, void* ws, size_t ws_bytes, void* stream) {
  uly_status st = validate_attn(q_head, k_head, v_head, position_ids, shape, rank, ws, ws_bytes,
                                shape ? ulysses_attn_bwd_workspace(shape, g_dtype) : 0);
  if (st != ULY_OK) return st;
  if (!o_head || !lse || !do_head || !dq_head || !dk_head || !dv_head) return ULY_ERR_INVALID_ARG;
  if (!dtype_ok(o_dtype) || !dtype_ok(g_dtype)) return ULY_ERR_INVALID_ARG;
  if (!aligned(o_head, 16) || !aligned(lse, 16) || !aligned(do_head, 16) || !aligned(dq_head, 16) ||
      !aligned(dk_head, 16) || !aligned(dv_head, 16))
    return ULY_ERR_INVALID_ARG;
  const uly_shape& s = *shape;
  const int64_t hq = s.h_q / s.P, hkv = s.h_kv / s.P, Pb = int64_t(s.P) * s.b;
  const size_t gsz = dtype_size(g_dtype);
  const size_t dqb = size_t(Pb * s.n * hq * s.d) * gsz, dkb = size_t(Pb * s.n * hkv * s.d) * gsz;
  const size_t qb = size_t(Pb * s.n * hq * s.d) * 2, kb = size_t(Pb * s.n * hkv * s.d) * 2;
  const size_t ob = size_t(Pb * s.n * hq * s.d) * dtype_size(o_dtype), lb = size_t(Pb * hq * s.n) * 4;
  const void* ins[6] = {q_head, k_head, v_head, o_head, lse, do_head};
  const size_t insz[6] = {qb, kb, kb, ob, lb, qb};
  void* outs[3] = {dq_head, dk_head, dv_head};
  const size_t outsz[3] = {dqb, dkb, dkb};
  for (int a = 0; a < 3; ++a) {
    for (int b2 = 0; b2 < 6; ++b2)
      if (overlaps(outs[a], outsz[a], ins[b2], insz[b2])) return ULY_ERR_INVALID_ARG;
    for (int b2 = a + 1; b2 < 3; ++b2)
      if (overlaps(outs[a], outsz[a], outs[b2], outsz[b2])) return ULY_ERR_INVALID_ARG;
    if (overlaps(outs[a], outsz[a], ws, ws_bytes)) return ULY_ERR_INVALID_ARG;
  }

  CUtensorMap mq, mk, mv, mdo;
  if (!make_head_map(&mq, q_head, Pb, s.n, hq, s.d, bwd::BQ) || !make_head_map(&mdo, do_head, Pb, s.n, hq, s.d, bwd::BQ) ||
      !make_head_map(&mk, k_head, Pb, s.n, hkv, s.d, bwd::BKV) || !make_head_map(&mv, v_head, Pb, s.n, hkv, s.d, bwd::BKV))
    return ULY_ERR_CUDA;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  const size_t tab = (size_t(s.b) * size_t(s.n) * 4 + 255) & ~size_t(255);
  int32_t* segstart = reinterpret_cast<int32_t*>(wsb + 256);
  int32_t* segend = reinterpret_cast<int32_t*>(wsb + 256 + tab);
  float* delta = reinterpret_cast<float*>(wsb + bwd_ws_delta_off(&s));
  float* dq_acc = g_dtype == ULY_F32 ? static_cast<float*>(dq_head)
                                     : reinterpret_cast<float*>(wsb + bwd_ws_delta_off(&s) + bwd_ws_delta_bytes(&s));

  cudaError_t e = launch_segments(position_ids, segstart, segend, s.b, s.n, cs);
  if (e != cudaSuccess) return ULY_ERR_CUDA;

  const int64_t P_sel = rank < 0 ? s.P : 1;
  const int64_t rank0 = rank < 0 ? 0 : rank;
  const int64_t rb0 = rank0 * s.b, nrb = P_sel * s.b;
  const int64_t rows_per_rb = s.n * hq;
  const int64_t total_rows = nrb * rows_per_rb;
  {
    const int64_t blocks = (total_rows * 32 + 255) / 256;
    if (blocks > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    const bool of32 = o_dtype == ULY_F32;
    if (s.d == 128) {
      if (of32) bwd::bwd_pre_kernel<128, true><<<unsigned(blocks), 256, 0, cs>>>(o_head, static_cast<const uint16_t*>(do_head), delta, dq_acc, rb0, rows_per_rb, total_rows, s.n, int32_t(hq));
      else bwd::bwd_pre_kernel<128, false><<<unsigned(blocks), 256, 0, cs>>>(o_head, static_cast<const uint16_t*>(do_head), delta, dq_acc, rb0, rows_per_rb, total_rows, s.n, int32_t(hq));
    } else {
      if (of32) bwd::bwd_pre_kernel<64, true><<<unsigned(blocks), 256, 0, cs>>>(o_head, static_cast<const uint16_t*>(do_head), delta, dq_acc, rb0, rows_per_rb, total_rows, s.n, int32_t(hq));
      else bwd::bwd_pre_kernel<64, false><<<unsigned(blocks), 256, 0, cs>>>(o_head, static_cast<const uint16_t*>(do_head), delta, dq_acc, rb0, rows_per_rb, total_rows, s.n, int32_t(hq));
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return ULY_ERR_CUDA;
  }

  bwd::Params p;
  p.segstart = segstart;
  p.segend = segend;
  p.lse = lse;
  p.delta = delta;
  p.dq_acc = dq_acc;
  p.dk = dk_head;
  p.dv = dv_head;
  p.status = reinterpret_cast<int*>(wsb);
  p.n = s.n;
  p.b = int32_t(s.b);
  p.P_sel = int32_t(P_sel);
  p.rank0 = int32_t(rank0);
  p.hq = int32_t(hq);
  p.hkv = int32_t(hkv);
  p.G = int32_t(s.h_q / s.h_kv);
  p.nkt = int32_t((s.n + bwd::BKV - 1) / bwd::BKV);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(float(s.d));
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.g_f32 = g_dtype == ULY_F32;
  p.limit_ns = 2000000000ull;
  const int64_t grid = int64_t(p.nkt) * P_sel * s.b * hkv;
  if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
  e = s.d == 128 ? bwd::launch_main<128>(mq, mk, mv, mdo, p, grid, cs) : bwd::launch_main<64>(mq, mk, mv, mdo, p, grid, cs);
  if (e != cudaSuccess) return ULY_ERR_CUDA;

  if (g_dtype == ULY_BF16) {
    const int64_t first = rb0 * rows_per_rb * s.d, count = total_rows * s.d;
    const int64_t nvec = count / 4;
    bwd::bwd_post_kernel<<<1184, 256, 0, cs>>>(reinterpret_cast<const float4*>(dq_acc + first),
                                               reinterpret_cast<uint2*>(static_cast<uint16_t*>(dq_head) + first), nvec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return ULY_ERR_CUDA;
  }
  return ULY_OK;
}
