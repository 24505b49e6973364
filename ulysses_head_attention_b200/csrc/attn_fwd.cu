// Local causal attention forward of every virtual rank on its head slice.
//
// Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts":
// "How Ulysses works", step 4 (each rank runs ordinary attention for its
// heads over the full sequence); causal masking and sample boundaries come
// from position_ids, not a 4D mask (position_ids paragraph).  Accelerate
// guide "Sequence parallelism", "ALST/Ulysses SP backend configuration":
// samples packed into one row must not attend to one another.
//
// Kernel structure (one CTA per (rank, batch row, query head, 128-row tile),
// heaviest tiles first):
//   warp 0      TMA producer: Q once, then K/V tiles into a 2-stage ring
//   warp 1      TMEM owner and single-thread tcgen05 MMA issuer
//   warps 4..7  softmax: thread = query row; reads S from TMEM, writes
//               P (bf16) back over S for the PV MMA, rescales O lazily
// TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D).
// Keys a tile cannot see are never loaded: the key-tile range starts at the
// tile holding the sample start of the tile's first row and ends at the
// diagonal tile; per-element masks run only on tiles that straddle the
// diagonal or a sample start.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"
#include "segments.cuh"

namespace uly {
namespace fwd {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // keys per tile
constexpr int NS = 2;          // K/V stages
constexpr int kThreads = 256;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8
constexpr int kMufuPairs = 48;              // of the 64 column pairs per row, the rest use exp2_poly

struct Params {
  const int32_t* segstart;   // [b][n]
  float* lse;                // [P][b][hq][n]
  void* o;                   // [P][b][n][hq][D]
  int* status;
  int64_t n;
  int32_t b, P_sel, rank0, hq, G, ntiles;
  float scale_log2;
  int32_t o_f32;
  uint64_t limit_ns;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTileBytes = BM * D * 2;   // a Q, K or V tile
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTileBytes;
  static constexpr uint32_t kV = kK + NS * kTileBytes;
  static constexpr uint32_t kBar = kV + NS * kTileBytes;
  static constexpr uint32_t kBytes = kBar + 256;
  static constexpr uint32_t kDynamic = kBytes + 1024;  // alignment slack
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NS], v_full[NS], k_empty[NS], v_empty[NS];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_final;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBar);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: heaviest (last) query tiles first
  const int per_tile = p.P_sel * p.b * p.hq;
  const int tile = p.ntiles - 1 - int(blockIdx.x / per_tile);
  int rem = int(blockIdx.x % per_tile);
  const int j = rem % p.hq;
  rem /= p.hq;
  const int bb = rem % p.b;
  const int r = p.rank0 + rem / p.b;
  const int rb = r * p.b + bb;
  const int g = j / p.G;
  const int64_t t0 = int64_t(tile) * BM;
  const int64_t last_row = (t0 + BM - 1 < p.n - 1) ? (t0 + BM - 1) : (p.n - 1);
  const int32_t* ss = p.segstart + int64_t(bb) * p.n;
  const int64_t seg_lo = ss[t0];
  const int64_t seg_hi = ss[last_row];
  const int kv_first = int(seg_lo / BN);
  const int nkv = int(last_row / BN) - kv_first + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_final, 1);
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
  const uint32_t tS0 = tmem;   // S buffer sb lives at tS0 + 128 * sb
  const uint32_t tO = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&mq);
      tma_prefetch_desc(&mk);
      tma_prefetch_desc(&mv);
      mbar_arrive_expect_tx(&bars->q_full, L::kTileBytes);
      for (int dc = 0; dc < D / 64; ++dc)
        tma_load_4d(&mq, &bars->q_full, smem + L::kQ + dc * BM * 128, dc * 64, j, int(t0), rb);
      int issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int st = it % NS, rnd = it / NS;
        const int k0 = (kv_first + it) * BN;
        if (rnd > 0 && !mbar_wait(&bars->k_empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        mbar_arrive_expect_tx(&bars->k_full[st], L::kTileBytes);
        for (int dc = 0; dc < D / 64; ++dc)
          tma_load_4d(&mk, &bars->k_full[st], smem + L::kK + st * L::kTileBytes + dc * BN * 128, dc * 64, g, k0, rb);
        if (rnd > 0 && !mbar_wait(&bars->v_empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) {
          issued = it * 2 + 1;
          break;
        }
        mbar_arrive_expect_tx(&bars->v_full[st], L::kTileBytes);
        for (int dc = 0; dc < D / 64; ++dc)
          tma_load_4d(&mv, &bars->v_full[st], smem + L::kV + st * L::kTileBytes + dc * BN * 128, dc * 64, g, k0, rb);
        issued = it * 2 + 2;
      }
      // Error path only: let every copy this thread started land before exit.
      if (*abort_flag) {
        mbar_wait(&bars->q_full, 0, nullptr, nullptr, p.limit_ns);
        for (int x = max(0, issued - 2 * NS); x < issued; ++x) {
          const int it = x / 2, st = it % NS, rnd = it / NS;
          mbar_wait((x & 1) ? &bars->v_full[st] : &bars->k_full[st], rnd & 1, nullptr, nullptr, p.limit_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
      const uint32_t idesc_o = idesc_bf16(BM, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::kQ);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, p.status, p.limit_ns);
      tc_fence_after();
      auto issue_pv = [&](int jt) -> bool {
        const int sb = jt & 1, st = jt % NS, rnd = jt / NS;
        if (!mbar_wait(&bars->p_full[sb], (jt >> 1) & 1, abort_flag, p.status, p.limit_ns)) return false;
        if (!mbar_wait(&bars->v_full[st], rnd & 1, abort_flag, p.status, p.limit_ns)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + L::kV + st * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = sdesc_sw128(v_addr + kk * 2048, BN * 128, 1024);
          umma_ts(tO, (tS0 + 128u * sb) + kk * 8, bdesc, idesc_o, (jt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&bars->o_done);
        umma_commit(&bars->v_empty[st]);
        return true;
      };
      for (int it = 0; ok && it < nkv; ++it) {
        const int st = it % NS, rnd = it / NS, sb = it & 1;
        if (!mbar_wait(&bars->k_full[st], rnd & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + L::kK + st * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_ss((tS0 + 128u * sb), sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), idesc_s,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[sb]);
        umma_commit(&bars->k_empty[st]);
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(nkv - 1);
      umma_commit(&bars->o_final);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int row = (warp - 4) * 32 + lane;
    const uint32_t lane_off = uint32_t((warp - 4) * 32) << 16;
    const int64_t i = t0 + row;
    const bool valid = i < p.n;
    const int64_t s_i = valid ? ss[i] : seg_hi;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    float m_used = -INFINITY, l = 0.f;   // running max (log2 units, scaled) and row sum
    bool ok = true;
    for (int it = 0; it < nkv; ++it) {
      const int sb = it & 1;
      const int64_t k0 = int64_t(kv_first + it) * BN;
      if (!mbar_wait(&bars->s_full[sb], (it >> 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t a0[32], a1[32], a2[32], a3[32];
      tmem_ld32((tS0 + 128u * sb) + lane_off + 0, a0);
      tmem_ld32((tS0 + 128u * sb) + lane_off + 32, a1);
      tmem_ld32((tS0 + 128u * sb) + lane_off + 64, a2);
      tmem_ld32((tS0 + 128u * sb) + lane_off + 96, a3);
      tmem_ld_wait();
      float x[BN];   // raw scores q.k
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        x[c] = __uint_as_float(a0[c]);
        x[32 + c] = __uint_as_float(a1[c]);
        x[64 + c] = __uint_as_float(a2[c]);
        x[96 + c] = __uint_as_float(a3[c]);
      }
      // visible key columns: lo <= c < hi (keys s_i .. i)
      const int64_t lo64 = s_i - k0, hi64 = valid ? i + 1 - k0 : lo64;
      if (lo64 > 0 || hi64 < BN) {
        const int lo = int(lo64 < 0 ? 0 : (lo64 > BN ? BN : lo64));
        const int hi = int(hi64 < lo ? lo : (hi64 > BN ? BN : hi64));
#pragma unroll
        for (int c = 0; c < BN; ++c)
          if (unsigned(c - lo) >= unsigned(hi - lo)) x[c] = -INFINITY;
      }
      // row max of the raw scores (scale > 0), four independent chains
      float m0 = x[0], m1 = x[1], m2 = x[2], m3 = x[3];
#pragma unroll
      for (int c = 4; c + 8 <= BN; c += 8) {
        m0 = fmax3(m0, x[c], x[c + 1]);
        m1 = fmax3(m1, x[c + 2], x[c + 3]);
        m2 = fmax3(m2, x[c + 4], x[c + 5]);
        m3 = fmax3(m3, x[c + 6], x[c + 7]);
      }
      m0 = fmax3(m0, x[BN - 4], x[BN - 3]);
      m1 = fmax3(m1, x[BN - 2], x[BN - 1]);
      const float mx = fmaxf(fmax3(m0, m1, m2), m3) * p.scale_log2;
      const float m_new = fmaxf(m_used, mx);
      const bool grow = m_new > m_used + kRescaleThreshold;   // also true when m_used is -inf and m_new finite
      float factor = 1.f;
      if (grow) {
        factor = ex2_approx(m_used - m_new);   // 0 when m_used is -inf
        l *= factor;
      }
      // O already holds contributions only if an earlier tile had a finite max.
      const bool rescale_o = grow && m_used != -INFINITY;
      if (grow) m_used = m_new;
      if (__any_sync(0xffffffffu, rescale_o)) {
        if (!mbar_wait(&bars->o_done, (it - 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; }
        __syncwarp();
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        tc_fence_after();
        const float f = rescale_o ? factor : 1.f;
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(tO + lane_off + c, o);
        }
      }
      const float ms = (m_used == -INFINITY) ? 0.f : m_used;
      const uint64_t nms2 = f2_pack(-ms, -ms);
      // P = 2^(scale*x - m): column pairs [0, kMufuPairs) on the MUFU unit,
      // the rest on the FMA pipe (exp2_poly), so both pipes share the load.
      uint32_t pk0[32], pk1[32];
      uint64_t sum0 = f2_pack(0.f, 0.f), sum1 = sum0, sum2 = sum0, sum3 = sum0;
#pragma unroll
      for (int c2 = 0; c2 < BN / 2; ++c2) {
        float e0, e1;
        f2_unpack(f2_fma(f2_pack(x[2 * c2], x[2 * c2 + 1]), sl2, nms2), e0, e1);
        if (c2 < kMufuPairs) {
          e0 = ex2_approx(e0);
          e1 = ex2_approx(e1);
        } else {
          e0 = exp2_poly(e0);
          e1 = exp2_poly(e1);
        }
        const uint64_t ee = f2_pack(e0, e1);
        if ((c2 & 3) == 0) sum0 = f2_add(sum0, ee);
        else if ((c2 & 3) == 1) sum1 = f2_add(sum1, ee);
        else if ((c2 & 3) == 2) sum2 = f2_add(sum2, ee);
        else sum3 = f2_add(sum3, ee);
        if (c2 < 32) pk0[c2] = pack_bf16x2(e0, e1);
        else pk1[c2 - 32] = pack_bf16x2(e0, e1);
      }
      float sa, sb2;
      f2_unpack(f2_add(f2_add(sum0, sum1), f2_add(sum2, sum3)), sa, sb2);
      l += sa + sb2;
      tmem_st32((tS0 + 128u * sb) + lane_off + 0, pk0);
      tmem_st32((tS0 + 128u * sb) + lane_off + 32, pk1);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[sb]);
    }
    // ---- epilogue: O / l and LSE
    if (mbar_wait(&bars->o_final, 0, abort_flag, p.status, p.limit_ns) && ok && !*abort_flag) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const int64_t orow = (int64_t(rb) * p.n + i) * p.hq + j;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + c, o);
        tmem_ld_wait();
        if (valid) {
          if (p.o_f32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow * D + c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(o[4 * e]) * inv_l, __uint_as_float(o[4 * e + 1]) * inv_l,
                                   __uint_as_float(o[4 * e + 2]) * inv_l, __uint_as_float(o[4 * e + 3]) * inv_l);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow * D + c);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv_l, __uint_as_float(o[8 * e + 1]) * inv_l);
              w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv_l, __uint_as_float(o[8 * e + 3]) * inv_l);
              w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv_l, __uint_as_float(o[8 * e + 5]) * inv_l);
              w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv_l, __uint_as_float(o[8 * e + 7]) * inv_l);
              dst[e] = w;
            }
          }
        }
      }
      if (valid) p.lse[(int64_t(rb) * p.hq + j) * p.n + i] = (m_used + log2f(l)) * 0.69314718055994531f;
    }
  }

  // ---- teardown: every MMA has completed once o_final fired (or the wait gave up)
  if (warp == 1 && lane == 0) mbar_wait(&bars->o_final, 0, nullptr, nullptr, p.limit_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p,
                   int64_t grid, cudaStream_t s) {
  auto kern = attn_fwd_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<D>::kDynamic);
  if (e != cudaSuccess) return e;
  kern<<<unsigned(grid), kThreads, Layout<D>::kDynamic, s>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace fwd

// Workspace layout shared by the forward and backward entry points:
//   [0, 256)                      status word (int32) + padding
//   [256, 256 + 4*b*n)            sample start of every token (int32)
//   [.., + 4*b*n)                 one past the sample end of every token (int32)
size_t seg_workspace_bytes(int64_t b, int64_t n) {
  const size_t tab = (size_t(b) * size_t(n) * 4 + 255) & ~size_t(255);
  return 256 + 2 * tab;
}

uly_status validate_attn(const void* q, const void* k, const void* v, const int64_t* pos, const uly_shape* s,
                         int32_t rank, const void* ws, size_t ws_bytes, size_t need) {
  if (!q || !k || !v || !pos || !s) return ULY_ERR_INVALID_ARG;
  uly_status st = check_shape(s);
  if (st != ULY_OK) return st;
  if (rank < -1 || rank >= s->P) return ULY_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(pos, 8)) return ULY_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return ULY_ERR_UNSUPPORTED;
  if (s->n > 0x7FFFFF00) return ULY_ERR_UNSUPPORTED;
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return ULY_ERR_WORKSPACE;
  return ULY_OK;
}

}  // namespace uly

using namespace uly;

extern "C" size_t ulysses_attn_fwd_workspace(const uly_shape* s) {
  if (check_shape(s) != ULY_OK) return 0;
  return seg_workspace_bytes(s->b, s->n);
}

extern "C" uly_status ulysses_attn_fwd(const void* q_head, const void* k_head, const void* v_head,
                                       const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                       float softmax_scale, void* o_head, uly_dtype o_dtype, float* lse, void* ws,
                                       size_t ws_bytes, void* stream) {
  uly_status st = validate_attn(q_head, k_head, v_head, position_ids, shape, rank, ws, ws_bytes,
                                shape ? ulysses_attn_fwd_workspace(shape) : 0);
  if (st != ULY_OK) return st;
  if (!o_head || !lse || !dtype_ok(o_dtype)) return ULY_ERR_INVALID_ARG;
  if (!aligned(o_head, 16) || !aligned(lse, 16)) return ULY_ERR_INVALID_ARG;
  const uly_shape& s = *shape;
  const int64_t hq = s.h_q / s.P, hkv = s.h_kv / s.P, Pb = int64_t(s.P) * s.b;
  const int64_t ntiles = (s.n + fwd::BM - 1) / fwd::BM;
  const int64_t P_sel = rank < 0 ? s.P : 1;
  const int64_t grid = ntiles * P_sel * s.b * hq;
  if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
  // Outputs must not overlap inputs.
  const size_t qbytes = size_t(Pb * s.n * hq * s.d) * 2, kvbytes = size_t(Pb * s.n * hkv * s.d) * 2;
  const size_t obytes = size_t(Pb * s.n * hq * s.d) * dtype_size(o_dtype), lbytes = size_t(Pb * hq * s.n) * 4;
  if (overlaps(o_head, obytes, q_head, qbytes) || overlaps(o_head, obytes, k_head, kvbytes) ||
      overlaps(o_head, obytes, v_head, kvbytes) || overlaps(o_head, obytes, lse, lbytes) ||
      overlaps(lse, lbytes, q_head, qbytes) || overlaps(lse, lbytes, ws, ws_bytes) ||
      overlaps(o_head, obytes, ws, ws_bytes))
    return ULY_ERR_INVALID_ARG;

  CUtensorMap mq, mk, mv;
  if (!make_head_map(&mq, q_head, Pb, s.n, hq, s.d, fwd::BM) || !make_head_map(&mk, k_head, Pb, s.n, hkv, s.d, fwd::BN) ||
      !make_head_map(&mv, v_head, Pb, s.n, hkv, s.d, fwd::BN))
    return ULY_ERR_CUDA;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int32_t* segstart = reinterpret_cast<int32_t*>(wsb + 256);
  int32_t* segend = reinterpret_cast<int32_t*>(wsb + 256 + ((size_t(s.b) * size_t(s.n) * 4 + 255) & ~size_t(255)));
  cudaError_t e = launch_segments(position_ids, segstart, segend, s.b, s.n, cs);
  if (e != cudaSuccess) return ULY_ERR_CUDA;

  fwd::Params p;
  p.segstart = segstart;
  p.lse = lse;
  p.o = o_head;
  p.status = reinterpret_cast<int*>(wsb);
  p.n = s.n;
  p.b = int32_t(s.b);
  p.P_sel = int32_t(P_sel);
  p.rank0 = rank < 0 ? 0 : rank;
  p.hq = int32_t(hq);
  p.G = int32_t(s.h_q / s.h_kv);
  p.ntiles = int32_t(ntiles);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(float(s.d));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_f32 = o_dtype == ULY_F32;
  p.limit_ns = 2000000000ull;
  e = s.d == 128 ? fwd::launch<128>(mq, mk, mv, p, grid, cs) : fwd::launch<64>(mq, mk, mv, p, grid, cs);
  return cuda_status(e);
}

// ---------------------------------------------------------------------------
// Forward with library-owned scratch (ulysses_attn_fwd_noalloc).
//
// For callers that may not allocate device memory themselves.  The scratch
// the forward needs (status word + the two per-token segment tables) lives
// in a fixed file-scope device array instead of a caller workspace.  Host
// code never hands the array's name to a kernel: in host code that name is
// only a stand-in, so the device address is looked up with
// cudaGetSymbolAddress, once per device, the first time this entry point
// runs on that device.
// ---------------------------------------------------------------------------
namespace uly {
namespace {

constexpr int64_t kNoAllocMaxTokens = int64_t(1) << 19;                     // b * n limit
constexpr size_t kNoAllocScratchBytes = 256 + 2 * size_t(kNoAllocMaxTokens) * 4;   // 4 MiB + 256 B

static __device__ __align__(256) uint8_t g_fwd_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_fwd_scratch on the current device; set up on first use.
uly_status scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ULY_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) return ULY_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return ULY_OK;
}

}  // namespace
}  // namespace uly

extern "C" uly_status ulysses_attn_fwd_noalloc(const void* q_head, const void* k_head, const void* v_head,
                                               const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                               float softmax_scale, void* o_head, uly_dtype o_dtype, float* lse,
                                               void* stream) {
  if (!shape) return ULY_ERR_INVALID_ARG;
  const uly_status sst = check_shape(shape);
  if (sst != ULY_OK) return sst;
  // Sizes beyond the fixed scratch are refused before anything is enqueued.
  if (ulysses_attn_fwd_workspace(shape) > kNoAllocScratchBytes) return ULY_ERR_WORKSPACE;
  void* scratch = nullptr;
  const uly_status st = scratch_on_current_device(&scratch);
  if (st != ULY_OK) return st;
  // Nothing in the scratch has to start at zero: every call rewrites both
  // segment tables before reading them, and the status word is only written
  // (on a pipeline timeout), never read, on this path.
  return ulysses_attn_fwd(q_head, k_head, v_head, position_ids, shape, rank, softmax_scale, o_head, o_dtype, lse,
                          scratch, kNoAllocScratchBytes, stream);
}
