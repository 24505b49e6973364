// Local causal attention backward of every virtual rank on its head slice.
//
// Training through the Ulysses layer (Accelerate guide "Sequence
// parallelism", custom training loop: the loss is backpropagated through the
// attention); the gradient of the local attention of blog "Ulysses Sequence
// Parallelism: Training with Million-Token Contexts", "How Ulysses works",
// step 4, with the forward's position_ids causality.
//
//   D_i   = dO_i . O_i
//   P_ij  = exp(scale q_i.k_j - LSE_i)        (recomputed from the forward LSE)
//   dS_ij = P_ij (dO_i . v_j - D_i)
//   dV_j  = sum_{group heads} sum_i P_ij dO_i
//   dK_j  = scale sum_{group heads} sum_i dS_ij q_i
//   dQ_i  = scale sum_j dS_ij k_j
//
// Operand precision.  The tensor-core products take fp16 copies of q, k, v
// and dO, each scaled by a power of two chosen from its largest magnitude,
// so that P and dS (rounded to 16 bits before they feed dV, dK and dQ) carry
// 11 significant bits instead of bf16's 8: the bf16 rounding of P and dS
// alone gave dV and dK errors above 1e-2 on short rows and in GQA group
// sums.  Scaling by 2^-s is exact, so the products are the same numbers up
// to the known factor, which the kernels fold back in:
//   q' = q 2^-sq, k' = k 2^-sk, v' = v 2^-sv, dO' = dO 2^-sdo
//   max|q'|, max|k'| in [2^14, 2^15); max|v'| in [4, 8); max|dO'| in [8, 16)
// (v and dO are kept small so that dP' - D' = (dP - D) 2^-(sdo+sv) stays
// below 2 d 8 16 <= 32768, inside fp16's range, for d <= 128).
//  * bwd_scale: the largest magnitude of each of q, k, v, dO (rows of the
//               selected ranks), then their fp16 copies and shifts.
//
// Three attention kernels, no atomics in them (results are bitwise
// reproducible):
//  * bwd_pre:   -LSE_i*log2(e) and -D_i per (rank, head, row), written into
//               a padded workspace table of 64-row blocks, each holding the
//               block's 64 values of -LSE*log2e followed by its 64 values of
//               -D 2^-(sdo+sv) (negated so they feed packed fused
//               multiply-adds; scaled to the units of dP' = dO' v'^T).
//  * bwd_dkdv:  one CTA per (rank, batch row, kv head, 128-key tile),
//               group by group, heaviest key tile first in each.  Loops over
//               the G query heads of the kv head and the 128-row query tiles
//               that can see the key tile:
//                 warp 0      TMA producer: K, V once; the Q ring (3 stages)
//                 warp 2      TMA producer: the dO ring (2)
//                 warp 3      bulk-copy producer: the row-statistics ring (2)
//                 warp 1      TMEM owner; issues the MMAs as a converged warp
//                 warps 4..11 thread = key row, two warpgroups each taking
//                             64 of the 128 query columns
//               S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 128: the
//               shape runs the tensor core at full rate, N = 64 does not)
//               go to TMEM; the softmax frees S^T as soon as it has read it,
//               then writes P^T and dS^T as fp16 over dP^T, and they feed
//               dV += P^T dO, dK += dS^T Q as A-from-TMEM MMAs accumulating
//               in TMEM across the whole group (details at the kernel).
//               TMEM: dK [0,128) dV [128,256) S^T [256,384) dP^T [384,512).
//  * bwd_dq:    one CTA per (rank, batch row, query head, 128-row tile),
//               heaviest first; the forward's structure (K and V rings fed
//               by separate producer warps; the K ring is three deep because
//               dQ reads a K tile one step after S did, so a two-deep ring
//               would leave no time to load the next one).  S = Q K^T into a
//               double-buffered TMEM tile, dP = dO V^T, two softmax
//               warpgroups (64 columns each) turn them into dS (fp16, over S)
//               and dQ += dS K accumulates in TMEM.
//               TMEM: S_0 [0,128) S_1 [128,256) dP [256,384) dQ [384,512).
// Every kernel also takes a key range [k_lo, k_hi) (the whole sequence for
// ulysses_attn_bwd): one ring block's share of the gradients.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "common.cuh"
#include "segments.cuh"
#include "sm100.cuh"

namespace uly {
namespace bwd {

constexpr float kLog2e = 1.4426950408889634f;

// Shifts of q, k, v, dO as written by the fp16-copy kernels (f16copy.cu).
enum { kShQ = 0, kShK = 1, kShV = 2, kShDO = 3 };

// ============================================================================
// bwd_pre: D = rowsum(dO * O) and LSE*log2(e), one warp per (rank, row, head)
// ============================================================================
// stats layout: [P*b][hq][n_pad/64] blocks of {64 x -LSE*log2e, 64 x -D}
// (n_pad a multiple of 128, so a 128-row query tile is two whole blocks);
// rows n..n_pad-1 are zero.
__device__ __forceinline__ int64_t stats_index(int64_t rbh, int64_t n_pad, int64_t i) {
  return (rbh * (n_pad / 64) + i / 64) * 128 + (i & 63);
}

template <int D, bool kOF32>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const void* __restrict__ o, const uint16_t* __restrict__ dO,
                                                      const float* __restrict__ lse, float* __restrict__ stats,
                                                      const int32_t* __restrict__ shifts, int64_t rb0, int64_t n,
                                                      int64_t n_pad, int32_t hq, int64_t total, int64_t elems,
                                                      int64_t stats_elems, int* status) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= total) return;
  const int64_t per_rb = n_pad * hq;
  const int64_t rb = rb0 + w / per_rb;
  const int64_t rem = w % per_rb;
  const int64_t i = rem / hq;          // token (head fastest: consecutive warps read adjacent rows)
  const int64_t h = rem % hq;
  const int64_t sidx = stats_index(rb * hq + h, n_pad, i);
  if (!in_bounds(sidx >= 0 && sidx + 64 < stats_elems, status)) return;
  if (i >= n) {
    if (lane == 0) {
      stats[sidx] = 0.f;
      stats[sidx + 64] = 0.f;
    }
    return;
  }
  const int64_t row = (rb * n + i) * hq + h;
  if (!in_bounds((row + 1) * D <= elems, status)) return;
  constexpr int E = D / 32;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t x = row * D + lane * E + e;
    const float dv = __uint_as_float(uint32_t(dO[x]) << 16);
    const float ov = kOF32 ? static_cast<const float*>(o)[x]
                           : __uint_as_float(uint32_t(static_cast<const uint16_t*>(o)[x]) << 16);
    acc = fmaf(dv, ov, acc);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    stats[sidx] = -lse[(rb * hq + h) * n + i] * kLog2e;
    stats[sidx + 64] = -acc * pow2i(-shifts[kShDO]) * pow2i(-shifts[kShV]);
  }
}

// ============================================================================
// bwd_dkdv
// ============================================================================
namespace dkdv {

constexpr int BKV = 128;   // keys per CTA
constexpr int BQ = 128;    // query rows per inner tile (N = 128 MMAs)
// A Q tile is read by S at the start of step i - 1 and by dK at the end of
// step i, so its ring is three deep (two would expose the whole load
// latency every step); dO and the row statistics live one step less.
constexpr int NSQ = 3;     // Q stages
constexpr int NSO = 2;     // dO + row-statistics stages
#ifndef DKDV_NWG
#define DKDV_NWG 2
#endif
constexpr int kNWG = DKDV_NWG;         // softmax warpgroups, each taking kCW query columns of a tile
constexpr int kCW = BQ / kNWG;
constexpr int kThreads = 128 + 128 * kNWG;
static_assert(kNWG == 2 || kNWG == 4, "two or four softmax warpgroups");
// of each thread's kCW / 2 column pairs per tile, the first kMufuPairs take
// their exponentials on the MUFU unit, the rest on the FMA pipe (exp2_poly)
#ifndef DKDV_MUFU_PAIRS
#define DKDV_MUFU_PAIRS 32
#endif
constexpr int kMufuPairs = DKDV_MUFU_PAIRS < kCW / 2 ? DKDV_MUFU_PAIRS : kCW / 2;
constexpr uint32_t kSmemOptin = 232448;   // per-CTA dynamic shared memory limit (227 KB)
// register split: 384 threads at 168 registers, or 640 at 96
constexpr int kRegsLaunch = kNWG == 2 ? 168 : 96;
#ifndef DKDV_REGS_LO
#define DKDV_REGS_LO 72
#define DKDV_REGS_HI (DKDV_NWG == 2 ? 216 : 96)
#endif
constexpr int kRegsLo = DKDV_REGS_LO, kRegsHi = DKDV_REGS_HI;

struct Params {
  const int32_t* segend;
  const float* stats;    // see stats_index
  const int32_t* shifts; // q, k, v, dO scale shifts (launch_f16_copies)
  void* dk;              // [P*b][k_rows][hkv][D]
  void* dv;
  int* status;
  int64_t n, n_pad;      // tokens of the whole sequence; the statistics table's rows (q_rows rounded up)
  int64_t q_base, q_rows, k_base, k_rows;   // global rows held by the Q-side and K-side buffers
  int64_t k_lo, k_hi;    // only keys in [k_lo, k_hi) take part (one ring block); 0, n otherwise
  int32_t b, P_sel, rank0, hq, hkv, G;
  float scale, scale_log2;
  int32_t g_f32;
  uint64_t limit_ns;
  int64_t g_elems, stats_elems, se_elems;   // dK/dV, statistics and segment-table extents (debug build checks)
};

template <int D>
struct Layout {
  static constexpr uint32_t kKV = BKV * D * 2;
  static constexpr uint32_t kQ = BQ * D * 2;
  static constexpr uint32_t kSt = BQ * 8;                // two 64-row blocks of {-LSE*log2e, -D}
  static constexpr uint32_t oK = 0;
  static constexpr uint32_t oV = oK + kKV;
  static constexpr uint32_t oQ = oV + kKV;
  static constexpr uint32_t oDO = oQ + NSQ * kQ;
  static constexpr uint32_t oSt = oDO + NSO * kQ;
  static constexpr uint32_t oBar = oSt + NSO * kSt;
  static constexpr uint32_t kUsed = oBar + 256;
  // room to round the base up to 1024 bytes; at D = 128 the limit leaves
  // 768, and the kernel checks the base it actually got
  static constexpr uint32_t kDynamic = kUsed + 1024 < kSmemOptin ? kUsed + 1024 : kSmemOptin;
  static constexpr uint32_t kSlack = kDynamic - kUsed;
  static_assert(kUsed + 256 <= kDynamic, "dynamic shared memory above the per-CTA limit");
};

struct Bars {
  uint64_t kv_full;
  uint64_t q_full[NSQ], q_empty[NSQ], do_full[NSO], do_empty[NSO];
  uint64_t st_full[NSO], st_empty[NSO];   // row statistics: loaded by warp 3, released by the softmax
  uint64_t s_full, dp_full, x_free, p_ready, ds_ready;
  uint64_t mma_final;
  uint32_t tmem_base;
  int abort_flag;
  float score_scale;   // scale*log2(e) in the units of the fp16 copies' scores
};
static_assert(sizeof(Bars) <= 256, "barrier block outgrew its slot");

// Key-stationary dK/dV.  Per (query head, 128-row query tile) i:
//   S^T = K Q^T -> X, dP^T = V dO^T -> Y   (M = 128 keys, N = 128 queries)
//   softmax warpgroups: read S^T (then X is free), P^T = exp(...) in
//   registers; once dP^T is in, P^T goes back to Y as bf16 (dV may start),
//   then dS^T, packed side by side in the columns each chunk has just read
//   dV += P^T dO, dK += dS^T Q   (A from Y, N = D)
// TMEM: dK [0,128) dV [128,256) X [256,384) Y [384,512).  Issue order
//   S(0) dP(0) | S(1) dV(0) dK(0) dP(1) | S(2) dV(1) dK(1) dP(2) | ...
// S(i+1) only waits for the softmax to have read S^T(i), so the
// exponentials of tile i+1 run while dV(i), dK(i) and dP(i+1) do; a region
// is rewritten only after the MMAs that read it were issued (the pipe runs
// one warp's MMAs in order).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                     const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mdo,
                     const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (uint32_t(smem - smem_raw) > L::kSlack) {   // uniform across the CTA: nothing has started yet
    if (threadIdx.x == 0) atomicExch(p.status, kDevSmemAlign);
    return;
  }
  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // (rank, batch row, kv head) groups run one after another, so the CTAs
  // resident at any time share their query heads' Q / dO tiles in L2; inside
  // a group the key tiles go heaviest (first) to lightest (last)
  const int nkt = int((p.k_rows + BKV - 1) / BKV);
  const int kt = int(blockIdx.x % nkt);
  int rem = int(blockIdx.x / nkt);
  const int g = rem % p.hkv;
  rem /= p.hkv;
  const int bb = rem % p.b;
  const int r = p.rank0 + rem / p.b;
  const int rb = r * p.b + bb;
  const int64_t k0 = p.k_base + int64_t(kt) * BKV;   // global key rows [k0, k0 + BKV)
  const int64_t k_end = p.k_base + p.k_rows, q_blk_end = p.q_base + p.q_rows;
  const int64_t last_key = (k0 + BKV - 1 < k_end - 1) ? (k0 + BKV - 1) : (k_end - 1);
  const int32_t* se = p.segend + int64_t(bb) * p.n;
  // query rows that see this key tile, inside the Q block: [max(k0, q_base), q_end)
  const int64_t q_end = se[last_key] < q_blk_end ? int64_t(se[last_key]) : q_blk_end;
  const int qt_first = int((k0 > p.q_base ? k0 : p.q_base) / BQ);
  const int nqt_raw = int((q_end + BQ - 1) / BQ) - qt_first;
  const int nqt = nqt_raw > 0 ? nqt_raw : 0;
  // (query head, query tile) pairs, head-major; none when the key tile lies
  // outside [k_lo, k_hi) (its dK, dV are then zero)
  const int niter = (k0 < p.k_hi && k0 + BKV > p.k_lo && nqt > 0) ? nqt * p.G : 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < NSQ; ++s) {
      mbar_init(&bars->q_full[s], 1);
      mbar_init(&bars->q_empty[s], 1);
    }
    for (int s = 0; s < NSO; ++s) {
      mbar_init(&bars->do_full[s], 1);
      mbar_init(&bars->do_empty[s], 1);
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 128 * kNWG);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->x_free, 128 * kNWG);
    mbar_init(&bars->p_ready, 128 * kNWG);
    mbar_init(&bars->ds_ready, 128 * kNWG);
    mbar_init(&bars->mma_final, 1);
    bars->abort_flag = 0;
    bars->score_scale = p.scale_log2 * pow2i(p.shifts[kShQ]) * pow2i(p.shifts[kShK]);
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
  const uint32_t tDK = tmem, tDV = tmem + 128, tX = tmem + 256, tY = tmem + 384;


  if (warp < 4) {
  regs_split_n<kRegsLo, kRegsHi, kThreads, kRegsLaunch>(false);   // producers and the MMA issuer
  if (warp != 1) {
    // producers, one ring each so that no ring's loads wait behind another's
    // free slots: warp 0 loads K, V and the Q ring, warp 2 the dO ring (read
    // by the MMAs only), warp 3 the row-statistics ring (read by the softmax
    // only, which releases a stage once it has read it)
    if (lane == 0) {
      const bool is_q = warp == 0, is_st = warp == 3;
      const int ns = is_q ? NSQ : NSO;
      uint64_t* full = is_q ? bars->q_full : (is_st ? bars->st_full : bars->do_full);
      uint64_t* empty = is_q ? bars->q_empty : (is_st ? bars->st_empty : bars->do_empty);
      if (!is_st) tma_prefetch_desc(is_q ? &mq : &mdo);
      if (is_q && niter > 0) {
        mbar_arrive_expect_tx(&bars->kv_full, 2 * L::kKV);
        if (in_bounds(k0 - p.k_base >= 0 && k0 - p.k_base < p.k_rows, p.status))
          for (int dc = 0; dc < D / 64; ++dc) {
            tma_load_4d(&mk, &bars->kv_full, smem + L::oK + dc * BKV * 128, dc * 64, g, int(k0 - p.k_base), rb);
            tma_load_4d(&mv, &bars->kv_full, smem + L::oV + dc * BKV * 128, dc * 64, g, int(k0 - p.k_base), rb);
          }
      }
      int issued = 0;
      for (int it = 0; it < niter; ++it) {
        const int st = it % ns, rnd = it / ns;
        const int h = g * p.G + it / nqt;
        const int q0 = int((qt_first + it % nqt) * int64_t(BQ) - p.q_base);   // row in the Q-side buffers
        if (rnd > 0 && !mbar_wait(&empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        const bool q_in = in_bounds(q0 >= 0 && q0 < p.q_rows, p.status);
        if (is_q) {
          mbar_arrive_expect_tx(&full[st], L::kQ);
          if (q_in)
            for (int dc = 0; dc < D / 64; ++dc)
              tma_load_4d(&mq, &full[st], smem + L::oQ + st * L::kQ + dc * BQ * 128, dc * 64, h, q0, rb);
        } else if (is_st) {
          mbar_arrive_expect_tx(&full[st], L::kSt);
          const int64_t si = stats_index(int64_t(rb) * p.hq + h, p.n_pad, q0);
          if (q_in && in_bounds(si >= 0 && si + L::kSt / 4 <= p.stats_elems, p.status))
            bulk_load(smem + L::oSt + st * L::kSt, p.stats + si, L::kSt, &full[st]);
        } else {
          mbar_arrive_expect_tx(&full[st], L::kQ);
          if (q_in)
            for (int dc = 0; dc < D / 64; ++dc)
              tma_load_4d(&mdo, &full[st], smem + L::oDO + st * L::kQ + dc * BQ * 128, dc * 64, h, q0, rb);
        }
        issued = it + 1;
      }
      if (*abort_flag) {   // error path only: let every copy this thread started land
        if (is_q && niter > 0) mbar_wait(&bars->kv_full, 0, nullptr, nullptr, p.limit_ns);
        for (int x = max(0, issued - ns); x < issued; ++x)
          mbar_wait(&full[x % ns], (x / ns) & 1, nullptr, nullptr, p.limit_ns);
      }
    }
  } else if (warp == 1) {
    {   // whole warp; the elected lane issues
      const uint32_t id_s = idesc_f16(BKV, BQ, false, false);
      const uint32_t id_g = idesc_f16(BKV, D, false, true);
      const uint64_t k_desc = sdesc_sw128(smem_u32(smem + L::oK), 16, 1024);
      const uint64_t v_desc = sdesc_sw128(smem_u32(smem + L::oV), 16, 1024);
      auto issue_s = [&](int it) {   // S^T = K Q^T into X
        const uint64_t qd = sdesc_sw128(smem_u32(smem + L::oQ + (it % NSQ) * L::kQ), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ka = uint64_t(((kk >> 2) * (BKV * 128) + (kk & 3) * 32) / 16);
          const uint64_t qa = uint64_t(((kk >> 2) * (BQ * 128) + (kk & 3) * 32) / 16);
          umma_ss_warp(tX, k_desc + ka, qd + qa, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bars->s_full);
      };
      auto issue_dp = [&](int it) {   // dP^T = V dO^T into Y
        const uint64_t dod = sdesc_sw128(smem_u32(smem + L::oDO + (it % NSO) * L::kQ), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ka = uint64_t(((kk >> 2) * (BKV * 128) + (kk & 3) * 32) / 16);
          const uint64_t qa = uint64_t(((kk >> 2) * (BQ * 128) + (kk & 3) * 32) / 16);
          umma_ss_warp(tY, v_desc + ka, dod + qa, id_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_warp(&bars->dp_full);
      };
      // The bf16 pairs of query columns [16kk, 16kk+16) sit in Y columns
      // 32 (kk/2) + 8 (kk%2) for P^T, 16 further on for dS^T: each 32-query
      // chunk is packed as 16 columns of P^T then 16 of dS^T.  B = dO / Q,
      // MN-major.
      auto issue_grad = [&](int it, uint32_t acc_tmem, uint32_t a_tmem, uint8_t* b_smem) {
        const uint64_t bd = sdesc_sw128(smem_u32(b_smem), BQ * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          const uint32_t a_col = 32 * (kk >> 1) + 8 * (kk & 1);
          umma_ts_warp(acc_tmem, a_tmem + a_col, bd + uint64_t(kk * 2048 / 16), id_g, (it > 0 || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = niter > 0 && mbar_wait_warp(&bars->kv_full, 0, abort_flag, p.status, p.limit_ns) &&
                mbar_wait_warp(&bars->q_full[0], 0, abort_flag, p.status, p.limit_ns) &&
                mbar_wait_warp(&bars->do_full[0], 0, abort_flag, p.status, p.limit_ns);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int it = 0; ok && it < niter; ++it) {
        const bool more = it + 1 < niter;
        if (more) {
          if (!mbar_wait_warp(&bars->x_free, it & 1, abort_flag, p.status, p.limit_ns) ||
              !mbar_wait_warp(&bars->q_full[(it + 1) % NSQ], ((it + 1) / NSQ) & 1, abort_flag, p.status, p.limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(it + 1);
        }
        if (!mbar_wait_warp(&bars->p_ready, it & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        issue_grad(it, tDV, tY, smem + L::oDO + (it % NSO) * L::kQ);        // dV += P^T dO
        umma_commit_warp(&bars->do_empty[it % NSO]);
        if (!mbar_wait_warp(&bars->ds_ready, it & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        issue_grad(it, tDK, tY + 16, smem + L::oQ + (it % NSQ) * L::kQ);    // dK += dS^T Q
        umma_commit_warp(&bars->q_empty[it % NSQ]);
        if (more) {
          if (!mbar_wait_warp(&bars->do_full[(it + 1) % NSO], ((it + 1) / NSO) & 1, abort_flag, p.status, p.limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_dp(it + 1);
        }
      }
      umma_commit_warp(&bars->mma_final);
    }
  }
  } else {
    regs_split_n<kRegsLo, kRegsHi, kThreads, kRegsLaunch>(true);   // softmax warpgroups and epilogue
    const int wg = (warp - 4) >> 2;                  // query columns [kCW wg, kCW wg + kCW) of each tile
    const int row = ((warp - 4) & 3) * 32 + lane;    // key row within the tile
    const uint32_t lane_off = uint32_t(((warp - 4) & 3) * 32) << 16;
    const int64_t kj = k0 + row;
    // query rows [kj, kj_end) see key kj (none for a key outside [k_lo, k_hi))
    const int64_t kj_end = (kj < k_end && kj >= p.k_lo && kj < p.k_hi &&
                            in_bounds(int64_t(bb) * p.n + kj < p.se_elems, p.status))
                               ? (se[kj] < q_blk_end ? int64_t(se[kj]) : q_blk_end) : kj;
    bool ok = true;
    for (int it = 0; it < niter; ++it) {
      const int st = it % NSO;
      // scores come out of the MMA in units of q'.k' = q.k 2^-(sq+sk); the
      // factor is re-read from shared memory each step rather than held
      const float sl = *reinterpret_cast<volatile float*>(&bars->score_scale);
      const uint64_t sl2 = f2_pack(sl, sl);
      const int64_t q0 = int64_t(qt_first + it % nqt) * BQ;
      if (!mbar_wait(&bars->st_full[st], (it / NSO) & 1, abort_flag, p.status, p.limit_ns) ||
          !mbar_wait(&bars->s_full, it & 1, abort_flag, p.status, p.limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // this warpgroup's query columns [c0, c0 + kCW) sit in statistics block
      // c0 / 64 ({64 x -LSE*log2e, 64 x -D}) from offset c0 % 64
      constexpr int NC = kCW / 32;   // 32-column chunks of this warpgroup
      const int c0 = kCW * wg;
      const float* stt = reinterpret_cast<const float*>(smem + L::oSt + st * L::kSt) + 128 * (c0 / 64) + (c0 % 64);
      // visible query columns c of this warpgroup: lo <= c < hi (queries kj .. kj_end-1)
      const int64_t qb = q0 + c0;
      const int64_t lo64 = kj - qb, hi64 = kj_end - qb;
      const bool need_mask = lo64 > 0 || hi64 < kCW;
      const int lo = int(lo64 < 0 ? 0 : (lo64 > kCW ? kCW : lo64));
      const int hi = int(hi64 < lo ? lo : (hi64 > kCW ? kCW : hi64));
      float pr[kCW];
      uint32_t pw[kCW / 2];
      {
        // all S^T chunks in one round trip, then X may be rewritten
        uint32_t sv[NC][32];
#pragma unroll
        for (int ch = 0; ch < NC; ++ch) tmem_ld32(tX + lane_off + c0 + 32 * ch, sv[ch]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bars->x_free);
#pragma unroll
        for (int c = 0; c < kCW / 2; ++c) {
          const int j = 2 * c;
          const uint32_t s0 = sv[j / 32][j % 32], s1 = sv[j / 32][(j + 1) % 32];
          const float2 nl = *reinterpret_cast<const float2*>(stt + j);   // -LSE*log2e
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(s0), __uint_as_float(s1)), sl2, f2_pack(nl.x, nl.y)), x0, x1);
#ifdef BWD_EX2_F16X2
          // both exponentials in one MUFU operation, in fp16 (the precision P^T is stored in)
          uint32_t ph = ex2_f16x2(pack_f16x2(x0, x1));
          if (need_mask) {
            if (unsigned(j - lo) >= unsigned(hi - lo)) ph &= 0xFFFF0000u;
            if (unsigned(j + 1 - lo) >= unsigned(hi - lo)) ph &= 0x0000FFFFu;
          }
          float p0, p1;
          unpack_f16x2(ph, p0, p1);
          pw[c] = ph;
#else
          float p0, p1;
          if (c < kMufuPairs) {
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          } else {
            f2_unpack(exp2_poly2(f2_pack(x0, x1)), p0, p1);
          }
          if (need_mask) {
            if (unsigned(j - lo) >= unsigned(hi - lo)) p0 = 0.f;
            if (unsigned(j + 1 - lo) >= unsigned(hi - lo)) p1 = 0.f;
          }
          pw[c] = pack_f16x2(p0, p1);
#endif
          pr[j] = p0;
          pr[j + 1] = p1;
        }
      }
      if (!mbar_wait(&bars->dp_full, it & 1, abort_flag, p.status, p.limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        uint32_t dp[NC][32];
#pragma unroll
        for (int ch = 0; ch < NC; ++ch) tmem_ld32(tY + lane_off + c0 + 32 * ch, dp[ch]);
        tmem_ld_wait();
        // each 32-query chunk goes back over the 32 columns it came from:
        // 16 columns of P^T, then 16 of dS^T.  P^T first, so dV can start
        // while dS is computed.
#pragma unroll
        for (int ch = 0; ch < NC; ++ch) {
          uint32_t pc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pc[c] = pw[16 * ch + c];
          tmem_st16(tY + lane_off + c0 + 32 * ch, pc);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_ready);
#pragma unroll
        for (int ch = 0; ch < NC; ++ch) {
          uint32_t dw[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int j = 32 * ch + 2 * c;
            const uint32_t a0 = dp[ch][2 * c], a1 = dp[ch][2 * c + 1];
            const float2 nd = *reinterpret_cast<const float2*>(stt + 64 + j);   // -D
            float d0, d1;
            f2_unpack(f2_mul(f2_pack(pr[j], pr[j + 1]),
                             f2_add(f2_pack(__uint_as_float(a0), __uint_as_float(a1)), f2_pack(nd.x, nd.y))), d0, d1);
            dw[c] = pack_f16x2(d0, d1);
          }
          tmem_st16(tY + lane_off + c0 + 32 * ch + 16, dw);
        }
      }
      mbar_arrive(&bars->st_empty[st]);   // this step's statistics are read (release)
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready);
    }
    if (mbar_wait(&bars->mma_final, 0, abort_flag, p.status, p.limit_ns) && ok && !*abort_flag) {
      tc_fence_after();
      const int64_t orow = (int64_t(rb) * p.k_rows + (kj - p.k_base)) * p.hkv + g;
      const bool valid = kj < k_end && in_bounds(orow >= 0 && (orow + 1) * D <= p.g_elems, p.status);
      {
        // the first half of the warpgroups stores dK, the second dV, each
        // warpgroup D / (kNWG / 2) of the head-dim columns
        const int which = wg / (kNWG / 2);
        const int cbeg = (wg % (kNWG / 2)) * (D / (kNWG / 2)), cend = cbeg + D / (kNWG / 2);
        const uint32_t base = which == 0 ? tDK : tDV;
        // dK' = dS'^T q' = scale^-1 dK 2^-(sdo+sv+sq), dV' = P^T dO' = dV 2^-sdo
        const float mul = which == 0 ? p.scale * pow2i(p.shifts[kShDO]) * pow2i(p.shifts[kShV]) * pow2i(p.shifts[kShQ])
                                     : pow2i(p.shifts[kShDO]);
        void* out = which == 0 ? p.dk : p.dv;
#pragma unroll
        for (int c = cbeg; c < cend; c += 32) {
          uint32_t o[32];
          tmem_ld32(base + lane_off + c, o);
          tmem_ld_wait();
          if (niter == 0) {   // no MMA ran: the accumulators were never written
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
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
  }

  if (warp == 1 && lane == 0) mbar_wait(&bars->mma_final, 0, nullptr, nullptr, p.limit_ns);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dkdv

// ============================================================================
// bwd_dq
// ============================================================================
namespace dq {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int NSK = 3;   // K ring: a K tile is read by S and, one step later, by dQ
constexpr int NSV = 2;   // V ring: read by dP only
#ifndef DQ_NWG
#define DQ_NWG 2
#endif
constexpr int kNWG = DQ_NWG;           // softmax warpgroups, each taking kCW key columns of a tile
constexpr int kCW = BN / kNWG;
constexpr int kThreads = 128 + 128 * kNWG;
static_assert(kNWG == 2 || kNWG == 4, "two or four softmax warpgroups");
// exponentials of the first kMufuPairs column pairs on MUFU, the rest on the
// FMA pipe (exp2_poly)
#ifndef DQ_MUFU_PAIRS
#define DQ_MUFU_PAIRS 32
#endif
constexpr int kMufuPairs = DQ_MUFU_PAIRS < kCW / 2 ? DQ_MUFU_PAIRS : kCW / 2;
// with four softmax warpgroups (640 threads, 96 registers each at launch) the
// first warpgroup hands registers to the softmax warpgroups
constexpr int kRegsLo = 56, kRegsHi = 104;
static_assert(kNWG == 2 || 128 * kRegsLo + 512 * kRegsHi <= 640 * 96, "register split over budget");

struct Params {
  const int32_t* segstart;
  const float* stats;    // see stats_index
  const int32_t* shifts; // q, k, v, dO scale shifts (launch_f16_copies)
  void* dq;              // [P*b][q_rows][hq][D]
  int* status;
  int64_t n, n_pad;      // tokens of the whole sequence; the statistics table's rows (q_rows rounded up)
  int64_t q_base, q_rows, k_base, k_rows;   // global rows held by the Q-side and K-side buffers
  int64_t k_lo, k_hi;    // only keys in [k_lo, k_hi) take part (one ring block); 0, n otherwise
  int32_t b, P_sel, rank0, hq, G, ntiles;
  float scale, scale_log2;
  int32_t g_f32;
  uint64_t limit_ns;
  int64_t g_elems, stats_elems, ss_elems;   // dQ, statistics and segment-table extents (debug build checks)
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = BM * D * 2;
  static constexpr uint32_t oQ = 0;
  static constexpr uint32_t oDO = oQ + kTile;
  static constexpr uint32_t oK = oDO + kTile;
  static constexpr uint32_t oV = oK + NSK * kTile;
  static constexpr uint32_t oBar = oV + NSV * kTile;
  static constexpr uint32_t kDynamic = oBar + 256 + 1024;
  static_assert(kDynamic <= 227 * 1024, "dynamic shared memory above the per-CTA limit");
};

struct Bars {
  uint64_t qdo_full;
  uint64_t k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV];
  uint64_t s_full[2], ds_ready[2];
  uint64_t dp_full, dp_free, mma_final;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
       const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mdo, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::oBar);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // (rank, batch row, kv head) groups one after another (resident CTAs share
  // one kv head's K / V in L2); inside a group: heaviest tile first, the G
  // query heads of a tile next to each other
  const int per_group = p.ntiles * p.G;
  const int w = int(blockIdx.x % per_group);
  int rem = int(blockIdx.x / per_group);
  const int tile = p.ntiles - 1 - w / p.G;
  const int hkv = p.hq / p.G;
  const int g = rem % hkv;
  const int h = g * p.G + w % p.G;
  rem /= hkv;
  const int bb = rem % p.b;
  const int r = p.rank0 + rem / p.b;
  const int rb = r * p.b + bb;
  const int64_t t0 = p.q_base + int64_t(tile) * BM;   // global rows [t0, t0 + BM)
  const int64_t q_blk_end = p.q_base + p.q_rows;
  const int64_t last_row = (t0 + BM - 1 < q_blk_end - 1) ? (t0 + BM - 1) : (q_blk_end - 1);
  const int32_t* ss = p.segstart + int64_t(bb) * p.n;
  const int64_t seg_lo = ss[t0];
  const int64_t seg_hi = ss[last_row];
  // key tiles: the tile's visible keys, clipped to [k_lo, k_hi); none -> dQ = 0
  const int64_t key_lo = seg_lo > p.k_lo ? seg_lo : p.k_lo;
  const int64_t key_hi = last_row < p.k_hi - 1 ? last_row : p.k_hi - 1;   // inclusive
  const int kv_first = int(key_lo / BN);
  const int nkv = key_hi >= key_lo ? int(key_hi / BN) - kv_first + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qdo_full, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->ds_ready[s], 128 * kNWG);
    }
    mbar_init(&bars->dp_full, 1);
    mbar_init(&bars->dp_free, 128 * kNWG);
    mbar_init(&bars->mma_final, 1);
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
  auto tS = [&](int b) { return tmem + 128u * uint32_t(b); };
  const uint32_t tDP = tmem + 256, tDQ = tmem + 384;

  if (warp == 0 || warp == 2) {
    if constexpr (kNWG > 2) regs_split_n<kRegsLo, kRegsHi, kThreads, 96>(false);
    // producers: warp 0 loads Q, dO and the K ring, warp 2 the V ring, so a
    // K load never waits behind a V stage that is still being read
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &mk : &mv;
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const uint32_t base = is_k ? L::oK : L::oV;
      const int ns = is_k ? NSK : NSV;
      tma_prefetch_desc(map);
      if (is_k) {
        mbar_arrive_expect_tx(&bars->qdo_full, 2 * L::kTile);
        for (int dc = 0; dc < D / 64; ++dc) {
          if (in_bounds(t0 - p.q_base >= 0 && t0 - p.q_base < p.q_rows, p.status)) {
            tma_load_4d(&mq, &bars->qdo_full, smem + L::oQ + dc * BM * 128, dc * 64, h, int(t0 - p.q_base), rb);
            tma_load_4d(&mdo, &bars->qdo_full, smem + L::oDO + dc * BM * 128, dc * 64, h, int(t0 - p.q_base), rb);
          }
        }
      }
      int issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int st = it % ns, rnd = it / ns;
        const int k0 = (kv_first + it) * BN;
        if (rnd > 0 && !mbar_wait(&empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        mbar_arrive_expect_tx(&full[st], L::kTile);
        if (in_bounds(k0 - p.k_base >= 0 && k0 - p.k_base < p.k_rows, p.status))
          for (int dc = 0; dc < D / 64; ++dc)
            tma_load_4d(map, &full[st], smem + base + st * L::kTile + dc * BN * 128, dc * 64, g, int(k0 - p.k_base),
                        rb);
        issued = it + 1;
      }
      if (*abort_flag) {
        if (is_k) mbar_wait(&bars->qdo_full, 0, nullptr, nullptr, p.limit_ns);
        for (int x = max(0, issued - ns); x < issued; ++x)
          mbar_wait(&full[x % ns], (x / ns) & 1, nullptr, nullptr, p.limit_ns);
      }
    }
  } else if (warp == 1) {
    if constexpr (kNWG > 2) regs_split_n<kRegsLo, kRegsHi, kThreads, 96>(false);
    {   // whole warp; the elected lane issues
      const uint32_t id_s = idesc_f16(BM, BN, false, false);
      const uint32_t id_q = idesc_f16(BM, D, false, true);
      const uint32_t q_addr = smem_u32(smem + L::oQ), do_addr = smem_u32(smem + L::oDO);
      bool ok = mbar_wait_warp(&bars->qdo_full, 0, abort_flag, p.status, p.limit_ns);
      tc_fence_after();
      auto issue_dq = [&](int jt) -> bool {
        const int b = jt & 1, st = jt % NSK;
        if (!mbar_wait_warp(&bars->ds_ready[b], (jt >> 1) & 1, abort_flag, p.status, p.limit_ns)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + L::oK + st * L::kTile);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // dS of keys [16kk, 16kk+16): warpgroup w's kCW keys sit, as fp16
          // pairs, in the first kCW/2 of its own kCW S columns
          const uint32_t a_col = kCW * ((16 * kk) / kCW) + 8 * (kk % (kCW / 16));
          umma_ts_warp(tDQ, tS(b) + a_col, sdesc_sw128(k_addr + kk * 2048, BN * 128, 1024), id_q,
                  (jt > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit_warp(&bars->k_empty[st]);
        return true;
      };
      for (int it = 0; ok && it < nkv; ++it) {
        const int sk = it % NSK, sv = it % NSV, b = it & 1;
        if (!mbar_wait_warp(&bars->k_full[sk], (it / NSK) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + L::oK + sk * L::kTile);
        const uint32_t v_addr = smem_u32(smem + L::oV + sv * L::kTile);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_ss_warp(tS(b), sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), id_s, kk > 0);
        }
        umma_commit_warp(&bars->s_full[b]);
        if (it >= 1 && !mbar_wait_warp(&bars->dp_free, (it - 1) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        if (!mbar_wait_warp(&bars->v_full[sv], (it / NSV) & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
          umma_ss_warp(tDP, sdesc_sw128(do_addr + off, 16, 1024), sdesc_sw128(v_addr + off, 16, 1024), id_s, kk > 0);
        }
        umma_commit_warp(&bars->dp_full);
        umma_commit_warp(&bars->v_empty[sv]);
        if (it >= 1 && !issue_dq(it - 1)) { ok = false; break; }
      }
      if (ok && nkv > 0) issue_dq(nkv - 1);
      umma_commit_warp(&bars->mma_final);
    }
  } else if (warp == 3) {
    if constexpr (kNWG > 2) regs_split_n<kRegsLo, kRegsHi, kThreads, 96>(false);
  } else if (warp >= 4) {
    if constexpr (kNWG > 2) regs_split_n<kRegsLo, kRegsHi, kThreads, 96>(true);
    const int wg = (warp - 4) >> 2;                 // key columns [kCW wg, kCW wg + kCW) of every tile
    const int row = ((warp - 4) & 3) * 32 + lane;
    const uint32_t lane_off = uint32_t(((warp - 4) & 3) * 32) << 16;
    const int64_t i = t0 + row;                  // global row
    const bool valid = i < q_blk_end;
    const int64_t s_i = valid && in_bounds(int64_t(bb) * p.n + i < p.ss_elems, p.status) ? ss[i] : seg_hi;
    // this row's keys: [row_lo, row_hi) = its sample's keys up to i, inside [k_lo, k_hi)
    const int64_t row_lo = s_i > p.k_lo ? s_i : p.k_lo;
    const int64_t row_hi = i + 1 < p.k_hi ? i + 1 : p.k_hi;
    float nl = 0.f, nd = 0.f;   // -LSE*log2e, -D of this row
    if (valid) {
      const int64_t si = stats_index(int64_t(rb) * p.hq + h, p.n_pad, i - p.q_base);
      if (in_bounds(si >= 0 && si + 64 < p.stats_elems, p.status)) {
        nl = p.stats[si];
        nd = p.stats[si + 64];
      }
    }
    const float sl = p.scale_log2 * pow2i(p.shifts[kShQ]) * pow2i(p.shifts[kShK]);   // q'.k' units, as dK/dV
    const uint64_t sl2 = f2_pack(sl, sl), nl2 = f2_pack(nl, nl), nd2 = f2_pack(nd, nd);
    bool ok = true;
    for (int it = 0; it < nkv; ++it) {
      const int b = it & 1;
      const int64_t k0 = int64_t(kv_first + it) * BN + kCW * wg;   // first key column of this warpgroup
      if (!mbar_wait(&bars->s_full[b], (it >> 1) & 1, abort_flag, p.status, p.limit_ns) ||
          !mbar_wait(&bars->dp_full, it & 1, abort_flag, p.status, p.limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      constexpr int NC = kCW / 32;   // 32-column chunks of this warpgroup
      uint32_t sv[NC][32], dv_[NC][32];
#pragma unroll
      for (int ch = 0; ch < NC; ++ch) {
        tmem_ld32(tS(b) + lane_off + kCW * wg + 32 * ch, sv[ch]);
        tmem_ld32(tDP + lane_off + kCW * wg + 32 * ch, dv_[ch]);
      }
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->dp_free);
      // visible key columns c of this warpgroup: lo <= c < hi (keys row_lo .. row_hi - 1)
      const int64_t lo64 = row_lo - k0, hi64 = valid ? row_hi - k0 : lo64;
      const bool need_mask = lo64 > 0 || hi64 < kCW;
      const int lo = int(lo64 < 0 ? 0 : (lo64 > kCW ? kCW : lo64));
      const int hi = int(hi64 < lo ? lo : (hi64 > kCW ? kCW : hi64));
      uint32_t w[kCW / 2];
#pragma unroll
      for (int c = 0; c < kCW / 2; ++c) {
        const uint32_t sa = sv[(2 * c) / 32][(2 * c) % 32], sb = sv[(2 * c) / 32][(2 * c + 1) % 32];
        const uint32_t da = dv_[(2 * c) / 32][(2 * c) % 32], db = dv_[(2 * c) / 32][(2 * c + 1) % 32];
        float xa, xb;
        f2_unpack(f2_fma(f2_pack(__uint_as_float(sa), __uint_as_float(sb)), sl2, nl2), xa, xb);
#ifdef BWD_EX2_F16X2
        float pa, pb;
        unpack_f16x2(ex2_f16x2(pack_f16x2(xa, xb)), pa, pb);   // one MUFU operation, fp16 precision
#else
        float pa, pb;
        if (c < kMufuPairs) {
          pa = ex2_approx(xa);
          pb = ex2_approx(xb);
        } else {
          f2_unpack(exp2_poly2(f2_pack(xa, xb)), pa, pb);
        }
#endif
        if (need_mask) {
          if (unsigned(2 * c - lo) >= unsigned(hi - lo)) pa = 0.f;
          if (unsigned(2 * c + 1 - lo) >= unsigned(hi - lo)) pb = 0.f;
        }
        float ga, gb;
        f2_unpack(f2_mul(f2_pack(pa, pb), f2_add(f2_pack(__uint_as_float(da), __uint_as_float(db)), nd2)), ga, gb);
        w[c] = pack_f16x2(ga, gb);
      }
      if constexpr (kCW == 64) {
        tmem_st32(tS(b) + lane_off + kCW * wg, w);
      } else {
        tmem_st16(tS(b) + lane_off + kCW * wg, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->ds_ready[b]);
    }
    if (mbar_wait(&bars->mma_final, 0, abort_flag, p.status, p.limit_ns) && ok && !*abort_flag) {
      tc_fence_after();
      const int64_t orow = (int64_t(rb) * p.q_rows + (i - p.q_base)) * p.hq + h;
      const bool store = valid && in_bounds(orow >= 0 && (orow + 1) * D <= p.g_elems, p.status);
      // dQ' = dS' k' = scale^-1 dQ 2^-(sdo+sv+sk)
      const float mq = p.scale * pow2i(p.shifts[kShDO]) * pow2i(p.shifts[kShV]) * pow2i(p.shifts[kShK]);
      for (int c = kCW * wg; c < D; c += 128) {
        // warpgroup wg stores head-dim columns [kCW wg, kCW wg + kCW) (and the
        // same 128 further on); a warpgroup past D stores nothing
#pragma unroll
        for (int c2 = 0; c2 < kCW; c2 += 32) {
          uint32_t o[32];
          tmem_ld32(tDQ + lane_off + c + c2, o);
          tmem_ld_wait();
          if (nkv == 0) {   // no MMA ran: the accumulator was never written
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          if (store) {
            if (p.g_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.dq) + orow * D + c + c2);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(o[4 * e]) * mq, __uint_as_float(o[4 * e + 1]) * mq,
                                     __uint_as_float(o[4 * e + 2]) * mq, __uint_as_float(o[4 * e + 3]) * mq);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.dq) + orow * D + c + c2);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = make_uint4(
                    pack_bf16x2(__uint_as_float(o[8 * e]) * mq, __uint_as_float(o[8 * e + 1]) * mq),
                    pack_bf16x2(__uint_as_float(o[8 * e + 2]) * mq, __uint_as_float(o[8 * e + 3]) * mq),
                    pack_bf16x2(__uint_as_float(o[8 * e + 4]) * mq, __uint_as_float(o[8 * e + 5]) * mq),
                    pack_bf16x2(__uint_as_float(o[8 * e + 6]) * mq, __uint_as_float(o[8 * e + 7]) * mq));
            }
          }
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

}  // namespace dq

}  // namespace bwd

// Backward workspace:
//   [0, 256)      status word (bytes 0-3); the four largest magnitudes as
//                 bf16 bits (uint32, bytes 64-79) and the four shifts
//                 (int32, bytes 96-111) of q, k, v, dO
//   the segment tables (as the forward)
//   the padded row-statistics table (see stats_index; n_pad = n rounded up to 128)
//   the fp16 copies q', k', v', dO' (head layout, 256-byte aligned each)
static int64_t bwd_n_pad(int64_t n) { return (n + 127) / 128 * 128; }
static size_t bwd_ws_stats_off(const uly_shape* s) { return seg_workspace_bytes(s->b, s->n); }
static size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
static size_t bwd_ws_copies_off(const uly_shape* s) {
  return bwd_ws_stats_off(s) + round256(size_t(s->b) * size_t(s->h_q) * size_t(bwd_n_pad(s->n)) * 8);
}
// bytes of one fp16 copy of a head-layout tensor with h heads per rank
static size_t bwd_copy_bytes(const uly_shape* s, int64_t h) {
  return round256(size_t(s->P) * size_t(s->b) * size_t(s->n) * size_t(h) * size_t(s->d) * 2);
}

}  // namespace uly

using namespace uly;

extern "C" size_t ulysses_attn_bwd_workspace(const uly_shape* s, uly_dtype g_dtype) {
  if (check_shape(s) != ULY_OK || !dtype_ok(g_dtype)) return 0;
  const int64_t hq = s->h_q / s->P, hkv = kv_heads_per_rank(*s);
  return bwd_ws_copies_off(s) + 2 * bwd_copy_bytes(s, hq) + 2 * bwd_copy_bytes(s, hkv);
}

// events: null, or five caller-owned cudaEvent_t recorded on the stream
// before the segment-table kernel, before the preparation kernels (largest
// magnitudes, fp16 copies, row statistics), before dK/dV, before dQ and
// after dQ.
// k_lo, k_hi: the key range taking part ([0, n) for the plain backward).
// rows: the global rows the Q-side buffers (q, O, LSE, dO, dQ) and the K-side
// buffers (k, v, dK, dV) hold.
static uly_status attn_bwd_impl(const void* q_head, const void* k_head, const void* v_head, const void* o_head,
                                uly_dtype o_dtype, const float* lse, const void* do_head, const int64_t* position_ids,
                                const uly_shape* shape, int32_t rank, float softmax_scale, int64_t k_lo,
                                int64_t k_hi, const RowBlocks& rows, void* dq_head, void* dk_head, void* dv_head,
                                uly_dtype g_dtype, void* ws, size_t ws_bytes, void* stream, void* const* events) {
  uly_status st = validate_attn(q_head, k_head, v_head, position_ids, shape, rank, ws, ws_bytes,
                                shape ? ulysses_attn_bwd_workspace(shape, g_dtype) : 0);
  if (st != ULY_OK) return st;
  if (!rows_ok(rows, shape->n, 128)) return ULY_ERR_INVALID_ARG;
  if (k_lo < rows.k_base || k_hi <= k_lo || k_hi > rows.k_base + rows.k_rows) return ULY_ERR_INVALID_ARG;
  if (!o_head || !lse || !do_head || !dq_head || !dk_head || !dv_head) return ULY_ERR_INVALID_ARG;
  if (!dtype_ok(o_dtype) || !dtype_ok(g_dtype)) return ULY_ERR_INVALID_ARG;
  if (!aligned(o_head, 16) || !aligned(lse, 16) || !aligned(do_head, 16) || !aligned(dq_head, 16) ||
      !aligned(dk_head, 16) || !aligned(dv_head, 16))
    return ULY_ERR_INVALID_ARG;
  const uly_shape& s = *shape;
  const int64_t hq = s.h_q / s.P, hkv = kv_heads_per_rank(s), Pb = int64_t(s.P) * s.b;
  const size_t gsz = dtype_size(g_dtype);
  const int64_t qr = rows.q_rows, kr = rows.k_rows;
  const size_t dqb = size_t(Pb * qr * hq * s.d) * gsz, dkb = size_t(Pb * kr * hkv * s.d) * gsz;
  const size_t qb = size_t(Pb * qr * hq * s.d) * 2, kb = size_t(Pb * kr * hkv * s.d) * 2;
  const size_t ob = size_t(Pb * qr * hq * s.d) * dtype_size(o_dtype), lb = size_t(Pb * hq * qr) * 4;
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
  for (int b2 = 0; b2 < 6; ++b2)   // the workspace receives the fp16 copies of the inputs
    if (overlaps(ins[b2], insz[b2], ws, ws_bytes)) return ULY_ERR_INVALID_ARG;

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint32_t* amax = reinterpret_cast<uint32_t*>(wsb + 64);
  int32_t* shifts = reinterpret_cast<int32_t*>(wsb + 96);
  uint16_t* q16 = reinterpret_cast<uint16_t*>(wsb + bwd_ws_copies_off(&s));
  uint16_t* do16 = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(q16) + bwd_copy_bytes(&s, hq));
  uint16_t* k16 = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(do16) + bwd_copy_bytes(&s, hq));
  uint16_t* v16 = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(k16) + bwd_copy_bytes(&s, hkv));

  // the attention kernels read the fp16 copies
  CUtensorMap mk128, mv128, mq128, mdo128;
  if (!make_head_map(&mk128, k16, Pb, kr, hkv, s.d, 128) || !make_head_map(&mv128, v16, Pb, kr, hkv, s.d, 128) ||
      !make_head_map(&mq128, q16, Pb, qr, hq, s.d, 128) || !make_head_map(&mdo128, do16, Pb, qr, hq, s.d, 128))
    return ULY_ERR_CUDA;
  const size_t tab = (size_t(s.b) * size_t(s.n) * 4 + 255) & ~size_t(255);
  int32_t* segstart = reinterpret_cast<int32_t*>(wsb + 256);
  int32_t* segend = reinterpret_cast<int32_t*>(wsb + 256 + tab);
  float* stats = reinterpret_cast<float*>(wsb + bwd_ws_stats_off(&s));
  const int64_t n_pad = bwd_n_pad(qr);   // statistics rows of the Q-side block

  auto mark = [&](int i) { return !events || cudaEventRecord(static_cast<cudaEvent_t>(events[i]), cs) == cudaSuccess; };
  if (!mark(0)) return ULY_ERR_CUDA;
  cudaError_t e = launch_segments(position_ids, segstart, segend, s.b, s.n, cs);
  if (e != cudaSuccess) return ULY_ERR_CUDA;
  if (!mark(1)) return ULY_ERR_CUDA;

  const int64_t P_sel = rank < 0 ? s.P : 1;
  const int64_t rank0 = rank < 0 ? 0 : rank;
  const int64_t rb0 = rank0 * s.b, nrb = P_sel * s.b;
  {
    // fp16 copies of the selected ranks' rows, each scaled by its own power of
    // two: q, k to [2^14, 2^15), v to [4, 8), dO to [8, 16) (dP' - D' in range)
    F16Copies a;
    const void* srcs[4] = {q_head, k_head, v_head, do_head};
    uint16_t* dsts[4] = {q16, k16, v16, do16};
    const int64_t heads[4] = {hq, hkv, hkv, hq};
    const int64_t nrows[4] = {qr, kr, kr, qr};
    const int32_t targets[4] = {14, 14, 2, 3};
    a.count = 4;
    for (int t = 0; t < 4; ++t) {
      a.src[t] = static_cast<const uint16_t*>(srcs[t]);
      a.dst[t] = dsts[t];
      a.off[t] = rb0 * nrows[t] * heads[t] * s.d;
      a.cnt[t] = nrb * nrows[t] * heads[t] * s.d;
      a.target[t] = targets[t];
    }
    if (launch_f16_copies(a, amax, shifts, cs) != cudaSuccess) return ULY_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return ULY_ERR_CUDA;
  }
  const int64_t qelems = Pb * qr * hq * s.d;                       // Q-side buffer elements
  const int64_t stats_elems = int64_t(s.b) * s.h_q * bwd_n_pad(s.n) * 2;   // the workspace's statistics table
  int* st_word = reinterpret_cast<int*>(wsb);
  {
    const int64_t total = nrb * n_pad * hq;
    const int64_t blocks = (total * 32 + 255) / 256;
    if (blocks > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    const bool of32 = o_dtype == ULY_F32;
    const uint16_t* dop = static_cast<const uint16_t*>(do_head);
    const unsigned nb = unsigned(blocks);
    if (s.d == 128) {
      if (of32) bwd::bwd_pre_kernel<128, true><<<nb, 256, 0, cs>>>(o_head, dop, lse, stats, shifts, rb0, qr, n_pad, int32_t(hq), total, qelems, stats_elems, st_word);
      else bwd::bwd_pre_kernel<128, false><<<nb, 256, 0, cs>>>(o_head, dop, lse, stats, shifts, rb0, qr, n_pad, int32_t(hq), total, qelems, stats_elems, st_word);
    } else {
      if (of32) bwd::bwd_pre_kernel<64, true><<<nb, 256, 0, cs>>>(o_head, dop, lse, stats, shifts, rb0, qr, n_pad, int32_t(hq), total, qelems, stats_elems, st_word);
      else bwd::bwd_pre_kernel<64, false><<<nb, 256, 0, cs>>>(o_head, dop, lse, stats, shifts, rb0, qr, n_pad, int32_t(hq), total, qelems, stats_elems, st_word);
    }
    if (cudaGetLastError() != cudaSuccess) return ULY_ERR_CUDA;
  }

  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(float(s.d));
  if (!mark(2)) return ULY_ERR_CUDA;
  // ---- dK, dV
  {
    bwd::dkdv::Params p;
    p.segend = segend;
    p.stats = stats;
    p.shifts = shifts;
    p.dk = dk_head;
    p.dv = dv_head;
    p.status = reinterpret_cast<int*>(wsb);
    p.n = s.n;
    p.n_pad = n_pad;
    p.q_base = rows.q_base;
    p.q_rows = qr;
    p.k_base = rows.k_base;
    p.k_rows = kr;
    p.k_lo = k_lo;
    p.k_hi = k_hi;
    p.b = int32_t(s.b);
    p.P_sel = int32_t(P_sel);
    p.rank0 = int32_t(rank0);
    p.hq = int32_t(hq);
    p.hkv = int32_t(hkv);
    p.G = int32_t(group_per_rank(s));
    p.scale = scale;
    p.scale_log2 = scale * bwd::kLog2e;
    p.g_f32 = g_dtype == ULY_F32;
    p.limit_ns = 2000000000ull;
    p.g_elems = Pb * kr * hkv * s.d;
    p.stats_elems = stats_elems;
    p.se_elems = s.b * s.n;
    const int64_t grid = (kr + bwd::dkdv::BKV - 1) / bwd::dkdv::BKV * P_sel * s.b * hkv;
    if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    if (s.d == 128) {
      auto kern = bwd::dkdv::attn_bwd_dkdv_kernel<128>;
      const uint32_t sm = bwd::dkdv::Layout<128>::kDynamic;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess) return ULY_ERR_CUDA;
      kern<<<unsigned(grid), bwd::dkdv::kThreads, sm, cs>>>(mq128, mk128, mv128, mdo128, p);
    } else {
      auto kern = bwd::dkdv::attn_bwd_dkdv_kernel<64>;
      const uint32_t sm = bwd::dkdv::Layout<64>::kDynamic;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess) return ULY_ERR_CUDA;
      kern<<<unsigned(grid), bwd::dkdv::kThreads, sm, cs>>>(mq128, mk128, mv128, mdo128, p);
    }
    if (cudaGetLastError() != cudaSuccess) return ULY_ERR_CUDA;
  }
  if (!mark(3)) return ULY_ERR_CUDA;
  // ---- dQ
  {
    bwd::dq::Params p;
    p.segstart = segstart;
    p.stats = stats;
    p.shifts = shifts;
    p.dq = dq_head;
    p.status = reinterpret_cast<int*>(wsb);
    p.n = s.n;
    p.n_pad = n_pad;
    p.q_base = rows.q_base;
    p.q_rows = qr;
    p.k_base = rows.k_base;
    p.k_rows = kr;
    p.k_lo = k_lo;
    p.k_hi = k_hi;
    p.b = int32_t(s.b);
    p.P_sel = int32_t(P_sel);
    p.rank0 = int32_t(rank0);
    p.hq = int32_t(hq);
    p.G = int32_t(group_per_rank(s));
    p.ntiles = int32_t((qr + bwd::dq::BM - 1) / bwd::dq::BM);
    p.scale = scale;
    p.scale_log2 = scale * bwd::kLog2e;
    p.g_f32 = g_dtype == ULY_F32;
    p.limit_ns = 2000000000ull;
    p.g_elems = qelems;
    p.stats_elems = stats_elems;
    p.ss_elems = s.b * s.n;
    const int64_t grid = int64_t(p.ntiles) * P_sel * s.b * hq;
    if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
    if (s.d == 128) {
      auto kern = bwd::dq::attn_bwd_dq_kernel<128>;
      const uint32_t sm = bwd::dq::Layout<128>::kDynamic;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess) return ULY_ERR_CUDA;
      kern<<<unsigned(grid), bwd::dq::kThreads, sm, cs>>>(mq128, mk128, mv128, mdo128, p);
    } else {
      auto kern = bwd::dq::attn_bwd_dq_kernel<64>;
      const uint32_t sm = bwd::dq::Layout<64>::kDynamic;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, sm) != cudaSuccess) return ULY_ERR_CUDA;
      kern<<<unsigned(grid), bwd::dq::kThreads, sm, cs>>>(mq128, mk128, mv128, mdo128, p);
    }
    if (cudaGetLastError() != cudaSuccess) return ULY_ERR_CUDA;
  }
  if (!mark(4)) return ULY_ERR_CUDA;
  return ULY_OK;
}

extern "C" uly_status ulysses_attn_bwd(const void* q_head, const void* k_head, const void* v_head, const void* o_head,
                                       uly_dtype o_dtype, const float* lse, const void* do_head,
                                       const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                       float softmax_scale, void* dq_head, void* dk_head, void* dv_head,
                                       uly_dtype g_dtype, void* ws, size_t ws_bytes, void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  return attn_bwd_impl(q_head, k_head, v_head, o_head, o_dtype, lse, do_head, position_ids, shape, rank,
                       softmax_scale, 0, shape->n, whole_rows(shape->n), dq_head, dk_head, dv_head, g_dtype, ws,
                       ws_bytes, stream, nullptr);
}

extern "C" uly_status ulysses_attn_bwd_kv_range(const void* q_head, const void* k_head, const void* v_head,
                                                const void* o_head, uly_dtype o_dtype, const float* lse,
                                                const void* do_head, const int64_t* position_ids,
                                                const uly_shape* shape, int32_t rank, float softmax_scale,
                                                int64_t k_lo, int64_t k_hi, void* dq_head, void* dk_head,
                                                void* dv_head, uly_dtype g_dtype, void* ws, size_t ws_bytes,
                                                void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  return attn_bwd_impl(q_head, k_head, v_head, o_head, o_dtype, lse, do_head, position_ids, shape, rank,
                       softmax_scale, k_lo, k_hi, whole_rows(shape->n), dq_head, dk_head, dv_head, g_dtype, ws,
                       ws_bytes, stream, nullptr);
}

extern "C" uly_status ulysses_attn_bwd_block(const void* q_blk, const void* k_blk, const void* v_blk,
                                             const void* o_blk, uly_dtype o_dtype, const float* lse_blk,
                                             const void* do_blk, const int64_t* position_ids, const uly_shape* shape,
                                             int64_t q_base, int64_t q_rows, int64_t k_base, int64_t k_rows,
                                             float softmax_scale, void* dq_blk, void* dk_blk, void* dv_blk,
                                             uly_dtype g_dtype, void* ws, size_t ws_bytes, void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  const RowBlocks rows{q_base, q_rows, k_base, k_rows};
  if (!rows_ok(rows, shape->n, 128)) return ULY_ERR_INVALID_ARG;
  return attn_bwd_impl(q_blk, k_blk, v_blk, o_blk, o_dtype, lse_blk, do_blk, position_ids, shape, -1, softmax_scale,
                       k_base, k_base + k_rows, rows, dq_blk, dk_blk, dv_blk, g_dtype, ws, ws_bytes, stream, nullptr);
}

extern "C" uly_status ulysses_attn_bwd_timed(const void* q_head, const void* k_head, const void* v_head,
                                             const void* o_head, uly_dtype o_dtype, const float* lse,
                                             const void* do_head, const int64_t* position_ids,
                                             const uly_shape* shape, int32_t rank, float softmax_scale,
                                             void* dq_head, void* dk_head, void* dv_head, uly_dtype g_dtype,
                                             void* ws, size_t ws_bytes, void* stream, void* const* events) {
  if (!events) return ULY_ERR_INVALID_ARG;
  for (int i = 0; i < 5; ++i)
    if (!events[i]) return ULY_ERR_INVALID_ARG;
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  return attn_bwd_impl(q_head, k_head, v_head, o_head, o_dtype, lse, do_head, position_ids, shape, rank,
                       softmax_scale, 0, shape->n, whole_rows(shape->n), dq_head, dk_head, dv_head, g_dtype, ws,
                       ws_bytes, stream, events);
}
