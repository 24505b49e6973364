// Local causal attention forward of every virtual rank on its head slice.
//
// Blog "Ulysses Sequence Parallelism: Training with Million-Token Contexts":
// "How Ulysses works", step 4 (each rank runs ordinary attention for its
// heads over the full sequence); causal masking and sample boundaries come
// from position_ids, not a 4D mask (position_ids paragraph).  Accelerate
// guide "Sequence parallelism", "ALST/Ulysses SP backend configuration":
// samples packed into one row must not attend to one another.
//
// Kernel structure: one CTA per (rank, batch row, query head, pair of
// adjacent 128-row query tiles), heaviest pairs first.  Both query tiles
// share every K/V tile the CTA loads, which halves the L2 -> shared-memory
// traffic per flop (every CTA streams its head's whole visible K/V prefix).
//   warp 0       TMA producer: Q tiles once, then K tiles into a 2-stage ring
//   warp 2       TMA producer: V tiles into a 2-stage ring
//   warp 1       TMEM owner; issues the tcgen05 MMAs as a converged warp
//                (elect.sync picks the issuing lane)
//   warps 4..7   softmax of query tile 0, thread = query row
//   warps 8..11  softmax of query tile 1
// Per key tile j the MMAs are issued as PV_0(j-1), S_0(j), PV_1(j-1), S_1(j)
// (S_q = Q_q K^T, PV_q: O_q += P_q V), each pair as one burst after all of
// its waits (a wait in the issuing warp leaves the tensor pipe short of
// work, so waits are batched).  While one warpgroup turns S into P the
// tensor core works on the other tile, and S_q(j) completing implies
// PV_q(j-1) completed, so the lazy O rescale needs no extra wait.  The
// softmax writes P (bf16) back over S; PV reads it as the A operand from TMEM.
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
// The producer/MMA warpgroup hands registers to the two softmax warpgroups
// (setmaxnreg): 72 + 2 x 216 = 3 x 168 registers per thread slot.
// Keys a tile cannot see are never loaded: a tile's key range starts at the
// key tile holding the sample start of its first row and ends at its
// diagonal; per-element masks run only on tiles that straddle the diagonal
// or a sample start.  A key range [k_lo, k_hi) (the whole sequence for
// ulysses_attn_fwd; one ring block for ulysses_attn_fwd_kv_range) clips both;
// rows that see no key of it get O = 0 and LSE = -inf.
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
#ifndef FWD_NSK
#define FWD_NSK 2
#endif
constexpr int NSK = FWD_NSK;   // K stages
#ifndef FWD_NSV
#define FWD_NSV 2
#endif
constexpr int NSV = FWD_NSV;   // V stages
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8
#ifndef FWD_MUFU_PAIRS
#define FWD_MUFU_PAIRS 48
#endif
constexpr int kMufuPairs = FWD_MUFU_PAIRS;  // of the 64 column pairs per row, the rest use exp2_poly
#ifndef FWD_REGS_LO
#define FWD_REGS_LO 72
#define FWD_REGS_HI 216
#endif
constexpr int kRegsLo = FWD_REGS_LO, kRegsHi = FWD_REGS_HI;   // producer/MMA warpgroup, softmax warpgroups

// P as the A operand of PV: fp16 (11 significant bits, V read from its scaled
// fp16 copy) in the workspace forward; bf16 with bf16 V in the no-workspace
// forward, which has no room for a V copy.
template <bool kF16>
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
  return kF16 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

struct Params {
  const int32_t* segstart;   // [b][n]
  float* lse;                // [P][b][hq][q_rows]
  void* o;                   // [P][b][q_rows][hq][D]
  int* status;
  int64_t n;                 // tokens of the whole sequence (the segment tables')
  int64_t q_base, q_rows;    // Q, O, LSE hold the global rows [q_base, q_base + q_rows); 0, n for whole tensors
  int64_t k_base, k_rows;    // K, V hold the global keys [k_base, k_base + k_rows) (k_base a multiple of BN)
  int64_t k_lo, k_hi;        // keys outside [k_lo, k_hi) are not attended (one ring block); 0, n otherwise
  int32_t b, P_sel, rank0, hq, G, ntiles, npairs;
  float scale_log2;
  int32_t o_f32;
  uint64_t limit_ns;
  int64_t o_elems, lse_elems, ss_elems;   // buffer extents, for the debug build's bounds checks
  const int32_t* v_shift;    // fp16 P: V' = V 2^-s, s here (written by the copy kernel); null for bf16 P
};

template <int D>
struct Layout {
  static constexpr uint32_t kTileBytes = BM * D * 2;   // a Q, K or V tile
  static constexpr uint32_t kQ = 0;                     // two query tiles
  static constexpr uint32_t kK = kQ + 2 * kTileBytes;
  static constexpr uint32_t kV = kK + NSK * kTileBytes;
  static constexpr uint32_t kBar = kV + NSV * kTileBytes;
  static constexpr uint32_t kBytes = kBar + 256;
  static constexpr uint32_t kDynamic = kBytes + 1024;  // alignment slack
  static_assert(kDynamic <= 232448, "dynamic shared memory above the per-CTA limit");
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV];
  uint64_t s_full[2], p_full[2];
  uint64_t o_final[2];
  uint32_t tmem_base;
  int abort_flag;
};


// Key-tile range [first, last] of query tile `tile`, and the largest sample
// start among its rows.
struct TileRange {
  int first, last;
  int64_t t0, seg_hi;
  bool valid;
};

// Key tiles are also clipped to [k_lo, k_hi); first > last means the query
// tile sees no key there (0 <= k_lo < k_hi <= n).  `tile` counts query tiles
// from q_base (a multiple of BM); rows end at q_end.
__device__ __forceinline__ TileRange tile_range(const int32_t* ss, int64_t q_base, int64_t q_end, int tile, int ntiles,
                                                int64_t k_lo, int64_t k_hi) {
  TileRange tr;
  tr.valid = tile < ntiles;
  const int tl = tr.valid ? tile : ntiles - 1;
  tr.t0 = q_base + int64_t(tl) * BM;
  const int64_t last_row = (tr.t0 + BM - 1 < q_end - 1) ? (tr.t0 + BM - 1) : (q_end - 1);
  const int64_t key_lo = int64_t(ss[tr.t0]) > k_lo ? int64_t(ss[tr.t0]) : k_lo;
  const int64_t key_hi = last_row < k_hi - 1 ? last_row : k_hi - 1;   // last key, inclusive
  tr.first = int(key_lo / BN);
  tr.last = key_hi >= key_lo ? int(key_hi / BN) : tr.first - 1;
  tr.seg_hi = ss[last_row];
  return tr;
}

template <int D, bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                const __grid_constant__ CUtensorMap mv, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::kBar);
  volatile int* abort_flag = &bars->abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: heaviest (last) pairs of query tiles first
  // (rank, batch row, kv head) groups run one after another, so resident CTAs
  // share one kv head's K / V in L2; inside a group: heaviest pair first,
  // the G query heads of a pair next to each other
  const int per_group = p.npairs * p.G;
  const int w = int(blockIdx.x % per_group);
  int rem = int(blockIdx.x / per_group);
  const int pair = p.npairs - 1 - w / p.G;
  const int hkv = p.hq / p.G;
  const int g = rem % hkv;
  const int j = g * p.G + w % p.G;
  rem /= hkv;
  const int bb = rem % p.b;
  const int r = p.rank0 + rem / p.b;
  const int rb = r * p.b + bb;
  const int32_t* ss = p.segstart + int64_t(bb) * p.n;
  const int64_t q_end = p.q_base + p.q_rows;
  const TileRange tr0 = tile_range(ss, p.q_base, q_end, 2 * pair, p.ntiles, p.k_lo, p.k_hi);
  const TileRange tr1 = tile_range(ss, p.q_base, q_end, 2 * pair + 1, p.ntiles, p.k_lo, p.k_hi);
  const bool has0 = tr0.valid && tr0.last >= tr0.first, has1 = tr1.valid && tr1.last >= tr1.first;
  // key tiles of the pair: tile 1 starts no earlier and ends no earlier than tile 0
  const int j_lo = has0 ? tr0.first : (has1 ? tr1.first : 0);
  const int j_hi = has1 ? tr1.last : (has0 ? tr0.last : -1);
  const int nkv = j_hi - j_lo + 1;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
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
      mbar_init(&bars->p_full[s], 128);
      mbar_init(&bars->o_final[s], 1);
    }
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

  if (warp < 4) {
    regs_split<kRegsLo, kRegsHi>(false);
    if ((warp == 0 || warp == 2) && lane == 0) {
      // ---------------------------------------------------------- producers
      const bool is_k = warp == 0;
      const CUtensorMap* map = is_k ? &mk : &mv;
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const uint32_t base = is_k ? L::kK : L::kV;
      const int ns = is_k ? NSK : NSV;
      tma_prefetch_desc(map);
      if (is_k) {
        tma_prefetch_desc(&mq);
        mbar_arrive_expect_tx(&bars->q_full, (tr1.valid ? 2 : 1) * L::kTileBytes);
        for (int q = 0; q < (tr1.valid ? 2 : 1); ++q) {
          const int64_t qc = (q ? tr1 : tr0).t0 - p.q_base;
          if (in_bounds(qc >= 0 && qc < p.q_rows && rb < p.P_sel * p.b + p.rank0 * p.b, p.status))
            for (int dc = 0; dc < D / 64; ++dc)
              tma_load_4d(&mq, &bars->q_full, smem + L::kQ + q * L::kTileBytes + dc * BM * 128, dc * 64, j, int(qc),
                          rb);
        }
      }
      int issued = 0;
      for (int it = 0; it < nkv; ++it) {
        const int st = it % ns, rnd = it / ns;
        const int k0 = (j_lo + it) * BN;
        if (rnd > 0 && !mbar_wait(&empty[st], (rnd - 1) & 1, abort_flag, p.status, p.limit_ns)) break;
        mbar_arrive_expect_tx(&full[st], L::kTileBytes);
        if (in_bounds(k0 - p.k_base >= 0 && k0 - p.k_base < p.k_rows, p.status))
          for (int dc = 0; dc < D / 64; ++dc)
            tma_load_4d(map, &full[st], smem + base + st * L::kTileBytes + dc * BN * 128, dc * 64, g,
                        int(k0 - p.k_base), rb);
        issued = it + 1;
      }
      // Error path only: let every copy this thread started land before exit.
      if (*abort_flag) {
        if (is_k) mbar_wait(&bars->q_full, 0, nullptr, nullptr, p.limit_ns);
        for (int x = max(0, issued - ns); x < issued; ++x)
          mbar_wait(&full[x % ns], (x / ns) & 1, nullptr, nullptr, p.limit_ns);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer (whole warp, elected lane issues)
      const uint32_t idesc_s = idesc_bf16(BM, BN, false, false);
      const uint32_t idesc_o = kF16 ? idesc_f16(BM, D, false, true) : idesc_bf16(BM, D, false, true);
      bool ok = mbar_wait_warp(&bars->q_full, 0, abort_flag, p.status, p.limit_ns);
      int npv[2] = {0, 0};
      bool fin[2] = {false, false};   // o_final[q] committed
      for (int it = 0; ok && it <= nkv; ++it) {
        const int jj = j_lo + it;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const TileRange& tr = q ? tr1 : tr0;
          const uint32_t tS = tmem + 128u * q, tO = tmem + 256u + 128u * q;
          const bool do_pv = it >= 1 && tr.valid && jj - 1 >= tr.first && jj - 1 <= tr.last;
          const bool do_s = it < nkv && tr.valid && jj >= tr.first && jj <= tr.last;
          // All waits of this step first, then its MMAs in one burst: a wait
          // in the issuing warp leaves the tensor pipe short of work, so the
          // stage waits ride along with tile 0's P wait.
          if (do_pv && !mbar_wait_warp(&bars->p_full[q], npv[q] & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
          if (q == 0) {
            if (it >= 1 && !mbar_wait_warp(&bars->v_full[(it - 1) % NSV], ((it - 1) / NSV) & 1, abort_flag, p.status, p.limit_ns)) {
              ok = false;
              break;
            }
            if (it < nkv && !mbar_wait_warp(&bars->k_full[it % NSK], (it / NSK) & 1, abort_flag, p.status, p.limit_ns)) {
              ok = false;
              break;
            }
          }
          tc_fence_after();
          // PV_q of the previous key tile (its P sits in S_q: must precede S_q(jj))
          // Descriptors: base once, then + compile-time offsets (16-byte units)
          // so the issue loop is a few instructions per MMA.
          if (do_pv) {
            const uint64_t v_desc = sdesc_sw128(smem_u32(smem + L::kV + ((it - 1) % NSV) * L::kTileBytes), BN * 128, 1024);
            umma_ts_warp(tO, tS, v_desc, idesc_o, npv[q] > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < BN / 16; ++kk)
              umma_ts_warp(tO, tS + kk * 8, v_desc + uint64_t(kk * 2048 / 16), idesc_o, 1u);
            ++npv[q];
            if (jj - 1 == tr.last) {   // tile q's last PV: its epilogue overlaps the other tile's last step
              umma_commit_warp(&bars->o_final[q]);
              fin[q] = true;
            }
          }
          if (do_s) {
            const uint64_t q_desc = sdesc_sw128(smem_u32(smem + L::kQ + q * L::kTileBytes), 16, 1024);
            const uint64_t k_desc = sdesc_sw128(smem_u32(smem + L::kK + (it % NSK) * L::kTileBytes), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = uint64_t(((kk >> 2) * (BM * 128) + (kk & 3) * 32) / 16);
              umma_ss_warp(tS, q_desc + off, k_desc + off, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit_warp(&bars->s_full[q]);
          }
        }
        if (!ok) break;
        if (it >= 1) umma_commit_warp(&bars->v_empty[(it - 1) % NSV]);
        if (it < nkv) umma_commit_warp(&bars->k_empty[it % NSK]);
      }
      // tiles without work, and every tile on the error path, are released here
      if (!fin[0]) umma_commit_warp(&bars->o_final[0]);
      if (!fin[1]) umma_commit_warp(&bars->o_final[1]);
    }
  } else {
    regs_split<kRegsLo, kRegsHi>(true);
    // ------------------------------------------------------------ softmax
    const int q = (warp - 4) >> 2;                     // query tile of this warpgroup
    const TileRange tr = q ? tr1 : tr0;
    const uint32_t tS = tmem + 128u * q, tO = tmem + 256u + 128u * q;
    const int row = ((warp - 4) & 3) * 32 + lane;
    const uint32_t lane_off = uint32_t(((warp - 4) & 3) * 32) << 16;
    const int64_t i = tr.t0 + row;                 // global row
    const bool valid = tr.valid && i < q_end;
    const int64_t il = i - p.q_base;               // row in the Q / O / LSE buffers
    const int64_t s_i = valid && in_bounds(int64_t(bb) * p.n + i < p.ss_elems, p.status) ? ss[i] : tr.seg_hi;
    // this row's keys: [row_lo, row_hi) = its sample's keys up to i, inside [k_lo, k_hi)
    const int64_t row_lo = s_i > p.k_lo ? s_i : p.k_lo;
    const int64_t row_hi = i + 1 < p.k_hi ? i + 1 : p.k_hi;
    const bool row_vis = valid && row_hi > row_lo;
    const uint64_t sl2 = f2_pack(p.scale_log2, p.scale_log2);
    float m_used = -INFINITY, l = 0.f;   // running max (log2 units, scaled) and row sum
    bool ok = true;
    const int ntile = tr.valid && tr.last >= tr.first ? tr.last - tr.first + 1 : 0;
    for (int c = 0; c < ntile; ++c) {
      const int64_t k0 = int64_t(tr.first + c) * BN;
      if (!mbar_wait(&bars->s_full[q], c & 1, abort_flag, p.status, p.limit_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t a0[32], a1[32], a2[32], a3[32];
      tmem_ld32(tS + lane_off + 0, a0);
      tmem_ld32(tS + lane_off + 32, a1);
      tmem_ld32(tS + lane_off + 64, a2);
      tmem_ld32(tS + lane_off + 96, a3);
      tmem_ld_wait();
      float x[BN];   // raw scores q.k
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        x[e] = __uint_as_float(a0[e]);
        x[32 + e] = __uint_as_float(a1[e]);
        x[64 + e] = __uint_as_float(a2[e]);
        x[96 + e] = __uint_as_float(a3[e]);
      }
      // visible key columns: lo <= col < hi (keys row_lo .. row_hi - 1)
      const int64_t lo64 = row_lo - k0, hi64 = valid ? row_hi - k0 : lo64;
      if (lo64 > 0 || hi64 < BN) {
        const int lo = int(lo64 < 0 ? 0 : (lo64 > BN ? BN : lo64));
        const int hi = int(hi64 < lo ? lo : (hi64 > BN ? BN : hi64));
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (unsigned(e - lo) >= unsigned(hi - lo)) x[e] = -INFINITY;
      }
      // row max of the raw scores (scale > 0), four independent chains
      float m0 = x[0], m1 = x[1], m2 = x[2], m3 = x[3];
#pragma unroll
      for (int e = 4; e + 8 <= BN; e += 8) {
        m0 = fmax3(m0, x[e], x[e + 1]);
        m1 = fmax3(m1, x[e + 2], x[e + 3]);
        m2 = fmax3(m2, x[e + 4], x[e + 5]);
        m3 = fmax3(m3, x[e + 6], x[e + 7]);
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
      // O_q holds contributions only if an earlier tile had a finite max; all
      // of them are complete (S_q of this tile was issued after them).
      const bool rescale_o = grow && m_used != -INFINITY;
      if (grow) m_used = m_new;
      if (__any_sync(0xffffffffu, rescale_o)) {
        const float f = rescale_o ? factor : 1.f;
#pragma unroll
        for (int e0 = 0; e0 < D; e0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + e0, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(tO + lane_off + e0, o);
        }
      }
      const float ms = (m_used == -INFINITY) ? 0.f : m_used;
      const uint64_t nms2 = f2_pack(-ms, -ms);
      // P = 2^(scale*x - m): column pairs [0, kMufuPairs) on the MUFU unit,
      // the rest on the FMA pipe (exp2_poly), so both pipes share the load.
      uint64_t sum0 = f2_pack(0.f, 0.f), sum1 = sum0, sum2 = sum0, sum3 = sum0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {   // 64 columns at a time: P stored before the next half
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int c2 = 32 * half + c;
          const uint64_t xx = f2_fma(f2_pack(x[2 * c2], x[2 * c2 + 1]), sl2, nms2);
          float e0, e1;
#ifdef FWD_EX2_F16X2
          if (kF16 && c2 < kMufuPairs) {   // one MUFU op for both exponentials, in fp16
            f2_unpack(xx, e0, e1);
            pk[c] = ex2_f16x2(pack_f16x2(e0, e1));
            unpack_f16x2(pk[c], e0, e1);
          } else
#endif
          {
            if (c2 < kMufuPairs) {
              f2_unpack(xx, e0, e1);
              e0 = ex2_approx(e0);
              e1 = ex2_approx(e1);
            } else {
              f2_unpack(exp2_poly2(xx), e0, e1);
            }
            pk[c] = pack_p<kF16>(e0, e1);
          }
          const uint64_t ee = f2_pack(e0, e1);
          if ((c & 3) == 0) sum0 = f2_add(sum0, ee);
          else if ((c & 3) == 1) sum1 = f2_add(sum1, ee);
          else if ((c & 3) == 2) sum2 = f2_add(sum2, ee);
          else sum3 = f2_add(sum3, ee);
        }
        tmem_st32(tS + lane_off + 32 * half, pk);
      }
      float sa, sb;
      f2_unpack(f2_add(f2_add(sum0, sum1), f2_add(sum2, sum3)), sa, sb);
      l += sa + sb;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[q]);
    }
    // ---- epilogue: O / l and LSE
    if (ntile > 0 && mbar_wait(&bars->o_final[q], 0, abort_flag, p.status, p.limit_ns) && ok && !*abort_flag) {
      tc_fence_after();
      // a row that saw no key gets O = 0; the fp16 path folds V's scale 2^s back in
      const float inv_l = row_vis ? (kF16 ? pow2i(*p.v_shift) : 1.f) / l : 0.f;
      const int64_t orow = (int64_t(rb) * p.q_rows + il) * p.hq + j;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + lane_off + c, o);
        tmem_ld_wait();
        if (valid && in_bounds(orow >= 0 && (orow + 1) * D <= p.o_elems, p.status)) {
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
      const int64_t li = (int64_t(rb) * p.hq + j) * p.q_rows + il;
      if (valid && in_bounds(li >= 0 && li < p.lse_elems, p.status))
        p.lse[li] = row_vis ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    } else if (ntile == 0 && valid) {
      // no key of [k_lo, k_hi) is visible to this query tile: O = 0, LSE = -inf
      const int64_t orow = (int64_t(rb) * p.q_rows + il) * p.hq + j;
      const int64_t li = (int64_t(rb) * p.hq + j) * p.q_rows + il;
      if (in_bounds(orow >= 0 && (orow + 1) * D <= p.o_elems && li >= 0 && li < p.lse_elems, p.status)) {
        if (p.o_f32) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow * D);
          for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow * D);
          for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
        }
        p.lse[li] = -INFINITY;
      }
    }
  }

  // ---- teardown: every MMA has completed once both o_final fired (or the waits gave up)
  if (warp == 1 && lane == 0) {
    mbar_wait(&bars->o_final[0], 0, nullptr, nullptr, p.limit_ns);
    mbar_wait(&bars->o_final[1], 0, nullptr, nullptr, p.limit_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool kF16>
cudaError_t launch(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const Params& p,
                   int64_t grid, cudaStream_t s) {
  auto kern = attn_fwd_kernel<D, kF16>;
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

// Forward workspace: the segment tables (seg_workspace_bytes; bytes 64-67 of
// the status block hold V's largest magnitude, 96-99 its shift), then the
// scaled fp16 copy of V in the head layout, 256-byte aligned.
static size_t fwd_v_copy_bytes(const uly_shape* s) {
  return (size_t(s->P) * size_t(s->b) * size_t(s->n) * size_t(kv_heads_per_rank(*s)) * size_t(s->d) * 2 + 255) &
         ~size_t(255);
}

extern "C" size_t ulysses_attn_fwd_workspace(const uly_shape* s) {
  if (check_shape(s) != ULY_OK) return 0;
  return seg_workspace_bytes(s->b, s->n) + fwd_v_copy_bytes(s);
}

// k_lo, k_hi: the key range attended ([0, n) for the plain forward).  rows:
// the global rows the Q / O / LSE buffers and the K / V buffers hold (the
// whole sequence for the head-layout calls, one block for the block calls).
// f16_p: P and V enter the PV product as fp16 (V from a scaled fp16 copy in
// the workspace); otherwise as bf16 (the no-workspace forward).
static uly_status attn_fwd_impl(const void* q_head, const void* k_head, const void* v_head,
                                const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                float softmax_scale, int64_t k_lo, int64_t k_hi, const RowBlocks& rows,
                                void* o_head, uly_dtype o_dtype, float* lse, void* ws, size_t ws_bytes, void* stream,
                                bool f16_p = true) {
  const size_t need = shape == nullptr || check_shape(shape) != ULY_OK ? 0
                      : f16_p ? ulysses_attn_fwd_workspace(shape) : seg_workspace_bytes(shape->b, shape->n);
  uly_status st = validate_attn(q_head, k_head, v_head, position_ids, shape, rank, ws, ws_bytes, need);
  if (st != ULY_OK) return st;
  if (!rows_ok(rows, shape->n, fwd::BM)) return ULY_ERR_INVALID_ARG;
  if (k_lo < rows.k_base || k_hi <= k_lo || k_hi > rows.k_base + rows.k_rows) return ULY_ERR_INVALID_ARG;
  if (!o_head || !lse || !dtype_ok(o_dtype)) return ULY_ERR_INVALID_ARG;
  if (!aligned(o_head, 16) || !aligned(lse, 16)) return ULY_ERR_INVALID_ARG;
  const uly_shape& s = *shape;
  const int64_t hq = s.h_q / s.P, hkv = kv_heads_per_rank(s), Pb = int64_t(s.P) * s.b;
  const int64_t ntiles = (rows.q_rows + fwd::BM - 1) / fwd::BM;
  const int64_t npairs = (ntiles + 1) / 2;
  const int64_t P_sel = rank < 0 ? s.P : 1;
  const int64_t grid = npairs * P_sel * s.b * hq;
  if (grid > 0x7FFFFFFF) return ULY_ERR_UNSUPPORTED;
  // Outputs must not overlap inputs.
  const size_t qbytes = size_t(Pb * rows.q_rows * hq * s.d) * 2, kvbytes = size_t(Pb * rows.k_rows * hkv * s.d) * 2;
  const size_t obytes = size_t(Pb * rows.q_rows * hq * s.d) * dtype_size(o_dtype);
  const size_t lbytes = size_t(Pb * hq * rows.q_rows) * 4;
  if (overlaps(o_head, obytes, q_head, qbytes) || overlaps(o_head, obytes, k_head, kvbytes) ||
      overlaps(o_head, obytes, v_head, kvbytes) || overlaps(o_head, obytes, lse, lbytes) ||
      overlaps(lse, lbytes, q_head, qbytes) || overlaps(lse, lbytes, ws, ws_bytes) ||
      overlaps(o_head, obytes, ws, ws_bytes))
    return ULY_ERR_INVALID_ARG;

  if (overlaps(ws, ws_bytes, q_head, qbytes) || overlaps(ws, ws_bytes, k_head, kvbytes) ||
      overlaps(ws, ws_bytes, v_head, kvbytes))
    return ULY_ERR_INVALID_ARG;   // the workspace receives a copy of V

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* v16 = reinterpret_cast<uint16_t*>(wsb + seg_workspace_bytes(s.b, s.n));
  int32_t* v_shift = reinterpret_cast<int32_t*>(wsb + 96);
  CUtensorMap mq, mk, mv;
  if (!make_head_map(&mq, q_head, Pb, rows.q_rows, hq, s.d, fwd::BM) ||
      !make_head_map(&mk, k_head, Pb, rows.k_rows, hkv, s.d, fwd::BN) ||
      !make_head_map(&mv, f16_p ? static_cast<const void*>(v16) : v_head, Pb, rows.k_rows, hkv, s.d, fwd::BN))
    return ULY_ERR_CUDA;
  int32_t* segstart = reinterpret_cast<int32_t*>(wsb + 256);
  int32_t* segend = reinterpret_cast<int32_t*>(wsb + 256 + ((size_t(s.b) * size_t(s.n) * 4 + 255) & ~size_t(255)));
  cudaError_t e = launch_segments(position_ids, segstart, segend, s.b, s.n, cs);
  if (e != cudaSuccess) return ULY_ERR_CUDA;
  if (f16_p) {   // V' = V 2^-s in fp16, the selected ranks' rows, largest magnitude in [2^14, 2^15)
    F16Copies a{};
    const int64_t rb0 = int64_t(rank < 0 ? 0 : rank) * s.b, nrb = int64_t(rank < 0 ? s.P : 1) * s.b;
    a.src[0] = static_cast<const uint16_t*>(v_head);
    a.dst[0] = v16;
    a.off[0] = rb0 * rows.k_rows * hkv * s.d;
    a.cnt[0] = nrb * rows.k_rows * hkv * s.d;
    a.target[0] = 14;
    a.count = 1;
    if (launch_f16_copies(a, reinterpret_cast<uint32_t*>(wsb + 64), v_shift, cs) != cudaSuccess) return ULY_ERR_CUDA;
  }

  fwd::Params p;
  p.segstart = segstart;
  p.lse = lse;
  p.o = o_head;
  p.status = reinterpret_cast<int*>(wsb);
  p.n = s.n;
  p.q_base = rows.q_base;
  p.q_rows = rows.q_rows;
  p.k_base = rows.k_base;
  p.k_rows = rows.k_rows;
  p.k_lo = k_lo;
  p.k_hi = k_hi;
  p.b = int32_t(s.b);
  p.P_sel = int32_t(P_sel);
  p.rank0 = rank < 0 ? 0 : rank;
  p.hq = int32_t(hq);
  p.G = int32_t(group_per_rank(s));
  p.ntiles = int32_t(ntiles);
  p.npairs = int32_t(npairs);
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / sqrtf(float(s.d));
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_f32 = o_dtype == ULY_F32;
  p.limit_ns = 2000000000ull;
  p.v_shift = f16_p ? v_shift : nullptr;
  p.o_elems = Pb * rows.q_rows * hq * s.d;
  p.lse_elems = Pb * hq * rows.q_rows;
  p.ss_elems = s.b * s.n;
  if (f16_p)
    e = s.d == 128 ? fwd::launch<128, true>(mq, mk, mv, p, grid, cs) : fwd::launch<64, true>(mq, mk, mv, p, grid, cs);
  else
    e = s.d == 128 ? fwd::launch<128, false>(mq, mk, mv, p, grid, cs) : fwd::launch<64, false>(mq, mk, mv, p, grid, cs);
  return cuda_status(e);
}

extern "C" uly_status ulysses_attn_fwd(const void* q_head, const void* k_head, const void* v_head,
                                       const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                       float softmax_scale, void* o_head, uly_dtype o_dtype, float* lse, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  return attn_fwd_impl(q_head, k_head, v_head, position_ids, shape, rank, softmax_scale, 0, shape->n,
                       whole_rows(shape->n), o_head, o_dtype, lse, ws, ws_bytes, stream);
}

extern "C" uly_status ulysses_attn_fwd_kv_range(const void* q_head, const void* k_head, const void* v_head,
                                                const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                                float softmax_scale, int64_t k_lo, int64_t k_hi, void* o_head,
                                                uly_dtype o_dtype, float* lse, void* ws, size_t ws_bytes,
                                                void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  return attn_fwd_impl(q_head, k_head, v_head, position_ids, shape, rank, softmax_scale, k_lo, k_hi,
                       whole_rows(shape->n), o_head, o_dtype, lse, ws, ws_bytes, stream);
}

extern "C" uly_status ulysses_attn_fwd_block(const void* q_blk, const void* k_blk, const void* v_blk,
                                             const int64_t* position_ids, const uly_shape* shape, int64_t q_base,
                                             int64_t q_rows, int64_t k_base, int64_t k_rows, float softmax_scale,
                                             void* o_blk, uly_dtype o_dtype, float* lse_blk, void* ws,
                                             size_t ws_bytes, void* stream) {
  if (check_shape(shape) != ULY_OK) return check_shape(shape);
  const RowBlocks rows{q_base, q_rows, k_base, k_rows};
  if (!rows_ok(rows, shape->n, fwd::BM)) return ULY_ERR_INVALID_ARG;
  return attn_fwd_impl(q_blk, k_blk, v_blk, position_ids, shape, -1, softmax_scale, k_base, k_base + k_rows, rows,
                       o_blk, o_dtype, lse_blk, ws, ws_bytes, stream);
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
  if (seg_workspace_bytes(shape->b, shape->n) > kNoAllocScratchBytes) return ULY_ERR_WORKSPACE;
  void* scratch = nullptr;
  const uly_status st = scratch_on_current_device(&scratch);
  if (st != ULY_OK) return st;
  // Nothing in the scratch has to start at zero: every call rewrites both
  // segment tables before reading them, and the status word is only written
  // (on a pipeline timeout), never read, on this path.
  // The scratch holds the segment tables only, so P and V enter the PV
  // product as bf16 (no room for the fp16 copy of V the workspace forward uses).
  return attn_fwd_impl(q_head, k_head, v_head, position_ids, shape, rank, softmax_scale, 0, shape->n,
                       whole_rows(shape->n), o_head, o_dtype, lse, scratch, kNoAllocScratchBytes, stream, false);
}

// The status word of the current device's fixed scratch (its first 4 bytes,
// where the forward's kernels record a pipeline timeout), read and cleared
// exactly as ulysses_workspace_status does for a caller's workspace.
extern "C" uly_status ulysses_attn_fwd_noalloc_status(void* stream, int32_t* code) {
  if (!code) return ULY_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const uly_status st = scratch_on_current_device(&scratch);
  if (st != ULY_OK) return st;
  return ulysses_workspace_status(scratch, stream, code);
}
