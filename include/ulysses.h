/*
 * ulysses.h -- C ABI of the single-GPU Ulysses sequence-parallel hot path.
 *
 * Ulysses sequence parallelism (the SP part of Arctic Long Sequence Training)
 * shards a sequence over P ranks, uses an all-to-all to trade the sequence
 * sharding for a head sharding, runs ordinary attention per head over the
 * whole sequence, and uses a second all-to-all to return to the sequence
 * sharding (blog "Ulysses Sequence Parallelism: Training with Million-Token
 * Contexts", "How Ulysses works", steps 1-6; Transformers docs "Ulysses
 * sequence parallelism", the figure at the top of the page).  This library
 * runs that path for P *virtual* ranks that all live in one GPU's memory: the
 * two all-to-alls become the re-layouts below, and the local attention is the
 * forward/backward kernels below.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Sizes are full (unsharded) sizes: b = batch rows, n = tokens per row,
 *    h_q / h_kv = query / key-value heads, d = head dimension, P = ranks.
 *  - Layouts (row-major, innermost last, elements contiguous):
 *      seq-sharded   X_seq [P][b][n/P][H][d]   rank r holds tokens
 *                    [r*n/P, (r+1)*n/P) with all H heads ("How Ulysses
 *                    works", step 1).  For b == 1 this is byte-identical to
 *                    an unsharded [n][H][d] tensor.
 *      head-sharded  X_head[P][b][n][H/P][d]   rank r holds all n tokens of
 *                    heads [r*H/P, (r+1)*H/P) ("How Ulysses works", step 3).
 *      LSE           [P][b][h_q/P][n] float32, natural log.
 *      position_ids  [b][n] int64 on the device; a sample starts at t == 0
 *                    and wherever position_ids[t] == 0.
 *  - GQA: query head h reads kv head h / (h_q/h_kv); ranks split both head
 *    counts contiguously, so each rank's query heads read its own kv heads.
 *    With fewer kv heads than ranks (h_kv < P, P a multiple of h_kv; the
 *    pages are silent on this case) each rank holds one kv head, the copy
 *    of head r*h_kv/P its query heads read: k_head / v_head are then
 *    [P][b][n][1][d], made by ulysses_kv_seq_to_head, and the gradients
 *    dK / dV go back through ulysses_kv_head_to_seq, which sums the copies.
 *  - Pointers are device pointers owned by the caller, 16-byte aligned.
 *    `stream` is a cudaStream_t (NULL = legacy default stream), passed as
 *    void* so this header needs no CUDA header.
 *  - Calls only enqueue work on `stream` and return; results are valid once
 *    the stream has run.  Outputs are fully overwritten (the attention
 *    calls' rank >= 0 mode: that rank's part of them).  The library
 *    allocates no device memory; scratch space is the caller's workspace,
 *    sized by the *_workspace queries.  The only mutable global state is
 *    ulysses_attn_fwd_noalloc's fixed per-GPU scratch array (see there),
 *    plus caches of looked-up addresses (that array's per device, and the
 *    driver's tensor-map encoder), filled once.
 *  - Errors: every argument is checked on the host before anything is
 *    launched; a bad argument returns ULY_ERR_INVALID_ARG (or
 *    ULY_ERR_UNSUPPORTED for a valid but unimplemented size/type) and
 *    enqueues nothing.  A failed launch returns ULY_ERR_CUDA.  Kernels that
 *    wait on their own pipeline stages give up after a bounded time and
 *    record ULY_ERR_TIMEOUT in the workspace status word, which
 *    ulysses_workspace_status() reads.  No call throws or aborts.
 *  - position_ids contents are not validated (that would need a device
 *    sync); whatever they hold is read by the sample-start rule above.
 */
#ifndef ULYSSES_H_
#define ULYSSES_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ULY_OK = 0,
  ULY_ERR_INVALID_ARG = 1,
  ULY_ERR_UNSUPPORTED = 2,
  ULY_ERR_CUDA = 3,
  ULY_ERR_WORKSPACE = 4,
  ULY_ERR_TIMEOUT = 5,
  ULY_ERR_BOUNDS = 6   /* bounds-checked debug build only: an index fell outside its buffer */
} uly_status;

typedef enum { ULY_BF16 = 0, ULY_F32 = 1 } uly_dtype;

/* Full (unsharded) problem sizes. */
typedef struct {
  int64_t b, n, h_q, h_kv, d;
  int32_t P;
} uly_shape;

/*
 * ulysses_seq_to_head -- the first all-to-all ("How Ulysses works", step 3):
 *   x_head[r][bb][t][j][:] = x_seq[t / (n/P)][bb][t % (n/P)][r*(H/P) + j][:]
 * x_seq [P][b][n/P][H][d] -> x_head [P][b][n][H/P][d], elements of `dt`.
 * Requires n % P == 0 and H % P == 0 (Transformers docs "Ulysses sequence
 * parallelism", "Configuration": heads divisible by sp_size, sequence padded
 * to a multiple of sp_size).  Out of place: the buffers must not overlap.
 * Bit-exact copy.
 */
uly_status ulysses_seq_to_head(const void* x_seq, void* x_head, int64_t b, int64_t n, int64_t H,
                               int64_t d, int32_t P, uly_dtype dt, void* stream);

/*
 * ulysses_head_to_seq -- the second all-to-all ("How Ulysses works", step 5),
 * the exact inverse of ulysses_seq_to_head:
 *   x_seq[s][bb][u][g][:] = x_head[g / (H/P)][bb][s*(n/P) + u][g % (H/P)][:]
 * Same requirements.  Also the backward of ulysses_seq_to_head.
 */
uly_status ulysses_head_to_seq(const void* x_head, void* x_seq, int64_t b, int64_t n, int64_t H,
                               int64_t d, int32_t P, uly_dtype dt, void* stream);

/*
 * ulysses_kv_seq_to_head -- the first all-to-all for K and V, for any kv head
 * count the attention accepts.  H_kv a multiple of P: exactly
 * ulysses_seq_to_head.  H_kv < P with P a multiple of H_kv: every rank r
 * receives all n tokens of kv head g(r) = r*H_kv/P, the one its query heads
 * read (a reading: the pages are silent on this case):
 *   x_head[r][bb][t][0][:] = x_seq[t/(n/P)][bb][t%(n/P)][g(r)][:]
 * x_seq [P][b][n/P][H_kv][d], x_head [P][b][n][1][d]; dt ULY_BF16 or ULY_F32;
 * d * element size a multiple of 16 bytes for the replicating case.
 * Errors: as ulysses_seq_to_head; H_kv neither a multiple nor a divisor of
 * P returns ULY_ERR_INVALID_ARG.  Bit-exact copy.
 */
uly_status ulysses_kv_seq_to_head(const void* x_seq, void* x_head, int64_t b, int64_t n, int64_t H_kv,
                                  int64_t d, int32_t P, uly_dtype dt, void* stream);

/*
 * ulysses_kv_head_to_seq -- the backward of ulysses_kv_seq_to_head, for dK
 * and dV.  H_kv a multiple of P: exactly ulysses_head_to_seq.  H_kv < P: the
 * sum of the copies,
 *   x_seq[s][bb][u][g][:] = sum over r with g(r) == g, ascending, of
 *                           x_head[r][bb][s*(n/P) + u][0][:]
 * accumulated in float32 and rounded once to dt (bitwise reproducible).
 * Same layouts and errors as ulysses_kv_seq_to_head.
 */
uly_status ulysses_kv_head_to_seq(const void* x_head, void* x_seq, int64_t b, int64_t n, int64_t H_kv,
                                  int64_t d, int32_t P, uly_dtype dt, void* stream);

/*
 * ulysses_transpose_runs -- dst[j][i][:] = src[i][j][:] for i < A, j < B and
 * runs of run_bytes bytes: the local permutations around a real all-to-all
 * between processes ("How Ulysses works", steps 3 and 5, with each rank a
 * separate GPU).  Before the exchange, rank r's seq shard [b*n/P][P][h*d]
 * becomes P contiguous send chunks [P][b*n/P][h*d] (A = b*n/P, B = P,
 * run = h*d*element size); after it, the received chunks [P][b][n/P*h*d]
 * become the head layout [b][n][h][d] (A = P, B = b, run = n/P*h*d*element
 * size); the way back uses the same call with the roles swapped.  Any
 * alignment (the widest vector both pointers allow); out of place (buffers
 * must not overlap).  Errors: null pointer, A, B or run_bytes < 1, size
 * overflow, overlap: ULY_ERR_INVALID_ARG.  Bit-exact copy.
 */
uly_status ulysses_transpose_runs(const void* src, void* dst, int64_t A, int64_t B, int64_t run_bytes,
                                  void* stream);

/* Workspace bytes ulysses_attn_fwd needs for `shape` (0 on invalid shape). */
size_t ulysses_attn_fwd_workspace(const uly_shape* shape);

/*
 * ulysses_attn_fwd -- local causal attention of each rank on its head slice
 * ("How Ulysses works", step 4), with causality and sample boundaries from
 * position_ids (blog, position_ids paragraph; Accelerate guide "Sequence
 * parallelism", "ALST/Ulysses SP backend configuration": packed samples must
 * not attend to one another).  For rank r, local query head j (kv head j/G),
 * and row i:  O_i = sum_j softmax_j(scale * q_i . k_j) v_j over keys j <= i
 * in i's sample;  LSE_i = log sum_j exp(scale * q_i . k_j).
 *   q_head [P][b][n][h_q/P][d] bf16, k_head / v_head [P][b][n][h_kv/P][d]
 *   bf16 ([P][b][n][1][d] when h_kv < P), position_ids [b][n] int64
 *   (device).
 *   rank: -1 computes every rank; 0 <= rank < P computes only that rank's
 *   slice (rows of other ranks in o_head / lse are left untouched).
 *   softmax_scale <= 0 selects 1/sqrt(d).
 *   o_head [P][b][n][h_q/P][d] of o_dtype (ULY_BF16 or ULY_F32);
 *   lse [P][b][h_q/P][n] float32.
 *   ws / ws_bytes: device workspace of at least ulysses_attn_fwd_workspace()
 *   bytes, 256-byte aligned (else ULY_ERR_WORKSPACE).
 * Supports d in {64, 128} (else ULY_ERR_UNSUPPORTED).
 * Arithmetic: S = q k^T from the bf16 inputs with float32 accumulation; the
 * softmax in float32; P rounded to fp16 for P V, against an fp16 copy of v
 * scaled by a power of two (held in the workspace; the scale is folded back
 * exactly); O accumulated in float32.  No atomics: results are bitwise
 * reproducible from call to call.
 */
uly_status ulysses_attn_fwd(const void* q_head, const void* k_head, const void* v_head,
                            const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                            float softmax_scale, void* o_head, uly_dtype o_dtype, float* lse,
                            void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes ulysses_attn_bwd needs for `shape` and gradient dtype. */
size_t ulysses_attn_bwd_workspace(const uly_shape* shape, uly_dtype g_dtype);

/*
 * ulysses_attn_bwd -- gradients of the local attention (training through the
 * layer, Accelerate guide "Sequence parallelism", custom training loop):
 *   D_i = dO_i . O_i;  P_ij = exp(scale * q_i . k_j - LSE_i);
 *   dS_ij = P_ij (dO_i . v_j - D_i);
 *   dQ_i = scale * sum_j dS_ij k_j;
 *   dK_j = scale * sum_{query heads of j's group} sum_i dS_ij q_i;
 *   dV_j = sum_{query heads of j's group} sum_i P_ij dO_i.
 * Inputs in head layout as for ulysses_attn_fwd; o_head / lse are that call's
 * outputs (o_dtype must match); do_head has q_head's layout (bf16).
 * Outputs dq_head (q_head's layout), dk_head / dv_head (k_head's layout), of
 * g_dtype.  rank / softmax_scale as for the forward.
 * Arithmetic: the products take fp16 copies of q, k, v and dO, each scaled by
 * a power of two chosen from its largest magnitude (exact; folded back into
 * the results); P and dS are rounded to fp16 before they enter dV, dK and
 * dQ; all accumulation is float32.  No atomics: results are bitwise
 * reproducible from call to call.
 */
uly_status ulysses_attn_bwd(const void* q_head, const void* k_head, const void* v_head,
                            const void* o_head, uly_dtype o_dtype, const float* lse,
                            const void* do_head, const int64_t* position_ids,
                            const uly_shape* shape, int32_t rank, float softmax_scale,
                            void* dq_head, void* dk_head, void* dv_head, uly_dtype g_dtype,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * Ring attention / the Ulysses + ring hybrid (Accelerate guide "Sequence
 * parallelism", "How Ulysses SP differs from FSDP CP"; blog "Ulysses Sequence
 * Parallelism: Training with Million-Token Contexts", ring attention): the
 * sequence is cut into key/value blocks, every query meets one block at a
 * time, and the partial results are merged by their log-sum-exp.
 *
 * ulysses_attn_fwd_kv_range -- ulysses_attn_fwd over the keys of one block:
 * key j takes part for query i only if k_lo <= j < k_hi besides the usual
 * rule (same sample, j <= i).  A row that sees no key of the block gets
 * O = 0 and LSE = -inf.  Requires 0 <= k_lo < k_hi <= n (else
 * ULY_ERR_INVALID_ARG); everything else as ulysses_attn_fwd.
 */
uly_status ulysses_attn_fwd_kv_range(const void* q_head, const void* k_head, const void* v_head,
                                     const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                     float softmax_scale, int64_t k_lo, int64_t k_hi, void* o_head,
                                     uly_dtype o_dtype, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * ulysses_attn_bwd_kv_range -- one key block's share of the backward, given
 * the merged (all blocks) o_head and lse: with P_ij = exp(scale q_i.k_j -
 * LSE_i) over the block's visible keys, D_i = dO_i . O_i and
 * dS = P (dO V^T - D), dq_head gets this block's share of dQ (the blocks'
 * shares add up to dQ), dk_head / dv_head the complete dK, dV of the
 * block's keys and zeros for every other key.  Same arguments as
 * ulysses_attn_bwd plus k_lo, k_hi (0 <= k_lo < k_hi <= n).
 */
uly_status ulysses_attn_bwd_kv_range(const void* q_head, const void* k_head, const void* v_head,
                                     const void* o_head, uly_dtype o_dtype, const float* lse,
                                     const void* do_head, const int64_t* position_ids,
                                     const uly_shape* shape, int32_t rank, float softmax_scale,
                                     int64_t k_lo, int64_t k_hi, void* dq_head, void* dk_head,
                                     void* dv_head, uly_dtype g_dtype, void* ws, size_t ws_bytes,
                                     void* stream);

/*
 * ulysses_attn_lse_merge -- combines the partial results of nparts key
 * blocks:  LSE = log sum_b exp(LSE_b),  O = sum_b exp(LSE_b - LSE) O_b.
 * Rows where every LSE_b is -inf get O = 0, LSE = -inf.
 *   o_parts    float [nparts][P][b][n][h_q/P][d] (head layout, fp32)
 *   lse_parts  float [nparts][P][b][h_q/P][n]
 *   o_head     [P][b][n][h_q/P][d] of o_dtype; lse [P][b][h_q/P][n] float.
 * 1 <= nparts <= 32; d 64 or 128 (else ULY_ERR_UNSUPPORTED); outputs must
 * not overlap inputs or each other; 16-byte aligned.  One launch; float32
 * arithmetic.
 */
uly_status ulysses_attn_lse_merge(const float* o_parts, const float* lse_parts, int32_t nparts,
                                  const uly_shape* shape, void* o_head, uly_dtype o_dtype, float* lse,
                                  void* stream);

/*
 * Block calls: one block of query rows against one block of key rows, each
 * stored compactly (ring attention, where a rank holds only its own
 * sequence block and receives the others' key blocks one at a time).
 *   q_blk, o_blk, do_blk, dq_blk  [P][b][q_rows][h_q/P][d]: global rows
 *                                 [q_base, q_base + q_rows)
 *   k_blk, v_blk, dk_blk, dv_blk  [P][b][k_rows][kv heads per rank][d]:
 *                                 global keys [k_base, k_base + k_rows)
 *   lse_blk                       [P][b][h_q/P][q_rows]
 *   position_ids                  [b][n], the whole sequence's (sample
 *                                 starts are global)
 * q_base and k_base are multiples of 128, both blocks lie inside [0, n)
 * (ULY_ERR_INVALID_ARG otherwise).  All P ranks' head slices are computed.
 * Query i sees key j iff j <= i, both in one sample, and j in the key block.
 * ulysses_attn_fwd_block gives each query row's partial O and LSE over the
 * key block (O = 0, LSE = -inf for a row that sees none of it), to be
 * combined with ulysses_attn_lse_merge.  ulysses_attn_bwd_block takes the
 * merged O and LSE of the query block and gives the key block's share of
 * dQ and the query block's contributions to dK and dV (all overwritten).
 * Workspaces as for the whole-sequence calls with the same shape.  Only
 * the tiles of the two blocks are launched.
 */
uly_status ulysses_attn_fwd_block(const void* q_blk, const void* k_blk, const void* v_blk,
                                  const int64_t* position_ids, const uly_shape* shape, int64_t q_base,
                                  int64_t q_rows, int64_t k_base, int64_t k_rows, float softmax_scale,
                                  void* o_blk, uly_dtype o_dtype, float* lse_blk, void* ws, size_t ws_bytes,
                                  void* stream);
uly_status ulysses_attn_bwd_block(const void* q_blk, const void* k_blk, const void* v_blk, const void* o_blk,
                                  uly_dtype o_dtype, const float* lse_blk, const void* do_blk,
                                  const int64_t* position_ids, const uly_shape* shape, int64_t q_base,
                                  int64_t q_rows, int64_t k_base, int64_t k_rows, float softmax_scale,
                                  void* dq_blk, void* dk_blk, void* dv_blk, uly_dtype g_dtype, void* ws,
                                  size_t ws_bytes, void* stream);

/*
 * ulysses_accumulate -- dst[i] += src[i] for i < count, float32 (count a
 * multiple of 4, both 16-byte aligned; dst == src is allowed, other
 * overlaps are not).  The ring passes' sums of dQ shares and of the dK / dV
 * that travel with a key block.
 */
uly_status ulysses_accumulate(float* dst, const float* src, int64_t count, void* stream);

/*
 * ulysses_attn_bwd_timed -- ulysses_attn_bwd that also records five
 * caller-owned CUDA events on `stream` around its kernels, for measuring
 * each kernel's device time (the pages have no counterpart; this is
 * instrumentation).  events[0] before the sample-table kernel, events[1]
 * before the preparation kernels (largest magnitudes, fp16 operand copies,
 * row statistics), events[2] before the dK/dV kernel,
 * events[3] before the dQ kernel, events[4] after it.  `events` points to
 * five cudaEvent_t handles (as void*), created by the caller on the current
 * device; a null array or a null handle returns ULY_ERR_INVALID_ARG and
 * enqueues nothing.  A failed record returns ULY_ERR_CUDA.  All other
 * arguments, results and errors are those of ulysses_attn_bwd.
 */
uly_status ulysses_attn_bwd_timed(const void* q_head, const void* k_head, const void* v_head,
                                  const void* o_head, uly_dtype o_dtype, const float* lse,
                                  const void* do_head, const int64_t* position_ids,
                                  const uly_shape* shape, int32_t rank, float softmax_scale,
                                  void* dq_head, void* dk_head, void* dv_head, uly_dtype g_dtype,
                                  void* ws, size_t ws_bytes, void* stream, void* const* events);

/*
 * ulysses_attn_fwd_noalloc -- ulysses_attn_fwd without a caller workspace.
 * The pages have no counterpart for this call; it exists for callers that
 * cannot allocate device memory themselves: code that runs under a framework
 * whose allocator owns all device memory and forbids raw allocations on the
 * hot path, or a service that reserves its memory once at start-up and must
 * not allocate per request.  Same arguments and results as ulysses_attn_fwd,
 * minus ws / ws_bytes.
 *   Scratch: a fixed 4 MiB + 256 B device array inside the library, one per
 *   GPU that loads the library, held until the process exits.  It covers
 *   b * n <= 524288 tokens; larger shapes return ULY_ERR_WORKSPACE and
 *   enqueue nothing.  The call allocates nothing (no cudaMalloc, no
 *   allocating library routine).
 *   First call per device: looks up the scratch's device address
 *   (cudaGetSymbolAddress) with that device current and caches it for the
 *   life of the process; make that first call before any stream capture.
 *   cudaDeviceReset (which reloads the module and may move the array) is not
 *   supported while this library is loaded: the cached address would be
 *   stale.
 *   Sharing: every call on a device uses the same scratch and it keeps the
 *   last call's contents (nothing in it needs to start at zero).  Calls whose
 *   work overlaps on the GPU (e.g. on two concurrently running streams) race
 *   on it and give wrong results: serialise them.
 *   A pipeline timeout inside the kernel is not reported by this call: the
 *   kernels record it in the scratch's status word, which
 *   ulysses_attn_fwd_noalloc_status reads.
 */
uly_status ulysses_attn_fwd_noalloc(const void* q_head, const void* k_head, const void* v_head,
                                    const int64_t* position_ids, const uly_shape* shape, int32_t rank,
                                    float softmax_scale, void* o_head, uly_dtype o_dtype, float* lse,
                                    void* stream);

/*
 * ulysses_attn_fwd_noalloc_status -- the status word of the current device's
 * fixed no-alloc scratch, read and then cleared, as ulysses_workspace_status
 * does for a workspace: *code = ULY_OK, ULY_ERR_TIMEOUT (a kernel gave up
 * waiting on its own pipeline since the last read), ULY_ERR_CUDA or
 * ULY_ERR_BOUNDS.  Enqueues a 4-byte copy and a clear on `stream` and waits
 * for both (a host synchronisation: not for use under stream capture).  The
 * word is shared by every no-alloc call on the device, like the scratch.
 * Returns ULY_ERR_INVALID_ARG for a null code.  The pages have no
 * counterpart for this call.
 */
uly_status ulysses_attn_fwd_noalloc_status(void* stream, int32_t* code);

/*
 * ulysses_sp_loss_aggregate -- weighted loss aggregation across the P SP
 * ranks (Accelerate guide "Sequence parallelism", custom training loop: the
 * differentiable weighted per-rank loss aggregation; blog "Ulysses Sequence
 * Parallelism: Training with Million-Token Contexts", "Loss aggregation").
 *   good[r]    = number of shift_labels of rank r that are not ignore_index
 *                (the pages use -100);
 *   *loss      = (sum over r with good[r] > 0 of losses[r] * good[r])
 *                / max(sum_r good[r], 1);
 *   dlosses[r] = d(*loss)/d(losses[r]) = good[r] / max(sum good, 1) if
 *                good[r] > 0, else 0.
 * A rank without valid labels is skipped, not multiplied by zero, so a NaN
 * loss there does not reach the result.  Sums run in double precision in a
 * fixed order (bitwise reproducible); *loss and dlosses are rounded to
 * float once at the end.
 *   losses        float[P], device, the per-rank losses.
 *   shift_labels  int64 [P][b][n/P], device, seq-sharded like the inputs
 *                 (rank r's b rows of n/P labels are contiguous).
 *   loss          float[1], good int64[P], dlosses float[P]: device outputs,
 *                 fully overwritten; none may overlap the inputs or each other.
 * Errors: null pointer, P < 1 or P > 1024, b < 1, n < 1, n % P != 0,
 * misalignment (4 bytes for float, 8 for int64) or overlap return
 * ULY_ERR_INVALID_ARG and enqueue nothing; a failed launch ULY_ERR_CUDA.
 * Two kernel launches on `stream`.
 */
uly_status ulysses_sp_loss_aggregate(const float* losses, const int64_t* shift_labels, int64_t b,
                                     int64_t n, int32_t P, int64_t ignore_index, float* loss,
                                     int64_t* good, float* dlosses, void* stream);

/*
 * ulysses_workspace_status -- synchronizes `stream`, then reads and clears
 * the status word kept at the start of an attention workspace.  *code gets
 * ULY_OK, ULY_ERR_TIMEOUT when a kernel gave up waiting on one of its own
 * pipeline stages, ULY_ERR_CUDA when a kernel found its dynamic shared
 * memory too poorly aligned to lay out its tiles and did nothing, or (in
 * the bounds-checked debug build) ULY_ERR_BOUNDS when an index or a tile
 * coordinate fell outside its buffer and the access was skipped (in every
 * error case the outputs are invalid).
 */
uly_status ulysses_workspace_status(void* ws, void* stream, int32_t* code);

/*
 * ulysses_debug_status -- the bounds-checked debug build (libulysses_debug.so,
 * compiled with ULY_DEBUG_BOUNDS) checks every global index and TMA tile
 * coordinate of its kernels before the access, records one that falls
 * outside its buffer and skips it.  The attention kernels record into their
 * workspace status word; the re-layout kernels, which take no workspace,
 * into a word of the library's own, which this call synchronizes `stream`,
 * reads and clears: *code = ULY_OK or ULY_ERR_BOUNDS.  The release build
 * compiles no checks: it sets *code = ULY_OK and returns ULY_ERR_UNSUPPORTED.
 */
uly_status ulysses_debug_status(void* stream, int32_t* code);

/*
 * Between GPUs: the two all-to-alls fused with the re-layout
 * ----------------------------------------------------------
 * Blog "How Ulysses works", steps 3 and 5, with one GPU per rank: each rank
 * stores its chunks straight into its peers' buffers over NVLink (plain
 * stores through peer-mapped pointers; no collective library, no TMA), then
 * releases one flag per destination.  A consumer runs ulysses_wait_flags on
 * its own flag array before reading what it received.
 *
 * ulysses_seq_to_head_push -- rank `rank` of P sends its seq shard
 *   x_seq [b][n/P][H][d] (its own device memory) to every rank s:
 *     dst_heads[s][bb][rank*n/P + t][j] = x_seq[bb][t][s*H/P + j]
 *   dst_heads[s] is rank s's head-layout buffer [b][n][H/P][d] (for
 *   s != rank a peer-mapped pointer, e.g. from ulysses_ipc_open).  Once all
 *   of rank s's rows are stored and fenced at system scope, `epoch` is
 *   stored with release semantics into dst_flags[s][rank] (dst_flags[s]:
 *   rank s's uint32 flag array of P slots).
 * ulysses_head_to_seq_push -- the inverse, for O and the gradients: rank
 *   `rank` holds x_head [b][n][H/P][d] (heads [rank*H/P, (rank+1)*H/P) of
 *   all tokens) and sends tokens [s*n/P, (s+1)*n/P) to rank s:
 *     dst_seqs[s][bb][t][rank*H/P + j] = x_head[bb][s*n/P + t][j]
 *   then releases dst_flags[s][rank] = epoch.
 *   Both: arrays dst_* hold P pointers (host memory); P <= 64; dtype bf16
 *   or fp32; H/P*d*element size a multiple of 16 bytes (else
 *   ULY_ERR_UNSUPPORTED); epoch != 0 (a flag's 0 means "nothing yet"; use a
 *   new epoch per exchange); ws: device workspace of >= 4*P bytes, 256-byte
 *   aligned, for the per-destination completion counters (cleared by the
 *   call).  The caller guarantees that no destination is still reading the
 *   buffer from an earlier exchange (e.g. a barrier or double buffering).
 *
 * ulysses_wait_flags -- one warp polls flags[0..count) with acquire loads
 *   at system scope until every slot holds `epoch` or a later epoch
 *   (compared modulo 2^32: slot - epoch as a signed 32-bit number is >= 0;
 *   epochs grow by one per exchange, so a slot never lags or leads by 2^31 or
 *   more).  Kernels enqueued after
 *   it on `stream` then see the data the flags released.  Gives up after
 *   limit_ns (in [1 us, 60 s]) and records ULY_ERR_TIMEOUT in the status
 *   word at the start of ws (256-byte aligned device memory; read it with
 *   ulysses_workspace_status).
 *
 * ulysses_release_flags -- stores `epoch` (!= 0) into each of `count` (1..64)
 *   uint32 slots (device addresses, this GPU's or peer-mapped), each after a
 *   system-scope fence and with release semantics: everything enqueued on
 *   `stream` before it is visible to whoever acquires a slot.  The "buffer
 *   free" signal of a receiver to its senders; the push calls do the same
 *   for their data.
 *
 * ulysses_ipc_handle / ulysses_ipc_open / ulysses_ipc_close -- the CUDA IPC
 *   handle (64 bytes) of a device allocation, opened in another process as
 *   a peer-mapped pointer (peer access enabled lazily), and closed again.
 *   Host-side plumbing for the push calls; ULY_ERR_CUDA when CUDA refuses.
 */
uly_status ulysses_seq_to_head_push(const void* x_seq, void* const* dst_heads, uint32_t* const* dst_flags,
                                    int32_t rank, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                                    uly_dtype dtype, uint32_t epoch, void* ws, size_t ws_bytes, void* stream);
uly_status ulysses_head_to_seq_push(const void* x_head, void* const* dst_seqs, uint32_t* const* dst_flags,
                                    int32_t rank, int64_t b, int64_t n, int64_t H, int64_t d, int32_t P,
                                    uly_dtype dtype, uint32_t epoch, void* ws, size_t ws_bytes, void* stream);
uly_status ulysses_wait_flags(const uint32_t* flags, int32_t count, uint32_t epoch, uint64_t limit_ns, void* ws,
                              void* stream);
uly_status ulysses_release_flags(uint32_t* const* slots, int32_t count, uint32_t epoch, void* stream);
uly_status ulysses_ipc_handle(const void* dev_ptr, void* handle_out);
uly_status ulysses_ipc_open(const void* handle, void** dev_ptr_out);
uly_status ulysses_ipc_close(void* dev_ptr);

/*
 * ulysses_layer_step_host -- one whole Ulysses layer step, forward and
 * backward, from host memory to host memory ("How Ulysses works", steps
 * 1-6): the seq-sharded inputs are copied in, seq_to_head(q, k, v) ->
 * ulysses_attn_fwd -> head_to_seq(O); seq_to_head(dO) -> ulysses_attn_bwd ->
 * head_to_seq(dQ, dK, dV) run for all P virtual ranks, and the seq-sharded
 * outputs are copied out.  A convenience over the calls above, with the
 * copies overlapping the attention kernels:
 *   inputs   q_seq, do_seq [P][b][n/P][h_q][d] bf16; k_seq, v_seq
 *            [P][b][n/P][h_kv][d] bf16; position_ids [b][n] int64: host
 *            memory, page-locked for the copies to run asynchronously
 *   outputs  o_seq, dq_seq [P][b][n/P][h_q][d] float; dk_seq, dv_seq
 *            [P][b][n/P][h_kv][d] float: host memory, page-locked
 *   dev      caller-owned device memory of ulysses_layer_step_host_bytes()
 *            bytes, 256-byte aligned (ULY_ERR_WORKSPACE otherwise), zeroed
 *            once before the first call (it holds the attention workspaces'
 *            status words): device staging, head-layout buffers and both
 *            attention workspaces; reused by every call with the same shape
 *   streams  `stream` runs the kernels and the copy of position_ids,
 *            `h2d_stream` the other host-to-device and `d2h_stream` the
 *            device-to-host copies (three distinct streams of the current
 *            device)
 *   events   three caller-created cudaEvent_t (as void*), the same for every
 *            call on `dev`, that order consecutive calls: events[0] "this
 *            call's staged q, k, v and dO are consumed", recorded after its
 *            last seq_to_head and before its backward (the next call's input
 *            copies wait for it, so they overlap this call's backward; the
 *            host input buffers may be rewritten once it has completed),
 *            events[1] "O is on the host", events[2] "the gradients are on
 *            the host".  All outputs of a call are on the host once the
 *            events[2] it recorded has completed (cudaEventSynchronize).
 * Errors as for the calls it makes; ulysses_layer_status reads (and
 * clears) the attention workspaces' status words inside `dev`.
 */
size_t ulysses_layer_step_host_bytes(const uly_shape* shape);
uly_status ulysses_layer_step_host(const void* q_seq, const void* k_seq, const void* v_seq, const void* do_seq,
                                   const int64_t* position_ids, const uly_shape* shape, float softmax_scale,
                                   float* o_seq, float* dq_seq, float* dk_seq, float* dv_seq, void* dev,
                                   size_t dev_bytes, void* stream, void* h2d_stream, void* d2h_stream,
                                   void* const* events);
uly_status ulysses_layer_status(void* dev, const uly_shape* shape, void* stream, int32_t* code);

/*
 * ulysses_selftest_wait_timeout -- runs the failure path of the attention
 * kernels' bounded waits on purpose, so that it can be checked on a GPU.
 * (Not a step of the method: the pages have no counterpart; it tests the
 * library's own failure detection.)  One CTA of the attention kernels'
 * shape allocates TMEM, starts one bulk copy of workspace bytes
 * [256, 1280) into shared memory, and then waits on a barrier nothing
 * arrives at: the first wait to exceed limit_ns records ULY_ERR_TIMEOUT in
 * the workspace status word and raises the CTA's abort flag, the other
 * waits return on the flag, the copy is waited for (bounded), TMEM is freed
 * and the kernel returns.  The stream and context stay usable.
 *   ws, ws_bytes  device workspace, 256-byte aligned, >= 1280 bytes
 *                 (ULY_ERR_WORKSPACE otherwise); only its status word is
 *                 written.
 *   limit_ns      the waits' time limit, in [1000, 5e9] ns
 *                 (ULY_ERR_INVALID_ARG otherwise).
 * Returns once the kernel is enqueued; ulysses_workspace_status(ws, ...)
 * then reports ULY_ERR_TIMEOUT.
 */
uly_status ulysses_selftest_wait_timeout(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream);

/* Static English text for a status code. */
const char* ulysses_status_string(uly_status s);

#ifdef __cplusplus
}
#endif

#endif /* ULYSSES_H_ */
