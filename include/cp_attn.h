/*
 * cp_attn.h — C ABI of the B200 (sm_100a) context-parallel attention library.
 *
 * The method (page "序列与上下文并行", ai-infra-wiki, section
 * "上下文并行：注意力本身切分"): the sequence of S tokens is split over N ranks;
 * each rank holds its own Q/K/V block; K/V blocks travel around a ring so that
 * at ring step t rank r computes its Q block against the K/V block of rank
 * (r + t) mod N; the per-step partial results (O, logsumexp) are merged by
 * online softmax, which yields exactly full softmax attention. For causal
 * attention a zigzag assignment of chunks to ranks balances the work (same
 * section). Here the N ranks are virtual: all of them run on one GPU as tile
 * and CTA scheduling.
 *
 * Attention itself (page "Tensor并行与算子拆分", aiknowledge.cn, section
 * "注意力的并行化优化"): O = softmax(Q K^T * scale + mask) V with masked
 * scores set to -inf; scale defaults to 1/sqrt(D). The causal mask keeps key
 * j for query i iff pos(j) <= pos(i) in GLOBAL token positions (page
 * "序列与上下文并行", section "工程实践": positions are global under context
 * parallelism).
 *
 * Layouts (element order, outermost first; all tensors dense, no padding):
 *   natural              [B][S][H][D]
 *   CP_LAYOUT_CONTIGUOUS [N][B][S/N][H][D]  rank r holds tokens [r*S/N, (r+1)*S/N)
 *                        (page "序列并行：超长序列训练", guijiagi.com, split diagram)
 *   CP_LAYOUT_ZIGZAG     [N][B][2C][H][D], C = S/(2N): rank r holds chunk r then
 *                        chunk 2N-1-r of 2N equal chunks (the zigzag reading)
 *   CP_LAYOUT_ULYSSES    inputs/outputs as sequence shards [N][B][S/N][H][D];
 *                        internally head groups [N][B][S][H/N][D], group g holding
 *                        heads [g*H/N, (g+1)*H/N) (page "序列并行：超长序列训练",
 *                        UlyssesAttention example: all-to-all, local attention over
 *                        the full sequence, all-to-all back)
 *   lse                  float32 [B][H][S], natural token order, natural log of
 *                        the sum of exp of the scaled scores.
 *
 * Conventions for every entry point:
 *   - Status codes: CP_OK (0) or a negative CP_ERR_*; no exception crosses the ABI.
 *   - Device pointers must be 16-byte aligned (CP_ERR_ALIGNMENT otherwise).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Entry points
 *     that take a stream only enqueue work: they neither allocate device memory
 *     nor synchronise, except cp_attn_check, which synchronises `stream`.
 *   - The caller owns every input, output and workspace buffer. A plan owns only
 *     its host schedule and a small device table (work list + status word)
 *     allocated by cp_attn_plan and freed by cp_attn_plan_destroy.
 *   - Plans are immutable after creation; concurrent calls on one plan with
 *     distinct outputs and workspaces are safe.
 *   - Kernel waits are bounded: a wait that runs out sets the plan's status word,
 *     the kernel returns early, and the next cp_attn_check reports CP_ERR_TIMEOUT.
 */
#ifndef CP_ATTN_H_
#define CP_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CP_API __attribute__((visibility("default")))
#else
#define CP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA header. */
typedef void* cp_stream_t;

enum {
  CP_OK = 0,
  CP_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad enum value */
  CP_ERR_UNSUPPORTED = -2,   /* D not in {64,128}; S not divisible by N (2N for zigzag);
                                H not divisible by N (Ulysses); sizes beyond int32 indexing */
  CP_ERR_ALIGNMENT = -3,     /* a device pointer is not 16-byte aligned */
  CP_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed, or no device */
  CP_ERR_TIMEOUT = -5,       /* a bounded in-kernel wait ran out (reported by cp_attn_check) */
  CP_ERR_WORKSPACE = -6      /* workspace pointer null or smaller than required */
};

typedef enum {
  CP_LAYOUT_CONTIGUOUS = 0,
  CP_LAYOUT_ZIGZAG = 1,
  CP_LAYOUT_ULYSSES = 2
} cp_layout_t;

typedef struct cp_attn_plan_s* cp_attn_plan_t;

/*
 * Build a plan for B batches, H heads, S tokens, head dim D (64 or 128), N
 * virtual ranks, causal (0/1), a layout, and a softmax scale (<= 0 selects
 * 1/sqrt(D)). The plan holds the ring schedule (per rank r and step t the
 * key/value rank (r+t) mod N; per (query tile, key tile) pair of 128 tokens
 * the class full / masked / skipped), the work list of query-tile pairs sorted
 * by descending executed-tile count, and, when a CUDA device is present, a
 * device copy of the work list plus a status word. Without a device the plan
 * is still created (host queries work) and every launch returns CP_ERR_CUDA.
 * Ulysses plans take causal = 0 only (CP_ERR_UNSUPPORTED otherwise).
 * On success *out receives the plan; on failure *out is set to NULL.
 */
CP_API int cp_attn_plan(cp_attn_plan_t* out, int B, int H, int S, int D, int N, int causal,
                 int layout, float softmax_scale);

/* Free a plan and its device table. NULL is accepted. Not to be called while a
 * launch on the plan may still be running (synchronise first). */
CP_API int cp_attn_plan_destroy(cp_attn_plan_t plan);

/*
 * Executed 128x128 (query tile, key tile) pairs of each virtual rank, summed
 * over ring steps, batches and heads: per_rank[N] (host memory, may be NULL).
 * Returns the total over ranks, or a negative status. For the zigzag causal
 * layout every rank gets the same count; for the contiguous causal layout rank
 * r's count grows with r (the load imbalance of the causal section).
 */
CP_API int64_t cp_attn_plan_tile_counts(cp_attn_plan_t plan, int64_t* per_rank);

/* Number of work items (pairs of 128-row query tiles) in the plan's work list. */
CP_API int64_t cp_attn_plan_num_items(cp_attn_plan_t plan);

/*
 * Static schedule of the attention kernel: one persistent CTA per SM runs a
 * contiguous run of the work list, assigned at plan time by giving each item,
 * in list order, to the CTA with the earliest modelled finish. The model counts
 * two units per executed key tile of the item plus three per item. Writes each
 * CTA's modelled load to per_cta[n_cta] (host memory, may be NULL) and returns
 * n_cta (the SM count of the device current at plan time, 148 when none is
 * visible, capped by the number of items), or a negative status.
 */
CP_API int64_t cp_attn_plan_cta_loads(cp_attn_plan_t plan, int64_t* per_cta);

/*
 * Workspace bytes needed by cp_attn_fwd (with_partials = 0) or
 * cp_attn_fwd_partials (with_partials = 1). 0 for contiguous/zigzag fused
 * calls; 4 * B*S*H*D*2 bytes (Q, K, V and O head groups) for Ulysses.
 */
CP_API size_t cp_attn_workspace_bytes(cp_attn_plan_t plan, int with_partials);

/*
 * Fused forward: O and lse of full softmax attention, computed by visiting for
 * each query tile of each virtual rank r the key/value tiles of ranks
 * (r+t) mod N for t = 0..N-1 in that order, merging every step into one
 * running online-softmax state (the incremental merge of the context-parallel
 * section), skipping key tiles that lie wholly above the causal diagonal.
 *   q, k, v : bf16, in the plan's layout (see above), device
 *   o       : bf16, same layout and size as q, device (written)
 *   lse     : float32 [B][H][S] natural token order, device (written); may be NULL
 *   workspace : device, cp_attn_workspace_bytes(plan, 0) bytes (NULL if 0)
 * q, k, v must not overlap o or workspace.
 */
CP_API int cp_attn_fwd(cp_attn_plan_t plan, const void* q, const void* k, const void* v,
                void* o, float* lse, void* workspace, cp_stream_t stream);

/*
 * Unfused forward (contiguous/zigzag only; CP_ERR_UNSUPPORTED for Ulysses):
 * the per-ring-step partials of the context-parallel section, unmerged.
 *   o_parts   : float32 [N][rows][D], device (written)
 *   lse_parts : float32 [N][rows], device (written)
 * with rows = N*B*(S/N)*H ordered like q's tokens and heads,
 * row = ((r*B + b)*(S/N) + tl)*H + h, and part t holding rank r's rows
 * against the key/value block of rank (r+t) mod N. A row with no allowed key in
 * a step gets O = 0, lse = -inf. O_t is normalised (the softmax-weighted mean
 * over that step's keys) and lse_t is natural-log. cp_merge_partials over the
 * N parts gives O in q's layout and lse in row order.
 */
CP_API int cp_attn_fwd_partials(cp_attn_plan_t plan, const void* q, const void* k, const void* v,
                         float* o_parts, float* lse_parts, void* workspace,
                         cp_stream_t stream);

/*
 * One ring step of one rank, on rank-local buffers (contiguous and zigzag
 * layouts; CP_ERR_UNSUPPORTED for Ulysses). Page "序列与上下文并行", section
 * "上下文并行：注意力本身切分": rank r holds its own Q/K/V chunk and, at ring step
 * t, computes the partial attention of its queries against the key/value block
 * of rank (r+t) mod N, which it has received from the ring; the N partials are
 * merged by online softmax (cp_merge_partials). Causal masking uses the global
 * positions of the two ranks' tokens under the plan's layout.
 *   rank, step : 0 <= rank, step < N
 *   q          : bf16 [B][S/N][H][D], rank's own chunk (its local tokens in the
 *                layout's order: zigzag rank r holds chunks r and 2N-1-r), device
 *   k, v       : bf16 [B][S/N][H][D], the block of rank (rank+step) mod N, device
 *   o_part     : float32 [B*(S/N)*H][D], row = (b*(S/N) + tl)*H + h, device (written)
 *   lse_part   : float32 [B*(S/N)*H], same rows, device (written)
 * O is normalised over the step's keys, lse is natural-log; a row with no
 * allowed key in the step gets O = 0, lse = -inf. One kernel is enqueued on
 * `stream`. The first call for a rank builds that rank's per-step schedules and
 * copies them to the device synchronously (cp_attn_ring_prepare does it ahead of
 * time, e.g. before a stream capture). Errors: CP_ERR_INVALID_ARG (null pointer,
 * rank or step out of range), CP_ERR_ALIGNMENT (a pointer not 16-byte aligned),
 * CP_ERR_CUDA (no device, launch failure); an in-kernel wait that runs out is
 * reported by cp_attn_check as CP_ERR_TIMEOUT.
 */
CP_API int cp_attn_fwd_ring_step(cp_attn_plan_t plan, int rank, int step, const void* q, const void* k,
                                 const void* v, float* o_part, float* lse_part, cp_stream_t stream);

/*
 * One rank's whole ring forward in one launch, fetching the other ranks' blocks
 * itself. Page "序列与上下文并行", section "上下文并行：注意力本身切分": the rank
 * computes on the blocks it holds while the next ones arrive. The work runs on
 * persistent CTAs in two phases: ring steps t < split = ceil(N/2) (all N steps
 * for N <= 2) as one unit per (step, pair of query tiles), step-major, starting
 * on the rank's own block; then one unit per pair over steps [split, N), its
 * online-softmax state kept on chip across them. Part t < split holds step t's
 * partial, part split the merged partial of the remaining steps:
 * cp_attn_ring_num_parts(plan) parts in all. Meanwhile two copy warps of every CTA fetch the blocks of
 * ranks rank+1, rank+2, ... (mod N), in that order, in 32 KiB chunks, from
 * pull_k[j] / pull_v[j] into slot j of k_all / v_all, counting finished chunks in
 * arrived[j]; a unit reads slot j once all of its chunks have arrived. The
 * launch is cooperative (all CTAs resident), so every wait ends. Behind NVSwitch
 * pull_k[j] is rank j's own block in its memory, mapped here (cp_ipc_open_handle):
 * each block crosses NVLink once, by loads of the copy warps, with no copy
 * engine or stream between the transfer and the math.
 *   q            : bf16 [B][S/N][H][D], this rank's own chunk, device
 *   k_all, v_all : bf16 [N][B][S/N][H][D] (written: the pulled slots); slot
 *                  `rank` holds the rank's own block before the launch, device
 *   pull_k, pull_v : host arrays of N device pointers, entry j = rank j's own
 *                  K/V block [B][S/N][H][D] as addressable from this GPU (entry
 *                  `rank` unused), 16-byte aligned, unchanged until the kernel
 *                  ends; both NULL: no pull, every slot already holds its block
 *   arrived      : int32 [N] device workspace, needed when pulling (set to 0
 *                  on `stream` before the launch); must be NULL without pull
 *                  sources (see cp_attn_fwd_ring_external for a wait on
 *                  arrivals the caller raises)
 *   o_parts      : float32 [P][B*(S/N)*H][D], P = cp_attn_ring_num_parts(plan),
 *                  device (written)
 *   lse_parts    : float32 [P][B*(S/N)*H], device (written)
 * Rows as in cp_attn_fwd_ring_step; cp_merge_partials over the P parts gives the
 * rank's rows of full attention. Errors: as cp_attn_fwd_ring_step;
 * CP_ERR_UNSUPPORTED for N > 255;
 * CP_ERR_INVALID_ARG for a missing pull source or arrived when pulling, and
 * for a non-NULL arrived without pull sources;
 * CP_ERR_UNSUPPORTED when pulling with N > 64; CP_ERR_ALIGNMENT for a pull
 * source not 16-byte or arrived not 4-byte aligned. A wait that runs out (2 s)
 * ends the kernel with CP_ERR_TIMEOUT in cp_attn_check.
 */
CP_API int cp_attn_fwd_ring(cp_attn_plan_t plan, int rank, const void* q, void* k_all, void* v_all,
                            const void* const* pull_k, const void* const* pull_v, int* arrived,
                            float* o_parts, float* lse_parts, cp_stream_t stream);

/* cp_attn_fwd_ring without pull sources, for a caller whose own transfer fills
 * the other ranks' slots while the launch runs: before its first read of slot
 * j != rank a unit waits until arrived[j] >= 1 (slot j complete, stores visible
 * at GPU scope), then reads it. The caller raises arrived[j] from outside this
 * GPU's SMs (a peer's stores, the host through mapped memory), not by a copy
 * that needs them: the persistent kernel holds every SM. arrived is not reset
 * here. Same page and section as cp_attn_fwd_ring; same arguments without
 * pull_k / pull_v.
 *   arrived : int32 [N] device, 4-byte aligned, required (CP_ERR_INVALID_ARG
 *             when NULL)
 * A wait that runs out (2 s) ends the kernel with CP_ERR_TIMEOUT in
 * cp_attn_check; the context stays usable. */
CP_API int cp_attn_fwd_ring_external(cp_attn_plan_t plan, int rank, const void* q, void* k_all, void* v_all,
                                     int* arrived, float* o_parts, float* lse_parts, cp_stream_t stream);

/* Number of partials cp_attn_fwd_ring writes (N for N <= 3, else ceil(N/2) + 1),
 * or a negative status (CP_ERR_UNSUPPORTED for Ulysses). */
CP_API int cp_attn_ring_num_parts(cp_attn_plan_t plan);

/* Builds (and, with a device, uploads) the per-step schedules of one rank's ring
 * steps and of its one-launch forward. Idempotent. Errors: CP_ERR_INVALID_ARG, CP_ERR_UNSUPPORTED (Ulysses),
 * CP_ERR_CUDA (device allocation). */
CP_API int cp_attn_ring_prepare(cp_attn_plan_t plan, int rank);

/*
 * Host-side view of the schedule of one rank's ring step (works without a
 * device). Returns the number of items n (B*H*query-tile pairs) or a negative
 * status; when items is not NULL writes n records of five int32 (row block
 * rank*B + b, head, query-tile pair, executed key tiles of the step, CTA) in
 * run order; when cta_loads is not NULL writes each CTA's modelled load (as
 * cp_attn_plan_cta_loads counts it; min(n, SM count) CTAs). step = -1 gives
 * the units of cp_attn_fwd_ring with the query-tile pair field holding
 * pair | (first step << 16) | (end step << 24) and the key-tile field the
 * unit's total over its steps.
 */
CP_API int64_t cp_attn_ring_schedule(cp_attn_plan_t plan, int rank, int step, int32_t* items,
                                     int64_t* cta_loads);

/*
 * Plumbing of the multi-GPU ring (one process per GPU). A rank's slot buffer is
 * allocated with cp_ring_buffer_alloc so that the other ranks' processes can map
 * it: cp_ipc_get_handle writes the allocation's handle (cp_ipc_handle_bytes()
 * bytes, host memory) for another process to pass to cp_ipc_open_handle, which
 * returns a device pointer to the peer's memory, valid in this process until
 * cp_ipc_close_handle (the pointer cp_attn_fwd_ring's copy warps read from).
 * cp_copy_async enqueues one cudaMemcpyAsync of `bytes` between device pointers
 * (a peer's included) on `stream`; it does not wait for the peer, so the caller
 * orders it against the peer's writes and reads. Such a copy can need SM time:
 * one issued on a side stream did not progress while a persistent kernel held
 * every SM, so no kernel may wait for it.
 * Errors: CP_ERR_INVALID_ARG (null pointer, zero-byte allocation), CP_ERR_CUDA.
 */
CP_API int cp_ring_buffer_alloc(size_t bytes, void** out);
CP_API int cp_ring_buffer_free(void* p);
CP_API int cp_ipc_handle_bytes(void);
CP_API int cp_ipc_get_handle(const void* base, void* handle_out);
CP_API int cp_ipc_open_handle(const void* handle, void** base_out);
CP_API int cp_ipc_close_handle(void* base);
CP_API int cp_copy_async(void* dst, const void* src, size_t bytes, cp_stream_t stream);

/*
 * Backward pass: dQ, dK, dV from the forward's saved O and lse. The pages train
 * long-context models but print no backward; it is the chain rule of the
 * forward's softmax attention (page "Tensor并行与算子拆分", section
 * "注意力的并行化优化"), per (batch, head), with the same global-position causal
 * mask and ring walk as the forward:
 *   P = exp(scale Q K^T - lse), dV = P^T dO, dP = dO V^T, Dr = rowsum(dO * O),
 *   dS = P * (dP - Dr), dQ = scale dS K, dK = scale dS^T Q.
 *
 * q, k, v, o, dout, dq, dk, dv: bf16 device memory in the plan's attention input
 * layout (zigzag or contiguous rank-major [N][B][S/N][H][D]; o as cp_attn_fwd
 * wrote it); lse: fp32 [B][H][S] natural, as cp_attn_fwd wrote it. workspace:
 * device memory of cp_attn_bwd_workspace_bytes(plan) bytes (per-row lse and
 * rowsum(dO * O), caller-owned, overwritten). Three kernels are enqueued on
 * `stream` (row statistics, dK/dV per key tile, dQ per query tile); nothing is
 * allocated and nothing synchronises; results are deterministic (no atomics).
 * Errors: CP_ERR_INVALID_ARG (null argument), CP_ERR_UNSUPPORTED (Ulysses
 * layout, or S/N not a multiple of 4), CP_ERR_ALIGNMENT (a pointer not 16-byte
 * aligned), CP_ERR_CUDA (no device / launch failure); a bounded in-kernel wait
 * that runs out is reported by cp_attn_check as CP_ERR_TIMEOUT.
 */
CP_API int cp_attn_bwd(cp_attn_plan_t plan, const void* q, const void* k, const void* v, const void* o,
                       const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                       cp_stream_t stream);

/*
 * The sequence-parallel step after a tensor-parallel region (Megatron-style
 * sequence parallelism), for N virtual ranks on one GPU. Page "序列并行：超长序列
 * 训练" (guijiagi.com), the MegatronSP example: a reduce-scatter along the sequence
 * returns each rank its shard of the summed partial outputs, dropout is applied
 * and the residual added locally, LayerNorm is per token (no communication);
 * the 5688vip.com page's sequence_parallel_ln_dropout fixes the LayerNorm
 * (population variance, eps inside the square root, gamma * x_norm + beta) and
 * training-mode dropout (kept values divided by 1 - p). One fused pass:
 *   z = keep ? (sum_r partials[r]) / (1 - p) : 0  (+ residual),   y = LayerNorm(z).
 * On one GPU the ranks' shards are the contiguous row chunks of one buffer, so
 * the all-gather of the shards is the buffer itself.
 *
 * partials: bf16 [nparts][rows][H] (rank r's partial sum at offset r*rows*H);
 * keep_bits: dropout keep mask, ceil(rows*H/32) uint32 words, bit (i % 32) of
 *   word i / 32 for flat element i = row*H + h (a host-generated random draw), or
 *   NULL for no dropout;
 *   p: the drop rate, 0 <= p < 1;
 * residual: bf16 [rows][H] or NULL; gamma, beta: fp32 [H], both or neither;
 *   eps > 0 when y_out is written;
 * z_out, y_out: bf16 [rows][H] outputs, either may be NULL (not both; y_out needs
 *   gamma). All device memory, caller-owned, 16-byte aligned (keep_bits 4-byte).
 * 8 <= H <= 8192, H % 8 == 0 (CP_ERR_UNSUPPORTED otherwise); bad arguments give
 * CP_ERR_INVALID_ARG, misalignment CP_ERR_ALIGNMENT. Enqueued on `stream`.
 */
CP_API int cp_sp_rs_dropout_add_ln(const void* partials, int nparts, int64_t rows, int H, const uint32_t* keep_bits,
                                   float p, const void* residual, const float* gamma, const float* beta, float eps,
                                   void* z_out, void* y_out, cp_stream_t stream);

/* Workspace bytes of cp_attn_bwd (0 for a Ulysses plan, which has no backward). */
CP_API size_t cp_attn_bwd_workspace_bytes(cp_attn_plan_t plan);

/*
 * Walk lengths of the backward schedule, per (batch, head): *kv_pairs = the
 * (key tile, query tile) pairs the dK/dV kernel visits, *q_pairs = the (query
 * tile, key tile) pairs the dQ kernel visits (either may be NULL). Both equal
 * the executed tile pairs of the forward. Returns *q_pairs, or a negative status
 * (CP_ERR_UNSUPPORTED for Ulysses).
 */
CP_API int64_t cp_attn_plan_bwd_pairs(cp_attn_plan_t plan, int64_t* kv_pairs, int64_t* q_pairs);

/*
 * Merge num_parts partials per row (same section: online-softmax merge):
 *   M = max_t lse_t, lse = M + ln sum_t exp(lse_t - M), O = sum_t exp(lse_t - lse) O_t.
 * Partials with lse_t = -inf contribute nothing; rows whose partials are all
 * -inf give O = 0 and lse = -inf.
 *   o_parts   : float32 [num_parts][rows][D], device
 *   lse_parts : float32 [num_parts][rows], device
 *   o_out     : bf16 [rows][D], device (written, round-to-nearest-even)
 *   lse_out   : float32 [rows], device (written); may be NULL
 * D must be 64 or 128; 1 <= num_parts <= 64.
 */
CP_API int cp_merge_partials(int num_parts, int64_t rows, int D, const float* o_parts,
                      const float* lse_parts, void* o_out, float* lse_out,
                      cp_stream_t stream);

/*
 * Layout permutation (the all-to-all of the pages done as an index-mapped copy
 * on one GPU; page "4. 序列并行" (5688vip.com) simulates it the same way, by
 * index mapping). Elements are opaque: elem_bytes is 2 or 4.
 *   contiguous/zigzag: direction 0 = natural [B][S][H][D] -> rank-major,
 *                      direction 1 = rank-major -> natural.
 *   Ulysses:           direction 0 = shards [N][B][S/N][H][D] -> groups [N][B][S][H/N][D],
 *                      direction 1 = groups -> shards.
 * in/out: device, B*S*H*D*elem_bytes bytes each, must not overlap. Bit-exact copy.
 */
CP_API int cp_layout_permute(cp_attn_plan_t plan, int direction, const void* in, void* out,
                      int elem_bytes, cp_stream_t stream);

/*
 * Rotary position embedding at GLOBAL positions, fused into the forward layout
 * map. Page "序列与上下文并行" (ai-infra-wiki), section "工程实践": under context
 * parallelism position encodings are computed at each token's global position
 * (each rank must know its segment's global offset). Reading: feature pair
 * (2i, 2i+1) of every head of the token at global position p is rotated by the
 * angle p * theta_i, theta_i = base^(-2i/D) — the frequencies of the pages'
 * sinusoidal PositionalEncoding (page "Tensor并行与算子拆分"); base 10000 there:
 *   out[2i]   = in[2i] cos - in[2i+1] sin,   out[2i+1] = in[2i] sin + in[2i+1] cos.
 *
 * in:  bf16 device memory in the natural layout [B][S][H][D] (contiguous and
 *      zigzag plans) or the Ulysses sequence shards [N][B][S/N][H][D]; the global
 *      position of a token is its natural index s (shard rho, local sl: rho*S/N + sl)
 *      plus pos_offset (the position of token 0, e.g. after a cached prefix).
 * out: bf16 device memory in the plan's attention input layout, exactly what
 *      cp_layout_permute(plan, 0, in, out, 2) writes, with every head rotated:
 *      zigzag/contiguous rank-major [N][B][S/N][H][D]; for Ulysses the head
 *      groups [N][B][S][H/N][D] that cp_attn_fwd builds internally.
 * base > 1 (10000 for the pages' frequencies); 0 <= pos_offset <= 2^31 - S.
 * The angle is reduced to [-pi, pi] in fp64, then rotated in fp32; one bf16
 * rounding per output element. Enqueued on `stream`; `in` and `out` must not
 * overlap; both 16-byte aligned (CP_ERR_ALIGNMENT); bad arguments give
 * CP_ERR_INVALID_ARG; D must be 64 or 128 (CP_ERR_UNSUPPORTED).
 */
CP_API int cp_rope_permute(cp_attn_plan_t plan, const void* in, void* out, double base, int64_t pos_offset,
                           cp_stream_t stream);

/* Length of the index map written by cp_layout_index_map: B*S for
 * contiguous/zigzag (one entry per token), N*B*S for Ulysses (one entry per
 * (group, batch, token) run of H/N heads). */
CP_API int64_t cp_layout_index_map_len(cp_attn_plan_t plan);

/*
 * Write the layout's int64 index map (device, cp_layout_index_map_len entries):
 *   contiguous/zigzag: map[(r*B + b)*(S/N) + tl] = natural flat token b*S + pos,
 *                      pos = the global position of rank r's local token tl;
 *   Ulysses: map[(g*B + b)*S + s] = ((rho*B + b)*(S/N) + s mod (S/N))*N + g,
 *            rho = s div (S/N): the run of the shards tensor (viewed as runs of
 *            H/N heads) that lands at group g, batch b, token s.
 * Direction-0 permutation is out[i] = in[map[i]] over rows/runs.
 */
CP_API int cp_layout_index_map(cp_attn_plan_t plan, int64_t* map_out, cp_stream_t stream);

/*
 * Synchronise `stream`, then report the first error recorded since the last
 * check: CP_ERR_TIMEOUT if a bounded in-kernel wait ran out (the status word is
 * then cleared), CP_ERR_CUDA on an asynchronous CUDA error, else CP_OK.
 */
CP_API int cp_attn_check(cp_attn_plan_t plan, cp_stream_t stream);

/* Static, human-readable text for a status code. */
CP_API const char* cp_status_string(int status);

/*
 * Fault-detection self-test of the bounded wait used by every kernel: launches
 * one CTA that waits on a shared-memory barrier that nothing ever arrives on,
 * with a limit of timeout_us microseconds, then records the outcome in the
 * plan's status word and returns. The host sees it through cp_attn_check
 * (expected: CP_ERR_TIMEOUT). No fault, trap or unbounded spin is involved.
 * 1 <= timeout_us <= 1000000.
 */
CP_API int cp_debug_wait_timeout_probe(cp_attn_plan_t plan, int timeout_us, cp_stream_t stream);

/*
 * Ulysses forward that allocates nothing (no counterpart on the pages: this is
 * an interface convenience of this library, not part of the method).
 *
 * Who needs it: callers that must not call cudaMalloc at the point of the
 * call -- code whose device memory is owned by another allocator (a framework
 * caching allocator that would otherwise have to hand out a multi-megabyte
 * workspace), code that runs where allocation is forbidden or would
 * synchronise the device (a latency-critical loop), or code that simply has
 * no way to obtain a workspace buffer. cp_attn_fwd's Ulysses path needs
 * 4*B*S*H*D*2 bytes of workspace for the head-group copies of Q, K, V and O;
 * this variant takes them from a fixed scratch array that the library holds
 * in device memory instead.
 *
 * Same arguments and results as cp_attn_fwd for a CP_LAYOUT_ULYSSES plan,
 * minus the workspace: q, k, v, o are sequence shards [N][B][S/N][H][D] bf16,
 * lse is float32 [B][H][S] (may be NULL); the plan itself must have been
 * created beforehand (cp_attn_plan allocates its small work-list table once).
 *
 * Limits and behaviour:
 *   - The scratch is a static device array of CP_NOALLOC_SCRATCH_BYTES
 *     (32 MiB). Every GPU on which the library's kernels are loaded holds it
 *     until the process exits. Plans needing more (4*B*S*H*D*2 bytes) are
 *     rejected with CP_ERR_WORKSPACE before anything is launched; plans of
 *     another layout with CP_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it; make
 *     that first call before any stream capture on that device.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents. Nothing in it has to start at zero: each call writes every
 *     byte it reads. Two calls whose work can overlap on the GPU (different
 *     streams without ordering, or different host threads) race on it:
 *     serialise them.
 *   - The current device must be the one the plan was made on, and `stream`
 *     must belong to it: the scratch used is the current device's, the work
 *     list and status word are the plan's. A call made with another device
 *     current returns CP_ERR_INVALID_ARG and launches nothing.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define CP_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
CP_API int cp_attn_fwd_ulysses_noalloc(cp_attn_plan_t plan, const void* q, const void* k, const void* v,
                                       void* o, float* lse, cp_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* CP_ATTN_H_ */
