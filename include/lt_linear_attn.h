/*
 * lt_linear_attn.h -- C ABI of the B200 (sm_100a) kernelised linear
 * attention library (liblt.so).
 *
 * The operation (lineartile 1.0.0, PyPI page, sections "How It Works" and
 * "Reference"; the causal normalised form is the linear attention of
 * Katharopoulos et al. 2020 that the page cites):
 *
 *     phi(x) = ELU(x) + 1           (alpha = 1: x + 1 for x > 0, e^x else)
 *     causal:      O_i = phi(Q_i) S_i / (phi(Q_i) . z_i + eps),
 *                  S_i = sum_{j<=i} phi(K_j)^T V_j,  z_i = sum_{j<=i} phi(K_j)
 *     non-causal:  the same with S and z summed over the whole sequence,
 *                  i.e. phi(Q)(phi(K)^T V) ("compute K^T V first")
 *                  normalised row by row with phi(Q_i) . z + eps.
 *
 * No 1/sqrt(d) score scale is applied inside the operation; callers that
 * want one scale Q (or K) beforehand.  eps is added to the denominator only.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc / cudaMallocAsync
 *     / managed memory) owned by the caller; the library keeps no reference
 *     to them after the call returns.
 *   - Scratch memory: lt_linear_attn_fwd with LT_BF16 on a dense batch cuts
 *     each sequence into blocks and, when there is more than one, allocates
 *     a stream-ordered workspace on `stream` (cudaMallocAsync, released by
 *     cudaFreeAsync on the same stream before the call returns) for the
 *     per-block partial states; lt_linear_attn_fwd_plan() gives its size.
 *     lt_linear_attn_fwd_state and lt_linear_attn_state with LT_BF16
 *     allocate the same way (always); lt_linear_attn_bwd allocates its
 *     workspace the same way.  No other entry point allocates.
 *   - Layouts are token-major and dense (row-major, no padding):
 *       dense:   q [B][N][H_q][d],  k [B][N][H_kv][d],  v [B][N][H_kv][dv],
 *                out [B][N][H_q][dv]
 *       packed:  the same without the B dimension, [N][H][.], where
 *                N = total tokens = cu_seqlens[B].
 *   - Grouped-query attention: query head h reads KV head
 *     floor(h * H_kv / H_q), i.e. contiguous groups of G = H_q / H_kv.
 *   - Work is enqueued on `stream` and the call returns without waiting
 *     (asynchronous).  Results are valid once the stream reaches the work.
 *   - Argument errors are detected on the host before anything is
 *     enqueued; in that case nothing is written and nothing is launched.
 *   - Errors found by a kernel (an inconsistent cu_seqlens array, a stalled
 *     pipeline) are recorded in a per-device error word and reported by
 *     lt_get_last_device_error().
 *   - The caller must ensure that output buffers do not overlap inputs.
 */
#ifndef LT_LINEAR_ATTN_H
#define LT_LINEAR_ATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LT_API __attribute__((visibility("default")))
#else
#define LT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as the CUDA runtime's cudaStream_t (NULL = legacy default). */
typedef struct CUstream_st *lt_stream_t;

typedef enum {
  LT_OK = 0,
  LT_ERR_INVALID_ARG = 1,     /* null/misaligned/host pointer, bad size or eps */
  LT_ERR_UNSUPPORTED = 2,     /* d or dv not in {64, 128}, unknown dtype */
  LT_ERR_CUDA = 3,            /* a CUDA runtime call or launch failed */
  LT_ERR_DEVICE_TIMEOUT = 4,  /* a kernel gave up on a stalled wait */
  LT_ERR_DEVICE_BAD_SEQLENS = 5, /* a kernel found cu_seqlens inconsistent */
  LT_ERR_SCRATCH_TOO_SMALL = 6   /* lt_linear_attn_fwd_noalloc: the shape needs
                                    more than LT_NOALLOC_SCRATCH_BYTES */
} lt_status_t;

typedef enum {
  LT_F32 = 0,  /* fp32 inputs/outputs, fp32 FMA arithmetic */
  LT_BF16 = 1, /* bf16 inputs/outputs, tensor cores, fp32 accumulation */
  LT_F16 = 2   /* fp16 inputs/outputs, tensor cores on bf16 operands, fp32
                  accumulation; lt_linear_attn_fwd and lt_linear_attn_fwd_ex
                  only, d = dv = 64 or 128 */
} lt_dtype_t;

/* Feature maps phi of lt_linear_attn_fwd_ex (applied elementwise to Q and K). */
typedef enum {
  LT_PHI_ELU1 = 0, /* ELU(x) + 1 (alpha = 1): the method's map, the default */
  LT_PHI_RELU = 1, /* max(x, 0) */
  LT_PHI_EXP = 2   /* e^x */
} lt_feature_map_t;

/*
 * Forward pass of (causal or non-causal) linear attention.
 *
 * q, k, v   inputs of element type `dtype`, layouts above; 16-byte aligned.
 * out       output, same element type, layout [.][N][H_q][dv]; 16-byte
 *           aligned; must not overlap q, k or v.
 * B         dense: batch rows; packed: number of sequences.  1 <= B <= 65535.
 * H_q, H_kv query and KV heads, 1 <= H_kv <= 65535, H_q a multiple of H_kv.
 * N         dense: tokens per row; packed: total tokens.  N >= 1 and the
 *           total token count (B*N dense, N packed) below 2^31.
 * d, dv     key and value widths, each 64 or 128.
 * causal    1: prefix sums j <= i (diagonal included); 0: whole sequence.
 * eps       denominator offset, finite and >= 0 (1e-6 is typical).
 * cu_seqlens NULL for dense inputs; else a DEVICE int32 array of B+1
 *           non-decreasing offsets with cu_seqlens[0] = 0 and
 *           cu_seqlens[B] = N; sequence s is tokens [cu[s], cu[s+1]).
 *           Empty sequences are allowed.  An inconsistent array is skipped
 *           by the kernel and reported by lt_get_last_device_error().
 * stream    CUDA stream to enqueue on.
 * dtype     LT_BF16 (tensor-core path), LT_F16 (fp16 I/O on the same
 *           tensor-core path with bf16 operands; d = dv = 64 or 128) or
 *           LT_F32 (fp32 FMA path).
 *
 * Evaluation (bf16): chunks of 128 tokens; the intra-chunk part as masked
 * dense products and the inter-chunk part through the carried state
 * ("Why Stream Wins at Ultra-Long Context", section 5.3: chunk-local work
 * plus a carry).  A dense sequence is cut into blocks of consecutive chunks
 * so that every SM has work, and each block starts from the sum of the
 * earlier blocks' partial states.  Short blocks (d = dv = 64, at most four
 * chunks, every block resident at once) run as ONE cooperative launch whose
 * blocks exchange their partial states through the workspace; otherwise one
 * launch writes each block's partial state and a second runs the blocks
 * from the carry.  lt_linear_attn_fwd_plan tells which.
 *
 * Returns LT_OK when the work was enqueued.
 */
LT_API lt_status_t lt_linear_attn_fwd(const void *q, const void *k, const void *v, void *out,
                               int B, int H_q, int H_kv, int N, int d, int dv, int causal,
                               float eps, const int32_t *cu_seqlens, lt_stream_t stream,
                               lt_dtype_t dtype);

/*
 * lt_linear_attn_fwd_ex: lt_linear_attn_fwd with another feature map phi
 * (the lineartile page, "Features": "Replace phi kernel freely").  The
 * library's kernels take the map as a compile-time functor of their tile
 * transform, so a map is one small device function; the maps compiled in are
 * lt_feature_map_t.  Same arguments, layouts and results as
 * lt_linear_attn_fwd otherwise; with LT_PHI_ELU1 it IS lt_linear_attn_fwd.
 * Every phi here is >= 0, so the denominator stays >= eps (ReLU can make a
 * row's scores all zero: its output is then 0).
 *
 * Other maps and LT_F16 run the general kernel (the state launch plus the
 * forward launch) and support d = dv = 64 or 128 (LT_ERR_UNSUPPORTED
 * otherwise); LT_F32 supports every map and width pair.
 * Returns as lt_linear_attn_fwd; LT_ERR_INVALID_ARG for an unknown phi.
 */
LT_API lt_status_t lt_linear_attn_fwd_ex(const void *q, const void *k, const void *v, void *out,
                                         int B, int H_q, int H_kv, int N, int d, int dv,
                                         int causal, float eps, const int32_t *cu_seqlens,
                                         lt_stream_t stream, lt_dtype_t dtype,
                                         lt_feature_map_t phi);

/*
 * lt_linear_attn_fwd_window: sliding-window causal linear attention (the
 * lineartile page, "Features": sliding window attention).  Row i attends to
 * the `window` most recent keys, i - window < j <= i:
 *     O_i = phi(Q_i)(S_i - S_{i-w}) / (phi(Q_i).(z_i - z_{i-w}) + eps),
 * S_m = z_m = 0 for m < 0; window >= N is the causal form.
 *
 * q .. cu_seqlens, stream   as for lt_linear_attn_fwd (causal only).
 * window     >= 1 tokens.
 * dtype      LT_F32, LT_BF16 or LT_F16 (fp32 arithmetic for all three;
 *            outputs rounded once to the input's type).
 * Evaluation: 32-token chunks, one CTA per (sequence, query head); each
 * row's window split into a window state carried from chunk to chunk
 * (holding only the window's keys, never a difference of long prefix sums)
 * and two band-masked tiles.  No scratch memory.
 * Returns as lt_linear_attn_fwd; LT_ERR_INVALID_ARG for window < 1.
 */
LT_API lt_status_t lt_linear_attn_fwd_window(const void *q, const void *k, const void *v,
                                             void *out, int B, int H_q, int H_kv, int N, int d,
                                             int dv, int window, float eps,
                                             const int32_t *cu_seqlens, lt_stream_t stream,
                                             lt_dtype_t dtype);

/*
 * lt_linear_attn_fwd_noalloc: the bf16 forward pass of lt_linear_attn_fwd
 * (same arguments, dtype fixed to LT_BF16, same kernels and results) for
 * callers that cannot let a library allocate device memory.  The method has
 * no counterpart; it exists for integration only.
 *
 * Who needs it: lt_linear_attn_fwd takes a stream-ordered workspace
 * (cudaMallocAsync) for the per-block partial states.  A program that hands
 * all device memory to its own caching allocator at start-up, a set-up
 * without stream-ordered allocation (memory pools unsupported), or code that
 * must keep a fixed memory footprint with no allocator work in its launch
 * path cannot accept that.  This call allocates nothing: the workspace is a
 * fixed array of LT_NOALLOC_SCRATCH_BYTES inside the library, which every
 * device that loads the library holds until the process exits.  16 MiB
 * covers every shape at the default block count on a GPU with up to 254 SMs
 * (at most one partial state of d*dv + d floats per SM).
 *
 * Set-up: the first call on a device (with that device current) looks up
 * the array's device address with cudaGetSymbolAddress; make that first
 * call before any stream capture.
 *
 * Sharing: all calls on a device use the same array.  Calls whose work can
 * overlap on the GPU (unordered streams, concurrent host threads) race on it
 * and may return wrong results: order them.  Nothing in the array needs to
 * start at zero; each call writes every partial state it later reads.
 *
 * Returns LT_ERR_UNSUPPORTED, LT_ERR_INVALID_ARG, LT_ERR_CUDA as
 * lt_linear_attn_fwd does; LT_ERR_SCRATCH_TOO_SMALL (nothing enqueued) when
 * the shape's workspace (lt_linear_attn_fwd_plan) exceeds the array.
 */
#define LT_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
LT_API lt_status_t lt_linear_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                              void *out, int B, int H_q, int H_kv, int N,
                                              int d, int dv, int causal, float eps,
                                              const int32_t *cu_seqlens, lt_stream_t stream);

/*
 * How lt_linear_attn_fwd evaluates a shape: blocks each sequence is cut
 * into, kernel launches per call, and bytes of stream-ordered workspace the
 * call allocates (0: none).  Host-only arithmetic, nothing is launched.
 *
 * B .. causal, dtype   as for lt_linear_attn_fwd.
 * packed               1 when cu_seqlens will be passed (packed sequences
 *                      run one block each), 0 for dense inputs.
 * num_sms              SM count of the target device; <= 0 queries the
 *                      current device (needs a working CUDA runtime).
 * blocks, launches, workspace_bytes   outputs (non-NULL host pointers).
 * Returns LT_OK, LT_ERR_INVALID_ARG / LT_ERR_UNSUPPORTED for arguments that
 * lt_linear_attn_fwd would reject, LT_ERR_CUDA if the device query failed.
 */
LT_API lt_status_t lt_linear_attn_fwd_plan(int B, int H_q, int H_kv, int N, int d, int dv,
                                           int causal, int packed, lt_dtype_t dtype,
                                           int num_sms, int *blocks, int *launches,
                                           size_t *workspace_bytes);

/*
 * lt_linear_attn_fwd_state: the forward pass of lt_linear_attn_fwd continued
 * from a given state and/or returning the final state (prefill -> decode
 * handoff, a long sequence processed in pieces).  For linear attention the
 * KV cache is the fixed-size state (lineartile page, "Features": KV-cache
 * reuse; the recurrent view of the cited linear attention).
 *
 * With (S0, z0), sequence s starts from the state of its KV heads:
 *     causal:     O_i = phi(Q_i)(S0 + S_i) / (phi(Q_i) . (z0 + z_i) + eps)
 *     non-causal: the same with S_i, z_i summed over the whole sequence.
 * (S_out, z_out) receive S0 + (the sum over the whole sequence): the state
 * after the sequence's last token.  Cutting a sequence anywhere and passing
 * the first call's (S_out, z_out) as the second call's (S0, z0) reproduces
 * the uncut outputs; (S_out, z_out) can seed lt_linear_attn_decode_step.
 *
 * q .. cu_seqlens, stream, dtype   as for lt_linear_attn_fwd.
 * S0     [B][H_kv][d][dv] fp32 device (16-byte aligned), or NULL: zero.
 * z0     [B][H_kv][d] fp32 device, NULL exactly when S0 is.
 * S_out  [B][H_kv][d][dv] fp32 device (16-byte aligned), or NULL: not returned.
 * z_out  [B][H_kv][d] fp32 device, NULL exactly when S_out is.
 *        B counts sequences (packed: the cu_seqlens entries minus one); an
 *        empty sequence returns S0 (or zero).  S_out and z_out must not
 *        overlap each other or any input (no in-place update); out must not
 *        overlap S0 or z0.
 * Scratch: LT_BF16 always allocates a stream-ordered workspace (every
 * block's partial state, as lt_linear_attn_fwd; released before return).
 * Evaluation (bf16): where lt_linear_attn_fwd runs one cooperative launch,
 * so does this call: every block's starting state is S0 + (earlier blocks),
 * summed in block order, and the last block writes the final state.
 * Otherwise a state launch writes every block's partial state, a small
 * kernel turns them, in block order, into each block's starting state and
 * into the final state, and the forward launch starts every block from its
 * own.  With S0 = 0 the outputs equal lt_linear_attn_fwd's bit for bit.
 *
 * Returns as lt_linear_attn_fwd.
 */
LT_API lt_status_t lt_linear_attn_fwd_state(const void *q, const void *k, const void *v,
                                            void *out, int B, int H_q, int H_kv, int N, int d,
                                            int dv, int causal, float eps,
                                            const int32_t *cu_seqlens, const float *S0,
                                            const float *z0, float *S_out, float *z_out,
                                            lt_stream_t stream, lt_dtype_t dtype);

/*
 * lt_linear_attn_state: the final state of every (sequence, KV head) without
 * the outputs -- for linear attention the whole past of a sequence is this
 * fixed-size state (lineartile page, "Reference": the recurrent view;
 * "Features": KV-cache reuse).  For sequence s and KV head g:
 *     S_out = S0 + sum_t phi(K_t)^T V_t,   z_out = z0 + sum_t phi(K_t)
 * over the sequence's tokens.  It reads only K and V: a prefill that needs
 * just the state, or one segment's contribution when a sequence is cut into
 * segments across devices (context parallelism, with
 * lt_linear_attn_state_carry).
 *
 * k, v       as for lt_linear_attn_fwd (element type dtype, 16-byte aligned).
 * B, H_kv, N, d, dv, cu_seqlens, stream, dtype   as for lt_linear_attn_fwd.
 * S0, z0     [B][H_kv][d][dv] and [B][H_kv][d] fp32 device, or both NULL (zero).
 * S_out, z_out  the same shapes, fp32 device (S_out 16-byte aligned); they
 *            must not overlap the inputs or each other.
 * Evaluation: bf16 as the first launch of the block-parallel forward pass
 * (every block's partial state on the tensor cores, in a stream-ordered
 * workspace released before return) plus a summation in block order; fp32
 * with FMA arithmetic, one CTA per (sequence, KV head).
 * Returns as lt_linear_attn_fwd.
 */
LT_API lt_status_t lt_linear_attn_state(const void *k, const void *v, int B, int H_kv, int N,
                                        int d, int dv, const int32_t *cu_seqlens,
                                        const float *S0, const float *z0, float *S_out,
                                        float *z_out, lt_stream_t stream, lt_dtype_t dtype);

/*
 * lt_linear_attn_state_carry: the starting state of segment `rank` when every
 * sequence of a batch is cut into `world` contiguous segments in rank order
 * (context parallelism, lineartile page "Features": multi-GPU sharding; the
 * inter-segment carry of "Why Stream Wins at Ultra-Long Context", section
 * 5.3, across devices).  From the states of every segment computed from zero
 * (lt_linear_attn_state, gathered from the ranks):
 *     causal:     S_out = sum_{r < rank} S_all[r]   (z likewise)
 *     non-causal: S_out = sum_{r != rank} S_all[r]
 * summed in fp32 in rank order, so every rank and every run gets the same
 * bits.  Passing (S_out, z_out) as (S0, z0) of lt_linear_attn_fwd_state over
 * the rank's segment gives that segment's outputs of attention over the whole
 * sequence.
 *
 * S_all  [world][B][H_kv][d][dv] fp32 device;  z_all  [world][B][H_kv][d].
 * world >= 1, 0 <= rank < world, causal 0 or 1, d and dv 64 or 128.
 * S_out  [B][H_kv][d][dv], z_out [B][H_kv][d] fp32 device; no overlaps.
 * Returns LT_OK, LT_ERR_INVALID_ARG, LT_ERR_UNSUPPORTED or LT_ERR_CUDA.
 */
LT_API lt_status_t lt_linear_attn_state_carry(const float *S_all, const float *z_all, int world,
                                              int rank, int causal, int B, int H_kv, int d,
                                              int dv, float *S_out, float *z_out,
                                              lt_stream_t stream);

/*
 * lt_linear_attn_bwd: backward pass of lt_linear_attn_fwd.  For an upstream
 * gradient dout = dL/dO it returns dq = dL/dQ, dk = dL/dK, dv = dL/dV (the
 * lineartile page lists a backward pass, "Project Structure":
 * core/kernels/backward.py; its formulas follow from the forward definition).
 * With a_ij = phi(Q_i).phi(K_j) over the kept pairs, den_i = sum_j a_ij + eps:
 *     g_i = dout_i / den_i,  h_i = -(dout_i . O_i) / den_i,  da_ij = g_i.V_j + h_i,
 *     dQ_i = phi'(Q_i) * sum_j da_ij phi(K_j),  dK_j = phi'(K_j) * sum_i da_ij phi(Q_i),
 *     dV_j = sum_i a_ij g_i,   phi'(x) = 1 (x > 0), e^x (x <= 0);
 * a KV head's dk, dv sum over the query heads of its group.  O is recomputed.
 *
 * q, k, v, B .. cu_seqlens, stream, dtype   as for lt_linear_attn_fwd.
 * dout   the output's layout and element type; must not overlap q, k, v.
 * dq, dk, dv  q's, k's and v's layouts and element type (16-byte aligned,
 *        device); written whole; must not overlap any input or each other.
 * Evaluation: two chunked scans with fp32 FMA arithmetic (32-token chunks),
 * a forward scan for dq and a reverse scan for dk, dv ("Why Stream Wins at
 * Ultra-Long Context", section 4.2: the backward recurrence of a linear
 * scan), each sequence cut into blocks of whole chunks that run on their own
 * CTAs from carried block sums (added in block order: the results do not
 * depend on scheduling).  Scratch: a stream-ordered workspace of
 * tokens * H_q * (dv + 1) + B * (H_q + H_kv) * nb * (d * dv + d) floats (nb
 * blocks per sequence, at most four times the SM count), released before return.
 * Returns as lt_linear_attn_fwd.
 */
LT_API lt_status_t lt_linear_attn_bwd(const void *q, const void *k, const void *v,
                                      const void *dout, void *dq, void *dk, void *dv, int B,
                                      int H_q, int H_kv, int N, int d, int dv_width, int causal,
                                      float eps, const int32_t *cu_seqlens, lt_stream_t stream,
                                      lt_dtype_t dtype);

/*
 * One recurrent decode step: the fixed-size state (S, z) plays the role of
 * a KV cache (lineartile page, "KV Cache Reuse"; recurrent view of the
 * cited linear attention).  For every batch row b and KV head g:
 *     S[b][g] += phi(k[b][g])^T v[b][g];   z[b][g] += phi(k[b][g]);
 * then for every query head h of g's group:
 *     out[b][h] = phi(q[b][h]) S[b][g] / (phi(q[b][h]) . z[b][g] + eps).
 * The update comes first, so the new token attends to itself.
 *
 * q   [B][H_q][d],  k [B][H_kv][d],  v [B][H_kv][dv]   (element type dtype)
 * S   [B][H_kv][d][dv] fp32, updated in place (16-byte aligned)
 * z   [B][H_kv][d]     fp32, updated in place
 * out [B][H_q][dv]     (element type dtype); must not overlap the inputs.
 * A zero-initialised (S, z) starts a new sequence; chaining N steps gives
 * the causal forward pass row by row.
 */
LT_API lt_status_t lt_linear_attn_decode_step(const void *q, const void *k, const void *v, float *S,
                                       float *z, void *out, int B, int H_q, int H_kv, int d,
                                       int dv, float eps, lt_stream_t stream, lt_dtype_t dtype);

/*
 * Diagnostic schedule override, for tests and ablations only: makes every
 * later forward call of this process (every device, every thread) use a
 * given kernel path and/or block count instead of the one the library picks.
 * Results stay correct on every path; only the speed changes.  Not meant to
 * be changed while forward calls run on other threads.
 *
 * kernel  LT_SCHED_AUTO: the library's choice (the default);
 *         LT_SCHED_TWO_LAUNCH: the state launch plus the forward launch
 *           also where one cooperative launch would run;
 *         LT_SCHED_GENERAL: the general kernel (every width pair) also for
 *           d = dv = 64.
 * blocks  0: the library's choice; n > 0: n blocks per dense sequence (at
 *         most its chunk count).
 * Returns LT_OK, or LT_ERR_INVALID_ARG for an unknown kernel or blocks < 0.
 * The method has no counterpart.
 */
typedef enum {
  LT_SCHED_AUTO = 0,
  LT_SCHED_TWO_LAUNCH = 1,
  LT_SCHED_GENERAL = 2
} lt_schedule_t;
LT_API lt_status_t lt_debug_set_schedule(lt_schedule_t kernel, int blocks);

/*
 * Diagnostic: enqueue one small kernel whose bounded wait (the pipeline
 * wait every kernel uses) is on a barrier that nothing arrives on, so it
 * gives up after limit_us microseconds (1 .. 1000000), records a timeout and
 * returns.  lt_get_last_device_error(stream) then reports
 * LT_ERR_DEVICE_TIMEOUT and the device stays usable.  It exists to test the
 * timeout path without a GPU fault; the method has no counterpart.
 */
LT_API lt_status_t lt_selftest_wait_timeout(unsigned int limit_us, lt_stream_t stream);

/* Static, human-readable name of a status code. */
LT_API const char *lt_status_string(lt_status_t status);

/*
 * Synchronise `stream`, then read and clear the current device's error
 * word.  Returns LT_OK, LT_ERR_DEVICE_TIMEOUT, LT_ERR_DEVICE_BAD_SEQLENS,
 * or LT_ERR_CUDA if the synchronisation itself failed.
 */
LT_API lt_status_t lt_get_last_device_error(lt_stream_t stream);

/* ABI version of this header: 1. */
LT_API int lt_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LT_LINEAR_ATTN_H */
