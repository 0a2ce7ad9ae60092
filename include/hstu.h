/*
 * hstu.h -- C ABI of the jagged HSTU layer forward for NVIDIA B200 (sm_100a).
 *
 * One HSTU layer (blog "Generative Recommendation 16: HSTU", section
 * "HSTU Layer 到底改了什么", equations (1)-(3)):
 *
 *   (1)  U, V, Q, K = Split(SiLU(X W1^T + b1))            split order U, V, Q, K
 *   (2)  O_i = sum_{j visible to i} SiLU(q_i . k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j / n_norm
 *   (3)  Y = (LayerNorm(O) (.) U) W2^T + b2 + X
 *
 * per head (heads are contiguous column blocks of width head_dim), with no
 * softmax along the sequence (same blog, section "不对序列做 softmax").
 * Batches are jagged: user b owns rows seq_offsets[b] .. seq_offsets[b+1]-1
 * of every [T, *] tensor, with no padding ("Ragged/Jagged kernel" item of the
 * same blog); no query ever sees another user's keys.
 *
 * Visibility (mask_mode):
 *   HSTU_MASK_CAUSAL   key j visible to query i iff j <= i (same user).
 *   HSTU_MASK_MFALCON  the last num_candidates[b] rows of user b are ranking
 *                      candidates (ltzyclt blog on HSTU, section 5.2,
 *                      "M-FALCON"): a candidate sees the user's whole history
 *                      and itself, never another candidate; history rows are
 *                      causal and never see candidates.  Every candidate sits
 *                      at position n_h (the first position after the history),
 *                      so results do not depend on how candidates are split
 *                      into micro-batches.
 * Bias buckets (the rab^{p,t} of equation (2); the rules are fixed by the
 * layer configuration, not by the pages):
 *   p(i,j) = clamp(pos(i) - j, 0, pos_clamp), pos(i) = i for history rows and
 *            n_h for candidates (local indices inside the user);
 *   t(i,j) = min(floor(ln(1 + max(ts_i - ts_j, 0)) / time_log_div), time_buckets - 1),
 *            evaluated as that fp64 expression (the library turns it into an
 *            exact integer threshold table once, at hstu_create).
 *
 * Conventions for every entry point:
 *   - Pointers documented "device" must be device memory of the handle's GPU
 *     and 16-byte aligned; "host" pointers are ordinary host memory.
 *   - The caller owns every input, output, weight and stream.  The handle owns
 *     only its workspace (intermediates, scheduler tables, error word).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) except where stated.  A handle must not be used from two
 *     streams at once: its workspace is shared by all of its calls.
 *   - Host-detectable argument errors return a non-zero status before any
 *     launch.  Problems that only the GPU can see (non-monotone seq_offsets,
 *     seq_offsets[B] != T, num_candidates outside [0, length], timestamps that
 *     decrease inside a user or lie outside [0, 2^62)) set the handle's device
 *     error word and leave `out` undefined; hstu_get_device_error reads it.
 *   - No call traps, aborts or exits the process.
 */
#ifndef HSTU_B200_H_
#define HSTU_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,   /* a null pointer, bad size, bad enum, misaligned pointer */
  HSTU_ERR_UNSUPPORTED = 2,   /* a shape the kernels do not implement (see hstu_create) */
  HSTU_ERR_WORKSPACE = 3,     /* T or B above the max_tokens / max_users given at create */
  HSTU_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  HSTU_ERR_DEVICE_CHECK = 5,  /* the GPU found invalid offsets / candidates / timestamps */
  HSTU_ERR_TIMEOUT = 6        /* a kernel gave up a bounded wait (pipeline stall) */
} hstu_status;

typedef enum { HSTU_DTYPE_BF16 = 0, HSTU_DTYPE_FP32 = 1 } hstu_dtype;

typedef enum { HSTU_MASK_CAUSAL = 0, HSTU_MASK_MFALCON = 1 } hstu_mask_mode;

/* Device error bits reported through hstu_get_device_error. */
#define HSTU_DEVERR_OFFSETS     0x1  /* seq_offsets not monotone, [0] != 0 or [B] != T */
#define HSTU_DEVERR_CANDIDATES  0x2  /* num_candidates[b] < 0 or > length of user b */
#define HSTU_DEVERR_TIMESTAMPS  0x4  /* decreasing inside a user, or outside [0, 2^62) */
#define HSTU_DEVERR_TIMEOUT     0x8  /* a bounded pipeline wait expired */
#define HSTU_DEVERR_SL_TOO_LONG 0x10 /* Stochastic Length: a sequence to sub-sample is longer
                                        than HSTU_SL_MAX_SAMPLED_LEN (it is dropped) */

typedef struct {
  int32_t d_model;          /* d = num_heads * head_dim; BF16 compute: 128, 256, 384, 512, 768
                               or 1024; FP32 compute: also 64 */
  int32_t num_heads;
  int32_t head_dim;         /* BF16 compute: 64 or 128.  FP32 compute: 32, 64, 96 or 128 */
  hstu_dtype io_dtype;      /* dtype of X (values) and Y (out) in HBM */
  hstu_dtype compute_dtype; /* BF16: tcgen05 tensor-core path, bf16 operands, fp32 accumulate;
                               FP32: fp32 SIMT path (every product and sum in fp32) */
  int32_t n_norm;           /* > 0: fixed divisor; <= 0: the longest user of each call */
  int32_t pos_buckets;      /* rows of rab_pos; pos_clamp < pos_buckets */
  int32_t pos_clamp;        /* relative positions are clamped to [0, pos_clamp]; <= 4096 */
  int32_t time_buckets;     /* rows of rab_time; 1..256 */
  double time_log_div;      /* divisor of ln(1 + dt); > 0 */
  float ln_eps;             /* LayerNorm epsilon (biased variance) */
  int64_t max_tokens;       /* workspace sizing: largest T of any call; <= 2^30 */
  int32_t max_users;        /* workspace sizing: largest B of any call */
} hstu_config;

/* Parameters of one layer; all device pointers, caller-owned. */
typedef struct {
  const void* w1;        /* [4d, d] row-major (Linear layout), compute dtype */
  const float* b1;       /* [4d] */
  const void* w2;        /* [d, d] row-major, compute dtype */
  const float* b2;       /* [d] */
  const float* ln_gamma; /* [d] */
  const float* ln_beta;  /* [d] */
  const float* rab_pos;  /* [pos_buckets], shared by all heads */
  const float* rab_time; /* [time_buckets], shared by all heads */
} hstu_layer_weights;

typedef struct hstu_handle_s hstu_handle;

/* Validates `cfg` (host pointer), makes `device` current, allocates the
 * workspace for max_tokens / max_users and uploads the time-bucket threshold
 * table.  Synchronous.  *out receives the handle (NULL on error). */
hstu_status hstu_create(const hstu_config* cfg, int32_t device, hstu_handle** out);

/* Frees the workspace.  Synchronizes the device first.  NULL is a no-op. */
hstu_status hstu_destroy(hstu_handle* h);

/* One HSTU layer forward (equations (1)-(3) plus the residual).
 *   values         device [T, d] io_dtype, the layer input X
 *   total_tokens   T (0 <= T <= max_tokens)
 *   seq_offsets    device int32 [num_users + 1], 0 = offsets[0] <= ... <= offsets[B] = T
 *   num_users      B (0 <= B <= max_users); zero-length users are allowed
 *   timestamps     device int64 [T] seconds, non-decreasing inside each user, in [0, 2^62)
 *   weights        host pointer to device-pointer struct
 *   mask_mode      HSTU_MASK_CAUSAL or HSTU_MASK_MFALCON
 *   num_candidates device int32 [B]; required for MFALCON, ignored for CAUSAL
 *   out            device [T, d] io_dtype; may alias `values` exactly
 *   stream         cudaStream_t or NULL
 * Returns HSTU_OK once every kernel is enqueued. */
hstu_status hstu_layer_forward(hstu_handle* h, const void* values, int64_t total_tokens,
                               const int32_t* seq_offsets, int32_t num_users,
                               const int64_t* timestamps, const hstu_layer_weights* weights,
                               hstu_mask_mode mask_mode, const int32_t* num_candidates,
                               void* out, void* stream);

/* A stack of num_layers layers (blog "Generative Recommendation 16: HSTU",
 * section on the experiments: the largest configuration stacks 24 layers at
 * length 8192 and embedding 1024).  layers: host array of num_layers structs.
 * The residual stream stays in io_dtype between layers inside `out`; the
 * jagged schedule is built once for all layers.  Same arguments otherwise. */
hstu_status hstu_stack_forward(hstu_handle* h, const void* values, int64_t total_tokens,
                               const int32_t* seq_offsets, int32_t num_users,
                               const int64_t* timestamps, const hstu_layer_weights* layers,
                               int32_t num_layers, hstu_mask_mode mask_mode,
                               const int32_t* num_candidates, void* out, void* stream);

/* Human-readable name of a status.  Never NULL. */
const char* hstu_status_string(hstu_status s);

/* Synchronizes the handle's device, then returns the device error word of the
 * handle in *bits (HSTU_DEVERR_* flags; 0 = none) and clears it.  Returns
 * HSTU_ERR_DEVICE_CHECK or HSTU_ERR_TIMEOUT when bits are set, else HSTU_OK. */
hstu_status hstu_get_device_error(hstu_handle* h, int32_t* bits);

/* Host only, no GPU needed: the exact integer threshold table of the time
 * bucket rule.  out[k] (host int64 [num_buckets]) is the smallest gap dt >= 0
 * whose bucket floor(ln(1 + dt) / div) (fp64) is >= k, capped at 2^62 when no
 * gap below 2^62 reaches k; out[0] = 0.  bucket(dt) = #{k >= 1 : dt >= out[k]}. */
hstu_status hstu_time_bucket_thresholds(double time_log_div, int32_t num_buckets, int64_t* out);

/* ---- Bounded waits ----
 * Every pipeline wait of the tensor-core kernels (a TMA load landing, an MMA
 * finishing, a row group handing over its scores) gives up after a bound of
 * SM cycles; the kernel then sets HSTU_DEVERR_TIMEOUT in the handle's error
 * word, still waits (with the default bound) for the copies and MMAs it has
 * issued, frees its tensor memory and returns, so the context stays usable
 * and out is undefined.  This sets the bound for the handle's later launches
 * of the f1 / f2 GEMMs and the attention kernel; 0 restores the default of
 * 2^31 cycles (about a second).  A bound of a few cycles makes every launch
 * give up: the failure path can be exercised without a fault.
 * HSTU_ERR_INVALID_ARG for a NULL handle or a negative bound. */
hstu_status hstu_set_wait_limit(hstu_handle* h, int64_t cycles);

/* ---- Kernel timing (CUDA events on the launching stream) ----
 * When enabled, every kernel the handle launches is bracketed by a pair of
 * CUDA events recorded on the call's stream; the pairs are read back by
 * hstu_get_kernel_timing.  Kinds: 0 schedule (row facts + work order),
 * 1 fp32->bf16 cast of X, 2 f1 GEMM, 3 attention, 4 LayerNorm-gate, 5 f2 GEMM,
 * 6 candidate block of a history-cache call (row facts, order, row copies).
 * At most 4096 launches are recorded between resets. */
#define HSTU_KERNEL_KINDS 7

/* Enables (1) or disables (0) the event pairs; enabling also resets them. */
hstu_status hstu_set_kernel_timing(hstu_handle* h, int32_t enabled);

/* Synchronizes on the recorded events and returns, per kind k < HSTU_KERNEL_KINDS,
 * the summed duration in milliseconds (host double [HSTU_KERNEL_KINDS]) and the
 * number of launches (host int64 [HSTU_KERNEL_KINDS]).  Either pointer may be NULL. */
hstu_status hstu_get_kernel_timing(hstu_handle* h, double* total_ms, int64_t* launches);

/* ---- Attention without allocation ----
 * The pages have no counterpart of this entry point: it is an interface of
 * this library for callers that may not allocate device memory at call time
 * -- for instance code running inside a region where cudaMalloc is not
 * allowed, or a host framework that owns every allocation.  It runs the
 * attention step alone -- the scheduler and the fused tensor-core attention
 * kernel of the BF16 path, the same kernels that hstu_layer_forward launches --
 * with every piece of scratch (per-token row facts, pair order and cost,
 * counters, the error word, the time-bucket tables) in one fixed file-scope
 * device array of this library, about 1 MiB per device, instead of a handle's
 * workspace.  Apart from the set-up below, neither the call nor anything it
 * calls allocates host or device memory.
 *   cfg            host; uses d_model, num_heads, head_dim, n_norm, pos_buckets,
 *                  pos_clamp, time_buckets and time_log_div; compute_dtype must be
 *                  BF16 and head_dim 64 or 128 (else HSTU_ERR_UNSUPPORTED);
 *                  io_dtype, ln_eps, max_tokens and max_users are ignored
 *   uvqk           device bf16 [T, 4d]: SiLU(X W1^T + b1), columns U | V | Q | K
 *                  (only V, Q and K are read)
 *   total_tokens   T, 0 <= T <= HSTU_NOALLOC_MAX_TOKENS; larger T returns
 *                  HSTU_ERR_WORKSPACE before any launch
 *   seq_offsets, num_users, timestamps, mask_mode, num_candidates
 *                  as for hstu_layer_forward
 *   rab_pos        device fp32 [pos_buckets]
 *   rab_time       device fp32 [time_buckets]
 *   av             device fp32 [T, d]: for every row i and head, the sum over the
 *                  visible keys j of SiLU(q_i.k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j,
 *                  divided by n_norm once -- the tensor HSTU_TENSOR_AV of a layer
 *                  forward on the same U|V|Q|K
 *   device_error   device int32 or NULL: overwritten with this call's
 *                  HSTU_DEVERR_* bits (0 = none), in stream order
 *   stream         cudaStream_t or NULL
 * Set-up: the first call on a device looks up the address of the scratch
 * array there (cudaGetSymbolAddress, checked; HSTU_ERR_CUDA on failure) and
 * caches it.  With CUDA's lazy module loading that first call may also load
 * this library's device code, array included, which allocates: it is the only
 * call that can.  Make one warm-up call per device before any region where
 * allocation or stream capture is not allowed.  A device reset
 * (cudaDeviceReset) invalidates the cached address: do not call this entry
 * point on that device again in the same process.  The bucket tables are
 * rebuilt on the host when time_log_div or time_buckets changes.
 * Every call first clears the scratch that must start at zero (the counters
 * and the error word) and rewrites the tables, in stream order.
 * The scratch is one per device and process: two calls on one device whose
 * executions overlap (different streams, different host threads) race on it
 * and give undefined results, so serialise them.  The host-side caches are
 * not thread-safe either.  Calls are asynchronous on `stream`. */
#define HSTU_NOALLOC_MAX_TOKENS 65536

hstu_status hstu_attention_noalloc(const hstu_config* cfg, const void* uvqk, int64_t total_tokens,
                                   const int32_t* seq_offsets, int32_t num_users,
                                   const int64_t* timestamps, hstu_mask_mode mask_mode,
                                   const int32_t* num_candidates, const float* rab_pos,
                                   const float* rab_time, float* av, int32_t* device_error,
                                   void* stream);

/* ---- M-FALCON serving with a history cache ----
 * M-FALCON ranks a user's candidates against the user's history, and the
 * history's computation does not depend on the candidates (ltzyclt blog on
 * HSTU, section 5.2, "M-FALCON"; blog "Generative Recommendation 16", item 3:
 * the candidate-independent history computation is cached).  A cache holds,
 * for every layer of a stack, SiLU(f1(.)) of the history rows -- the keys and
 * values a candidate attends to -- plus the history timestamps and offsets.
 * hstu_cache_prefill runs the stack over the histories once (a causal batch);
 * each hstu_cache_score call then runs the stack over one micro-batch of
 * candidates only.  Candidate row outputs are those of hstu_stack_forward in
 * HSTU_MASK_MFALCON mode on the packed batch [history_b ; candidates_b] per
 * user: every candidate takes position n_h and sees the history and itself,
 * so the result of a candidate does not depend on which other candidates
 * share its call.  The n_norm of the handle must be fixed (> 0).
 * Inside a call every user's candidates are padded to a multiple of 256 rows
 * (one pair of 128-row query tiles), so counts that are multiples of 256
 * waste no work.
 * Memory of a cache: num_layers * rows_cap * 4d bf16 with
 * rows_cap = round_up(max_history_tokens, 256) + round_up(max_candidate_rows, 256),
 * plus a [round_up(max_candidate_rows, 256), d] io_dtype residual block.
 * A cache belongs to the handle it was created with and uses that handle's
 * workspace (rows_cap <= max_tokens); calls on one handle or one cache must
 * not overlap in execution (serialise them on one stream). */
typedef struct hstu_history_cache_s hstu_history_cache;

/* Allocates (and zeroes) a cache for `num_layers` layers.  Synchronous.
 *   max_history_tokens  largest T_h of any prefill (>= 0)
 *   max_candidate_rows  largest padded candidate count of any call, i.e. the sum
 *                       over users of round_up(n_c, 256); <= 2^21
 * HSTU_ERR_UNSUPPORTED: compute dtype FP32 or n_norm <= 0;
 * HSTU_ERR_WORKSPACE: rows_cap above the handle's max_tokens. */
hstu_status hstu_cache_create(hstu_handle* h, int32_t num_layers, int64_t max_history_tokens,
                              int64_t max_candidate_rows, hstu_history_cache** out);

/* Frees the cache (synchronizes its device first).  NULL is a no-op. */
hstu_status hstu_cache_destroy(hstu_history_cache* c);

/* Runs the stack over the histories (causal mode) and keeps each layer's
 * SiLU(f1(.)) of the history rows, the timestamps and the offsets.  Arguments
 * as for hstu_stack_forward with HSTU_MASK_CAUSAL; total_tokens <= the
 * cache's max_history_tokens (else HSTU_ERR_WORKSPACE); num_layers equals the
 * cache's.  `out` receives the histories' outputs (device [T_h, d] io_dtype,
 * may alias `values`).  Replaces any earlier history of the cache. */
hstu_status hstu_cache_prefill(hstu_handle* h, hstu_history_cache* c, const void* values,
                               int64_t total_tokens, const int32_t* seq_offsets,
                               int32_t num_users, const int64_t* timestamps,
                               const hstu_layer_weights* layers, int32_t num_layers, void* out,
                               void* stream);

/* Scores one micro-batch of candidates against the cached histories.
 *   values               device [T_c, d] io_dtype: the candidates' layer input,
 *                        packed by user in the prefill's user order
 *   num_candidates_host  HOST int32 [num_users of the prefill]: n_c per user
 *                        (>= 0; T_c = their sum)
 *   timestamps           device int64 [T_c] (M-FALCON: a candidate carries the
 *                        time of its user's last history action)
 *   layers, num_layers   the prefill's weights
 *   out                  device [T_c, d] io_dtype; may alias `values`
 * HSTU_ERR_INVALID_ARG before any prefill; HSTU_ERR_WORKSPACE when the padded
 * candidate rows exceed max_candidate_rows.  Asynchronous on `stream`; the
 * host array is read before the call returns.  The call's layout table and
 * pair order go to the device from one of four pinned staging slots; a slot
 * is reused only after its previous copy has finished, and the first call
 * after a prefill waits for the prefill's copy of the history offsets. */
hstu_status hstu_cache_score(hstu_handle* h, hstu_history_cache* c, const void* values,
                             const int32_t* num_candidates_host, const int64_t* timestamps,
                             const hstu_layer_weights* layers, int32_t num_layers, void* out,
                             void* stream);

/* ---- Stochastic Length on the device ----
 * Builds the sampled training batch (ltzyclt blog on HSTU, section 5.1; blog
 * "Generative Recommendation 16", item 2 "Stochastic Length"): a user's
 * sequence of n actions is kept whole with probability n_c^alpha / n^2 (capped
 * at 1), otherwise a sub-sequence of n_c actions is sampled uniformly without
 * replacement and kept in time order (alpha = 1.6, n_c = 776 keeps length 4096
 * mostly at 776).  The draws are inputs, so the result is a function of them:
 *   whole  iff  n <= n_c  or  user_uniform[b] * n^2 < n_c^alpha   (fp64, n^2
 *          exact, one rounding in the product; n_c^alpha from the host pow)
 *   else   the n_c actions with the smallest (token_keys[t], position) pairs.
 * Arguments (device pointers unless marked):
 *   seq_offsets     int32 [B + 1], 0 = offsets[0] <= ... <= offsets[B] = T
 *   num_users       B >= 0;  total_tokens  T, 0 <= T < 2^31
 *   user_uniform    fp64 [B] in [0, 1)
 *   token_keys      uint32 [T]
 *   n_c, alpha      n_c >= 1, alpha finite
 *   values          [T, row_bytes] rows to gather, or NULL (indices only);
 *                   row_bytes a positive multiple of 16, 16-byte aligned
 *   timestamps      int64 [T] or NULL
 *   out_offsets     int32 [B + 1]: offsets of the sampled batch
 *   out_index       int64 [T]: the first out_offsets[B] entries are the global
 *                   indices of the kept actions, user after user, in time order
 *   out_values      [T, row_bytes] (needed when values is not NULL): kept rows
 *   out_timestamps  int64 [T] or NULL: kept timestamps
 *   scratch         hstu_stochastic_length_scratch_bytes(T, B) bytes, 256-aligned
 *   device_error    int32 or NULL: overwritten with this call's HSTU_DEVERR_*
 *                   bits (OFFSETS for a bad offset table -- such users count as
 *                   empty; SL_TOO_LONG for a dropped sequence), in stream order
 * Allocates nothing; asynchronous on `stream`.  Sequences that are sampled must
 * not be longer than HSTU_SL_MAX_SAMPLED_LEN (the sort runs in shared memory). */
#define HSTU_SL_MAX_SAMPLED_LEN 8192

size_t hstu_stochastic_length_scratch_bytes(int64_t total_tokens, int32_t num_users);

hstu_status hstu_stochastic_length(const int32_t* seq_offsets, int32_t num_users,
                                   int64_t total_tokens, const double* user_uniform,
                                   const uint32_t* token_keys, int32_t n_c, double alpha,
                                   const void* values, int64_t row_bytes,
                                   const int64_t* timestamps, int32_t* out_offsets,
                                   int64_t* out_index, void* out_values,
                                   int64_t* out_timestamps, void* scratch,
                                   int32_t* device_error, void* stream);

/* ---- The attention step alone ----
 * Equation (2) of the layer (blog "Generative Recommendation 16: HSTU",
 * section "HSTU Layer 到底改了什么"; no softmax, section "不对序列做 softmax")
 * on U|V|Q|K the caller supplies: for every row i,
 *   av[i, h-th head] = sum over visible j of SiLU(q_i.k_j + rab_pos[p(i,j)] + rab_time[t(i,j)]) v_j / n_norm
 * with the same jagged schedule, masks, buckets and kernels as hstu_layer_forward
 * (BF16 compute: the tensor-core kernel; FP32 compute: the fp32 kernel).
 *   uvqk            device [T, 4d] compute dtype: columns U | V | Q | K (V, Q, K read)
 *   rab_pos         device fp32 [pos_buckets]
 *   rab_time        device fp32 [time_buckets]
 *   av              device fp32 [T, d] (overwritten; the tensor HSTU_TENSOR_AV of a
 *                   layer forward on the same U|V|Q|K)
 * Other arguments as for hstu_layer_forward; uses the handle's workspace (its
 * row facts and work order), so calls on one handle must not overlap.
 * Asynchronous on `stream`; device-side input errors go to the handle's error word. */
hstu_status hstu_attention_forward(hstu_handle* h, const void* uvqk, int64_t total_tokens,
                                   const int32_t* seq_offsets, int32_t num_users,
                                   const int64_t* timestamps, hstu_mask_mode mask_mode,
                                   const int32_t* num_candidates, const float* rab_pos,
                                   const float* rab_time, float* av, void* stream);

/* ---- Backward of the attention step ----
 * Gradients of sum(dO * O) for O of equation (2), computed by the handle's
 * tensor-core backward kernel: with s = q.k + rab and a = vis SiLU(s) / n_norm,
 *   dV = a^T dO,  dQ = dS K,  dK = dS^T Q,  dS = vis (dO V^T) SiLU'(s) / n_norm,
 * and every rab_pos / rab_time entry collects dS of each visible pair and head
 * reading it.  Builds the jagged schedule from the same arguments as the
 * forward.
 *   uvqk            device bf16 [T, 4d]: the forward's SiLU(X W1^T + b1)
 *   d_out           device bf16 [T, d]: dO
 *   dq, dk, dv      device fp32 [T, d] (overwritten)
 *   d_rab_pos       device fp32 [pos_buckets] (overwritten)
 *   d_rab_time      device fp32 [time_buckets] (overwritten)
 * Other arguments as for hstu_layer_forward; compute dtype BF16 only. */
hstu_status hstu_attention_backward(hstu_handle* h, const void* uvqk, const void* d_out,
                                    int64_t total_tokens, const int32_t* seq_offsets,
                                    int32_t num_users, const int64_t* timestamps,
                                    hstu_mask_mode mask_mode, const int32_t* num_candidates,
                                    const float* rab_pos, const float* rab_time, float* dq,
                                    float* dk, float* dv, float* d_rab_pos, float* d_rab_time,
                                    void* stream);

/* ---- Backward of one layer ----
 * Gradients of sum(dY * Y) for Y = hstu_layer_forward(X) (equations (1)-(3)
 * plus the residual), by the chain rule in the reverse order of the forward:
 * f2 and the residual, the gate, the LayerNorm, the attention step
 * (hstu_attention_backward's kernel), SiLU and f1.  Every product runs on the
 * tensor-core GEMM (operands transposed into K-major copies where needed);
 * H1 = X W1^T + b1 is recomputed, and the gate's statistics come from O.
 *   values          device [T, d] io_dtype: the layer input X
 *   uvqk, av        the forward's SiLU(X W1^T + b1) (bf16 [T, 4d]) and attention
 *                   output O (fp32 [T, d]) for the same X (hstu_copy_intermediate
 *                   after hstu_layer_forward)
 *   d_out           device [T, d] io_dtype: dY
 *   d_values        device [T, d] io_dtype: dX (may alias d_out)
 *   grads           host pointer to device pointers, all fp32, overwritten:
 *                   w1 [4d, d], b1 [4d], w2 [d, d], b2 [d], ln_gamma [d],
 *                   ln_beta [d], rab_pos [pos_buckets], rab_time [time_buckets]
 * The first call allocates the handle's backward buffers (about 68 d bytes
 * per max_tokens row, plus the transposed weights); compute dtype BF16 only. */
typedef struct {
  float* w1;
  float* b1;
  float* w2;
  float* b2;
  float* ln_gamma;
  float* ln_beta;
  float* rab_pos;
  float* rab_time;
} hstu_layer_grads;

hstu_status hstu_layer_backward(hstu_handle* h, const void* values, const void* uvqk,
                                const float* av, const void* d_out, int64_t total_tokens,
                                const int32_t* seq_offsets, int32_t num_users,
                                const int64_t* timestamps, const hstu_layer_weights* weights,
                                hstu_mask_mode mask_mode, const int32_t* num_candidates,
                                void* d_values, const hstu_layer_grads* grads, void* stream);

/* ---- Inspection entry points for tests (same library, same kernels) ---- */

typedef enum {
  HSTU_TENSOR_UVQK = 0,  /* [T, 4d] compute dtype: SiLU(f1(X)), columns U | V | Q | K */
  HSTU_TENSOR_AV = 1,    /* [T, d] fp32: the attention output O of equation (2) */
  HSTU_TENSOR_G = 2      /* [T, d] compute dtype: LayerNorm(O) (.) U */
} hstu_tensor;

/* Copies (device to device, async on `stream`) the first `bytes` of an
 * intermediate of the handle's most recent forward into caller memory `dst`.
 * For a stack, the intermediates are those of its last layer. */
hstu_status hstu_copy_intermediate(hstu_handle* h, hstu_tensor which, void* dst, size_t bytes,
                                   void* stream);

/* Runs the attention kernel of the BF16 path in its recording variant on the
 * handle's current Q/K/V workspace (zeroed first) and writes, for every
 * (query i, key j) pair the kernel visits, its position bucket, time bucket
 * and visibility into dense host-sized device arrays [T, T]: pidx_out and
 * tidx_out int32, vis_out uint8.  Pairs the kernel never visits (tiles it
 * skips) keep the caller's contents.  Only for small batches: T <= 4096.
 * Synchronous. */
hstu_status hstu_debug_attention_buckets(hstu_handle* h, int64_t total_tokens,
                                         const int32_t* seq_offsets, int32_t num_users,
                                         const int64_t* timestamps, hstu_mask_mode mask_mode,
                                         const int32_t* num_candidates, int32_t* pidx_out,
                                         int32_t* tidx_out, uint8_t* vis_out);

/* One 128 x n x k tile product on the tensor cores, to check the operand
 * layouts the kernels use: mode 0 = A[128,k] K-major (smem) x B[n,k] K-major
 * (smem); mode 1 = B given as [k, n] (N-major, smem); mode 2 = A staged in
 * tensor memory, B [k, n] N-major.  a, b bf16 device, c fp32 device [128, n].
 * n in {64, 128, 256} (mode >= 1: 64 or 128), k in {64, 128}.  Synchronous. */
hstu_status hstu_debug_umma_tile(int32_t mode, const void* a, const void* b, float* c, int32_t n,
                                 int32_t k);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_B200_H_ */
