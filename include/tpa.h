/*
 * tpa.h - C ABI of libtpa: softmax attention evaluated directly over a
 * Tensor Product Attention (TPA) factorized KV cache, on NVIDIA B200 (sm_100a).
 *
 * Method: "Tensor Product Attention Is All You Need" (NeurIPS 2025 notes),
 *   - section 关键设计 / 张量积分解 (tensor product decomposition):
 *       K_t = (1/R_K) A_K(x_t)^T B_K(x_t),  V_t = (1/R_V) A_V(x_t)^T B_V(x_t),
 *       A in R^{R x h} (head factor), B in R^{R x d_h} (feature factor);
 *       the cache holds A_K, B_K, A_V, B_V: (R_K+R_V)(h+d_h) numbers/token.
 *   - section 解决思路: Q_t = (1/R_Q) A_Q(x_t)^T B_Q(x_t).
 *   - section RoPE 兼容性 (Theorem 3.1): RoPE rotates the B factors only.
 *   - section FlashTPA: attention runs on the factors; dense K/V are never built.
 *
 * Readings where the page is silent (the CPU oracle uses the same ones):
 *   RoPE pairs are adjacent elements (2j, 2j+1), angle = pos * theta_j with
 *   theta_j = rope_base^(-2j/d_h), (x, y) -> (x cos a - y sin a, x sin a + y cos a);
 *   angles are formed and reduced modulo 2*pi in double precision, the reduced
 *   angle (|a| <= pi) is evaluated in fp32 (rotation error ~3e-7 relative),
 *   the rotation itself runs in fp32 and is rounded once to the storage dtype.
 *   The softmax scale is given by the caller (1/sqrt(d_h) in the workloads).
 *
 * Conventions for every call:
 *   - The caller owns all memory.  Pointers marked "device" point to device
 *     memory of the current CUDA device; the library allocates nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Host-side argument checks run first; a call that
 *     returns anything but TPA_OK has launched nothing.
 *   - Conditions only the device can see (a length above max_len or the
 *     capacity, an append past the capacity) are recorded in a sticky device
 *     error word read by tpa_read_device_error(); the kernel skips the
 *     offending work and never traps.
 *   - Supported: dtype TPA_F32 or TPA_BF16; head_dim in {16, 32, 64, 128};
 *     1 <= heads <= 32 with heads * element size a multiple of 16 bytes;
 *     1 <= r_k, r_v <= 4; 1 <= r_q <= 8.  Anything else: TPA_ERR_UNSUPPORTED.
 */
#ifndef TPA_H_
#define TPA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tpa_status {
  TPA_OK = 0,
  TPA_ERR_NULL = 1,        /* a required pointer is NULL */
  TPA_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  TPA_ERR_UNSUPPORTED = 3, /* outside the supported set listed above */
  TPA_ERR_CAPACITY = 4,    /* a host-visible length exceeds the capacity */
  TPA_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than required */
  TPA_ERR_ALIGNMENT = 6,   /* a pointer is not 16-byte aligned */
  TPA_ERR_CUDA = 7         /* a CUDA runtime call failed (see tpa_last_error_message) */
} tpa_status;

typedef enum tpa_dtype { TPA_F32 = 0, TPA_BF16 = 1 } tpa_dtype;

/* Kernel choice for decode and prefill.  AUTO picks the fastest kernel that
 * supports the shape: the tensor-core kernels for bf16 at head_dim 128,
 * heads 32, r_k == r_v <= 2 (decode: batch <= 1024); the CUDA-core kernels
 * otherwise.  For the tensor-core decodes, num_splits is the number of CTAs
 * that share the batch's token tiles evenly (default: one wave, i.e. one
 * CTA per SM for TPA_KERNEL_TENSOR and two for TPA_KERNEL_TENSOR_SYNC). */
typedef enum tpa_kernel {
  TPA_KERNEL_AUTO = 0,
  TPA_KERNEL_SIMT = 1,        /* CUDA-core fp32 FMA path (every supported shape) */
  TPA_KERNEL_TENSOR = 2,      /* tensor-core path (bf16 only; TPA_ERR_UNSUPPORTED otherwise):
                               * tcgen05 MMAs with TMEM accumulators */
  TPA_KERNEL_TENSOR_SYNC = 3  /* decode only: the same shapes on warp-level mma.sync tensor-core
                               * instructions, kept for comparison with TPA_KERNEL_TENSOR */
} tpa_kernel;

/* Device error word bits (tpa_read_device_error). */
#define TPA_DEVERR_APPEND_OVERFLOW 0x1u /* an append reached a slot >= capacity */
#define TPA_DEVERR_LEN_RANGE 0x2u       /* seq_lens[b] < 0, > capacity or > max_len */
#define TPA_DEVERR_PREFILL_LEN 0x4u     /* prefill n_tokens > seq_lens[b] */
#define TPA_DEVERR_TIMEOUT 0x8u         /* a tensor-core kernel's wait on its own pipeline (a
                                         * shared-memory barrier another role of the CTA completes)
                                         * ran past its 2 s limit; the kernel returned early and the
                                         * call's outputs are not valid */

/*
 * A factorized KV cache of `batch` sequences, `capacity` token slots each.
 * Planes are token-major per sequence, row-major, contiguous, 16-byte aligned:
 *   a_k [batch][capacity][r_k][heads]     head factor of the keys
 *   b_k [batch][capacity][r_k][head_dim]  feature factor of the keys, stored
 *                                         rotated at the token's position
 *   a_v [batch][capacity][r_v][heads]     head factor of the values
 *   b_v [batch][capacity][r_v][head_dim]  feature factor of the values
 *   seq_lens [batch] int32                tokens held by each sequence
 * All five pointers are device pointers owned by the caller.  Slots at or
 * past seq_lens[b] may hold anything (NaN included); no kernel reads them
 * into a result.
 */
typedef struct tpa_cache {
  int32_t batch;
  int32_t capacity;
  int32_t heads;    /* h */
  int32_t head_dim; /* d_h */
  int32_t r_k;
  int32_t r_v;
  int32_t dtype;    /* tpa_dtype of the four planes */
  int32_t reserved; /* must be 0 */
  double rope_base; /* RoPE base (10000 in the workloads); > 1 */
  void* a_k;
  void* b_k;
  void* a_v;
  void* b_v;
  int32_t* seq_lens;
} tpa_cache;

/* (r_k + r_v) * (heads + head_dim): numbers stored per cached token
 * (section 关键设计: 320 at h=32, d_h=128, R_K=R_V=1, against 2*h*d_h = 8192).
 * Returns 0 for non-positive arguments. */
size_t tpa_factor_elements_per_token(int32_t heads, int32_t head_dim, int32_t r_k, int32_t r_v);

/*
 * Append n_new tokens to every sequence (section 关键设计 for the factors,
 * Theorem 3.1 for RoPE on B_K only).
 *   positions [batch][n_new] int32, device: RoPE position of each new token (>= 0)
 *   a_k [batch][n_new][r_k][heads], b_k [batch][n_new][r_k][head_dim] (NOT rotated),
 *   a_v [batch][n_new][r_v][heads], b_v [batch][n_new][r_v][head_dim]: device,
 *   in the cache dtype, contiguous, 16-byte aligned.
 * Token j of sequence b goes to slot seq_lens[b] + j: A_K, A_V, B_V are copied
 * and B_K is rotated at positions[b][j]; then seq_lens[b] += n_new on the
 * device.  A token whose slot would be >= capacity is not written and sets
 * TPA_DEVERR_APPEND_OVERFLOW (seq_lens[b] is then left unchanged).
 * n_new == 0 is a no-op.  Errors: NULL, SHAPE (n_new < 0), UNSUPPORTED, ALIGNMENT, CUDA.
 */
tpa_status tpa_cache_append(const tpa_cache* cache, int32_t n_new, const int32_t* positions,
                            const void* a_k, const void* b_k, const void* a_v, const void* b_v,
                            void* stream);

/*
 * The same factor write as tpa_cache_append (copy A_K, A_V, B_V; rotate B_K at
 * positions[b][j]) at caller-chosen slots: token j of sequence b goes to slot
 * slots[b][j] (int32, device, [batch][n_new]).  seq_lens is neither read nor
 * changed, so a fixed-length cache (a ring buffer, or a benchmark that
 * rewrites its newest token every step) keeps its lengths.  A slot outside
 * [0, capacity) is skipped and sets TPA_DEVERR_APPEND_OVERFLOW.  Two tokens
 * with the same slot in one call race (one of them wins).
 * Errors: as tpa_cache_append.
 */
tpa_status tpa_cache_write_slots(const tpa_cache* cache, int32_t n_new, const int32_t* slots,
                                 const int32_t* positions, const void* a_k, const void* b_k,
                                 const void* a_v, const void* b_v, void* stream);

/* Splits of the token range that decode uses when num_splits == 0. */
int32_t tpa_decode_default_splits(const tpa_cache* cache, int32_t max_len, int32_t kernel);

/* Workspace bytes tpa_decode_attention needs for this split count
 * (num_splits == 0: the default).  0 when one split suffices. */
size_t tpa_decode_workspace_size(const tpa_cache* cache, int32_t max_len, int32_t num_splits,
                                 int32_t kernel);

/*
 * Decode: one query token per sequence attends every cached token
 * 0 .. seq_lens[b]-1 (the query's own token is attended only if it was
 * appended first).
 *   q [batch][heads][head_dim], device, cache dtype, NOT rotated;
 *   q_pos [batch] int32, device: position of the query (RoPE);
 *   scale: softmax scale (1/sqrt(head_dim) in the workloads);
 *   out [batch][heads][head_dim] float32, device:
 *     out[b][i] = sum_s softmax_s(scale * q~_i . K_s[i]) V_s[i],
 *     q~ = RoPE(q, q_pos), K_s, V_s the factor products of slot s;
 *     0 for an empty sequence.
 *   max_len: host upper bound on every seq_lens[b] (sizes the grid);
 *   num_splits: 0 = default; the token range is cut into this many splits
 *     whose partial softmax states are merged by log-sum-exp;
 *   kernel: tpa_kernel;
 *   workspace: device, >= tpa_decode_workspace_size(...) bytes, 256-byte
 *     aligned; may be NULL when that size is 0.  Its contents on entry do not
 *     matter; calls that share one workspace must be ordered on the GPU.
 * Errors: NULL, SHAPE (max_len < 0), CAPACITY (max_len > capacity),
 * UNSUPPORTED, WORKSPACE, ALIGNMENT, CUDA.
 */
tpa_status tpa_decode_attention(const tpa_cache* cache, const void* q, const int32_t* q_pos,
                                float scale, float* out, int32_t max_len, int32_t num_splits,
                                int32_t kernel, void* workspace, size_t workspace_bytes,
                                void* stream);

/*
 * Decode with the query in TPA form (section 解决思路: Q = (1/R_Q) A_Q^T B_Q,
 * RoPE on the B factor by Theorem 3.1), the full-TPA variant of
 * tpa_decode_attention:
 *   a_q [batch][r_q][heads] and b_q [batch][r_q][head_dim] (NOT rotated):
 *     device, bf16, b_q 16-byte aligned; 1 <= r_q <= 8;
 *   query of head i: q~_i = (1/r_q) sum_j a_q[b][j][i] RoPE(b_q[b][j], q_pos[b]),
 *     formed in fp32 inside the kernel, then the same attention as
 *     tpa_decode_attention (same out, max_len, num_splits, workspace: use
 *     tpa_decode_workspace_size(cache, max_len, num_splits, TPA_KERNEL_TENSOR)).
 * Runs on the tcgen05 kernel only: bf16, heads 32, head_dim 128,
 * r_k == r_v <= 2, batch <= 1024, kernel TPA_KERNEL_AUTO or TPA_KERNEL_TENSOR;
 * anything else returns TPA_ERR_UNSUPPORTED.
 * Errors: those of tpa_decode_attention, SHAPE (r_q < 1), UNSUPPORTED.
 */
tpa_status tpa_decode_attention_factored(const tpa_cache* cache, int32_t r_q, const void* a_q,
                                         const void* b_q, const int32_t* q_pos, float scale,
                                         float* out, int32_t max_len, int32_t num_splits,
                                         int32_t kernel, void* workspace, size_t workspace_bytes,
                                         void* stream);

/*
 * tpa_decode_attention that also returns, per (sequence, head), the natural
 * log of the sum of exp(scaled score) over the attended tokens:
 *   lse [batch][heads] float32, device, 4-byte aligned;
 *   lse[b][i] = log sum_s exp(scale * q~_i . K_s[i]); -inf for an empty sequence.
 * (out, lse) of disjoint token ranges of one sequence combine exactly with
 * tpa_merge_lse, so a long sequence can be split across devices by token
 * range (each device holds its range with the tokens' global positions).
 * Runs on the tcgen05 kernel only (same shapes as tpa_decode_attention_factored).
 * Errors: those of tpa_decode_attention, NULL (lse), UNSUPPORTED, ALIGNMENT.
 */
tpa_status tpa_decode_attention_lse(const tpa_cache* cache, const void* q, const int32_t* q_pos, float scale,
                                    float* out, float* lse, int32_t max_len, int32_t num_splits, int32_t kernel,
                                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Attention over the union of n_parts disjoint token sets, from each set's
 * result (section FlashTPA: softmax over all cached tokens):
 *   parts_out [n_parts][rows][head_dim] float32, parts_lse [n_parts][rows] float32
 *   (device; the layout an all-gather of per-device (out, lse) produces);
 *   out [rows][head_dim] float32 = sum_r exp(lse_r - lse) parts_out[r],
 *   lse_out [rows] (device, may be NULL) = log sum_r exp(lse_r).
 * A part with lse_r = -inf (no tokens) drops out; a row without any token gets
 * out = 0, lse = -inf.  rows = batch * heads; head_dim a multiple of 4 in
 * [4, 128]; parts_out and out 16-byte aligned.  rows == 0 is a no-op.
 * Errors: SHAPE (n_parts < 1, rows < 0), UNSUPPORTED (head_dim), NULL, ALIGNMENT, CUDA.
 */
tpa_status tpa_merge_lse(int32_t n_parts, int32_t rows, int32_t head_dim, const float* parts_out,
                         const float* parts_lse, float* out, float* lse_out, void* stream);

/*
 * One generation step of token x_t, fused: its factors are appended and its
 * query attends the cache including x_t itself (section 解决思路: Q_t, K_t, V_t
 * all come from x_t; Theorem 3.1: B_K and the query rotate at x_t's position).
 *   positions [batch] int32, device: x_t's position (its key's and its query's);
 *   a_k [batch][r_k][heads], b_k [batch][r_k][head_dim] (NOT rotated),
 *   a_v [batch][r_v][heads], b_v [batch][r_v][head_dim]: device, bf16,
 *     16-byte aligned: x_t's factors;
 *   the query: r_q == 0: q [batch][heads][head_dim] dense, a_q unused;
 *     r_q in [1, 8]: TPA form as in tpa_decode_attention_factored, a_q
 *     [batch][r_q][heads] and q = b_q [batch][r_q][head_dim]; not rotated;
 *   out [batch][heads][head_dim] float32: attention of the query over slots
 *     0 .. L of sequence b, where L = seq_lens[b] on entry and slot L now
 *     holds x_t (B_K stored rotated, exactly as tpa_cache_append stores it);
 *     device memory, or pinned host memory the device can address (the kernels
 *     then write the output to the host directly, with no copy to launch);
 *   advance: 1 = seq_lens[b] becomes L + 1 (generation); 0 = seq_lens is left
 *     at L, so the next call overwrites the same slot (a fixed-length cache,
 *     or a token that may be rejected);
 *   max_len: host upper bound on every seq_lens[b] on entry; num_splits,
 *     kernel, workspace, workspace_bytes: as tpa_decode_attention
 *     (tpa_decode_workspace_size(cache, max_len, num_splits, TPA_KERNEL_TENSOR)).
 * Two launches (the split kernel over the tokens cached before the step and
 * the merge, which forms x_t's own score and value, stores x_t and joins it
 * to the log-sum-exp), against three for tpa_cache_append followed by
 * tpa_decode_attention.  If L == capacity, x_t is neither stored nor
 * attended, seq_lens is unchanged and TPA_DEVERR_APPEND_OVERFLOW is set.
 * Runs on the tcgen05 kernel only (same shapes as
 * tpa_decode_attention_factored); anything else returns TPA_ERR_UNSUPPORTED.
 * Errors: those of tpa_decode_attention, SHAPE (r_q < 0 or advance not 0/1),
 * NULL (a factor of x_t), UNSUPPORTED.
 */
tpa_status tpa_decode_step(const tpa_cache* cache, const int32_t* positions, const void* a_k, const void* b_k,
                           const void* a_v, const void* b_v, int32_t r_q, const void* a_q, const void* q,
                           float scale, float* out, int32_t max_len, int32_t advance, int32_t num_splits,
                           int32_t kernel, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Copies a step's inputs, packed in one buffer, from host memory to device
 * memory on `stream`: one asynchronous copy, ordered before whatever the
 * caller launches next on that stream (tpa_decode_step).  This is a
 * deployment convenience for bindings with no CUDA runtime of their own; the
 * pages define no such call.
 *   dst: device memory; src: host memory, pinned (page-locked) for the copy to
 *   be asynchronous (pageable memory is copied through a driver staging buffer,
 *   and the call may then return only once the copy is done); bytes == 0 is a
 *   no-op.  The caller owns both buffers and must not change src until the
 *   copy has run.
 * Errors: NULL (dst or src NULL with bytes > 0), CUDA (the copy was not enqueued).
 */
tpa_status tpa_stage_async(void* dst, const void* src, size_t bytes, void* stream);

/*
 * A decode step bound once, for a generation loop: tpa_step_plan_init checks
 * and stores the arguments of tpa_decode_step (plus an optional input copy),
 * and each tpa_step_plan_run then launches the step with no argument
 * marshalling or checking.  A deployment convenience with no counterpart on
 * the pages; the step computed is exactly tpa_decode_step's.
 * The plan is caller-owned storage whose contents are private to libtpa; it
 * holds no resources (nothing to release) and may be copied.
 */
typedef struct tpa_step_plan {
  uint64_t opaque[256];
} tpa_step_plan;

/*
 * Fills `plan` for tpa_decode_step with these arguments (same meaning, layout
 * and checks as tpa_decode_step; the stream is given to each run instead).
 * stage_bytes > 0: every run first copies stage_bytes from stage_src (pinned
 * host memory) to stage_dst (device memory) on the run's stream, as
 * tpa_stage_async does, so a loop whose inputs come from the host packs them
 * into stage_src and the copy lands where the bound inputs live.
 * The buffers must stay allocated, and the cache's planes and seq_lens in
 * place, while the plan is used; their contents may change between runs.
 * Runs must use the device that was current at init.  On error the plan is
 * left unusable (a run returns TPA_ERR_SHAPE).
 * Errors: those of tpa_decode_step; NULL (plan, or stage_dst / stage_src with
 * stage_bytes > 0); UNSUPPORTED (stage_bytes > 0 and stage_dst is not device
 * memory of the current device, or stage_src is not page-locked host memory:
 * both are checked here, once, since runs copy without checks); CUDA (device
 * query).
 */
tpa_status tpa_step_plan_init(tpa_step_plan* plan, const tpa_cache* cache, const int32_t* positions,
                              const void* a_k, const void* b_k, const void* a_v, const void* b_v, int32_t r_q,
                              const void* a_q, const void* q, float scale, float* out, int32_t max_len,
                              int32_t advance, int32_t num_splits, int32_t kernel, void* workspace,
                              size_t workspace_bytes, void* stage_dst, const void* stage_src, size_t stage_bytes);

/*
 * One step of an initialised plan on `stream`: the input copy if the plan has
 * one, then the step's two launches, as tpa_decode_step.
 * Errors: NULL (plan), SHAPE (plan not initialised), UNSUPPORTED (another
 * device is current), CUDA (a copy or launch failed).
 */
tpa_status tpa_step_plan_run(const tpa_step_plan* plan, void* stream);

/*
 * tpa_decode_attention for callers that cannot allocate device memory (no
 * counterpart on the page; this is a deployment convenience).  Same
 * arguments and result as tpa_decode_attention minus the workspace: the
 * split partials live in a 16 MiB scratch array compiled into libtpa, held
 * on every GPU that loads the library until the process exits.  Nothing is
 * allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - num_splits == 0: the default split count, lowered if needed until the
 *     partials fit in the 16 MiB array (the CUDA-core kernel with one split
 *     needs no scratch; the tcgen05 kernel's partials, at its fixed grid of
 *     one CTA per SM, take about 5 MB at the largest batch and always fit).
 *   - num_splits > 0 whose partials exceed 16 MiB: TPA_ERR_WORKSPACE, nothing
 *     launched, and tpa_last_error_message() says how much was needed.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.  A lookup that fails returns TPA_ERR_CUDA
 *     and is not remembered: the next call tries again.
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents (no call depends on them); calls that overlap on the
 *     GPU race on the array: order them on one stream or with events.
 * Errors: those of tpa_decode_attention, plus WORKSPACE as above.
 */
tpa_status tpa_decode_attention_noalloc(const tpa_cache* cache, const void* q, const int32_t* q_pos,
                                        float scale, float* out, int32_t max_len, int32_t num_splits,
                                        int32_t kernel, void* stream);

/* Workspace bytes tpa_prefill_attention needs: on the tensor-core path, fp16
 * copies of the cache's B_K and B_V planes (2 * batch * capacity * r_k *
 * head_dim * 2 bytes) and the chunk's B_Q rank rows rotated at their
 * positions (batch * n_tokens32 * r_q * head_dim * 2 bytes, n_tokens32 =
 * n_tokens rounded up to a multiple of 32; the dense per-head queries are
 * formed inside the kernel and never stored), each part rounded up to 256
 * bytes; on the
 * CUDA-core path, the dense rotated fp32 queries (batch * n_tokens * heads *
 * head_dim * 4 bytes). */
size_t tpa_prefill_workspace_size(const tpa_cache* cache, int32_t n_tokens, int32_t r_q,
                                  int32_t kernel);

/*
 * Causal prefill of a chunk of n_tokens queries per sequence whose K/V
 * factors were appended first: query t of sequence b sits at slot
 * P + t, P = seq_lens[b] - n_tokens, and attends slots 0 .. P + t.
 *   a_q [batch][n_tokens][r_q][heads], b_q [batch][n_tokens][r_q][head_dim]
 *     (B_Q NOT rotated): device, cache dtype;
 *   q_pos [batch][n_tokens] int32, device: query positions (RoPE on B_Q);
 *   query t, head i: q = (1/r_q) sum_j A_Q[t][j][i] RoPE(B_Q[t][j], q_pos[t]);
 *   out [batch][n_tokens][heads][head_dim] float32, device.
 *   workspace: device, >= tpa_prefill_workspace_size(...) bytes, 256-byte aligned.
 * The tensor-core path (bf16, heads 32, head_dim 128, r_k == r_v <= 2)
 * multiplies in fp16 with fp32 accumulation: the cache's B_K and B_V rows
 * are copied to fp16 (exact for magnitudes up to fp16's 65504; larger
 * values are outside this path and give non-finite outputs), the rotated
 * B_Q rank rows, the queries formed from them and the softmax weights are
 * rounded once each to fp16 (about 4e-4 relative each on unit-variance
 * factors).
 * Errors: NULL, SHAPE (n_tokens < 0 or > capacity), UNSUPPORTED, WORKSPACE,
 * ALIGNMENT, CUDA.  n_tokens > seq_lens[b] sets TPA_DEVERR_PREFILL_LEN and
 * leaves out[b] untouched.
 */
tpa_status tpa_prefill_attention(const tpa_cache* cache, int32_t n_tokens, int32_t r_q,
                                 const void* a_q, const void* b_q, const int32_t* q_pos,
                                 float scale, float* out, int32_t kernel, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Synchronise `stream`, copy the current device's error word to *code_out and
 * clear it.  Errors: NULL, CUDA. */
tpa_status tpa_read_device_error(uint32_t* code_out, void* stream);

/* Self-test of the bounded waits: launches one CTA that waits, for at most
 * limit_ns nanoseconds, on a shared-memory barrier that nothing completes, the
 * same bounded wait the tensor-core kernels use on their pipelines, and sets
 * TPA_DEVERR_TIMEOUT when the limit passes.  The timeout path can thus be made
 * to run without a fault: the kernel returns and the context stays usable.
 * limit_ns in [1, 10^10].  Errors: SHAPE (limit_ns out of range), CUDA. */
tpa_status tpa_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Static description of a status code. */
const char* tpa_status_string(tpa_status status);

/* Detail of the last failing call on this host thread ("" if none). */
const char* tpa_last_error_message(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* TPA_H_ */
