// C ABI of libtpa (declared in include/tpa.h): argument checks, split
// planning, workspace carving and kernel dispatch.  No allocation, no state
// kept between calls beyond per-device constants (SM count, the address of
// the device error word).
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>

#include "tpa_internal.h"
#include "tpa_tensor.h"

namespace tpa {

__device__ unsigned int g_device_error;

namespace {

thread_local std::string t_last_error;

tpa_status fail(tpa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
tpa_status fail(tpa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

tpa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TPA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;
std::once_flag g_dev_once[kMaxDevices];
int g_dev_sms[kMaxDevices];
unsigned int* g_dev_err[kMaxDevices];
cudaError_t g_dev_status[kMaxDevices];

// Per-device constants, fetched once with that device current.
cudaError_t device_info(int* sms, unsigned int** err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_dev_once[dev], [dev]() {
    cudaError_t s = cudaDeviceGetAttribute(&g_dev_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (s == cudaSuccess) s = cudaGetSymbolAddress(reinterpret_cast<void**>(&g_dev_err[dev]), g_device_error);
    g_dev_status[dev] = s;
  });
  if (g_dev_status[dev] != cudaSuccess) return g_dev_status[dev];
  if (sms) *sms = g_dev_sms[dev];
  if (err) *err = g_dev_err[dev];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }
int esize(int dtype) { return dtype == TPA_F32 ? 4 : 2; }

tpa_status check_cache(const tpa_cache* c) {
  if (!c) return fail(TPA_ERR_NULL, "cache is NULL");
  if (!c->a_k || !c->b_k || !c->a_v || !c->b_v || !c->seq_lens)
    return fail(TPA_ERR_NULL, "a cache plane or seq_lens is NULL");
  if (c->batch < 1 || c->capacity < 1) return fail(TPA_ERR_SHAPE, "batch and capacity must be >= 1");
  if (c->reserved != 0) return fail(TPA_ERR_SHAPE, "reserved field must be 0");
  if (c->dtype != TPA_F32 && c->dtype != TPA_BF16) return fail(TPA_ERR_UNSUPPORTED, "dtype %d", c->dtype);
  if (c->head_dim != 16 && c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128)
    return fail(TPA_ERR_UNSUPPORTED, "head_dim %d not in {16,32,64,128}", c->head_dim);
  if (c->heads < 1 || c->heads > 32) return fail(TPA_ERR_UNSUPPORTED, "heads %d not in [1,32]", c->heads);
  if ((c->heads * esize(c->dtype)) % 16 != 0)
    return fail(TPA_ERR_UNSUPPORTED, "heads * element size (%d bytes) must be a multiple of 16",
                c->heads * esize(c->dtype));
  if (c->r_k < 1 || c->r_k > 4 || c->r_v < 1 || c->r_v > 4)
    return fail(TPA_ERR_UNSUPPORTED, "r_k=%d r_v=%d not in [1,4]", c->r_k, c->r_v);
  if (!(c->rope_base > 1.0) || !isfinite(c->rope_base))
    return fail(TPA_ERR_SHAPE, "rope_base must be finite and > 1");
  if (!aligned16(c->a_k) || !aligned16(c->b_k) || !aligned16(c->a_v) || !aligned16(c->b_v) ||
      (reinterpret_cast<uintptr_t>(c->seq_lens) & 3u))
    return fail(TPA_ERR_ALIGNMENT, "cache planes must be 16-byte aligned");
  return TPA_OK;
}

CacheView view_of(const tpa_cache* c) {
  CacheView v;
  v.batch = c->batch;
  v.capacity = c->capacity;
  v.heads = c->heads;
  v.head_dim = c->head_dim;
  v.r_k = c->r_k;
  v.r_v = c->r_v;
  v.dtype = c->dtype;
  v.a_k = c->a_k;
  v.b_k = c->b_k;
  v.a_v = c->a_v;
  v.b_v = c->b_v;
  v.seq_lens = c->seq_lens;
  return v;
}

// ---------------------------------------------------------------- decode planning
int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

bool use_tensor_decode(const tpa_cache* c, int kernel) {
  if (kernel == TPA_KERNEL_SIMT) return false;
  return tensor_decode_supported(c->dtype, c->heads, c->head_dim, c->r_k, c->r_v) &&
         tensor_decode_batch_ok(c->batch);
}

int decode_variant(int kernel) { return kernel == TPA_KERNEL_TENSOR_SYNC ? kDecodeSync : kDecodeUmma; }

// CUDA-core decode: split j of sequence b covers tokens [j*chunk, (j+1)*chunk).
SplitPlan plan_splits(const tpa_cache* c, int max_len, int num_splits, int sms) {
  SplitPlan p;
  const int granule = 16;
  if (max_len <= 0) {
    p.splits = 1;
    p.chunk = granule;
    return p;
  }
  int splits = num_splits;
  if (splits <= 0) {
    // about eight 256-thread CTAs per SM, splits no shorter than 64 tokens
    const int target = sms * 8;
    splits = ceil_div(target, c->batch);
    splits = splits < 1 ? 1 : splits;
    const int max_splits = ceil_div(max_len, 64);
    if (splits > max_splits) splits = max_splits;
  }
  if (splits < 1) splits = 1;
  int chunk = ceil_div(ceil_div(max_len, splits), granule) * granule;
  p.chunk = chunk;
  p.splits = ceil_div(max_len, chunk);
  return p;
}

struct DecodeWs {
  float* ml;
  float* o;
  size_t bytes;
};

DecodeWs carve_decode_ws(void* base, int n_queries, int heads, int head_dim, int splits) {
  DecodeWs w;
  if (splits <= 1) {
    w.ml = w.o = nullptr;
    w.bytes = 0;
    return w;
  }
  const size_t parts = static_cast<size_t>(n_queries) * splits * heads;
  const size_t ml_bytes = round256(parts * 2 * sizeof(float));
  const size_t o_bytes = round256(parts * head_dim * sizeof(float));
  char* p = static_cast<char*>(base);
  w.ml = reinterpret_cast<float*>(p);
  w.o = reinterpret_cast<float*>(p ? p + ml_bytes : nullptr);
  w.bytes = ml_bytes + o_bytes;
  return w;
}

}  // namespace

void set_last_error_message(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_last_error = buf;
}

// theta_j = base^(-2j/d_h); the last table built on this host thread is reused.
void make_rope_table(double base, int head_dim, RopeTable* t) {
  thread_local double t_base = 0.0;
  thread_local int t_dim = 0;
  thread_local RopeTable t_table;
  if (t_dim != head_dim || t_base != base) {
    memset(&t_table, 0, sizeof(t_table));
    for (int j = 0; j < head_dim / 2 && j < kMaxPairs; ++j)
      t_table.theta[j] = pow(base, -2.0 * static_cast<double>(j) / static_cast<double>(head_dim));
    t_base = base;
    t_dim = head_dim;
  }
  *t = t_table;
}

}  // namespace tpa

using namespace tpa;

extern "C" {

size_t tpa_factor_elements_per_token(int32_t heads, int32_t head_dim, int32_t r_k, int32_t r_v) {
  if (heads <= 0 || head_dim <= 0 || r_k <= 0 || r_v <= 0) return 0;
  return static_cast<size_t>(r_k + r_v) * static_cast<size_t>(heads + head_dim);
}

namespace {
tpa_status write_factors(const tpa_cache* cache, int32_t n_new, const int32_t* slots, const int32_t* positions,
                         const void* a_k, const void* b_k, const void* a_v, const void* b_v, void* stream) {
  tpa_status s = check_cache(cache);
  if (s != TPA_OK) return s;
  if (n_new < 0) return fail(TPA_ERR_SHAPE, "n_new = %d < 0", n_new);
  if (n_new == 0) return TPA_OK;
  if (!positions || !a_k || !b_k || !a_v || !b_v) return fail(TPA_ERR_NULL, "append input is NULL");
  if (!aligned16(a_k) || !aligned16(b_k) || !aligned16(a_v) || !aligned16(b_v) ||
      (reinterpret_cast<uintptr_t>(positions) & 3u) || (reinterpret_cast<uintptr_t>(slots) & 3u))
    return fail(TPA_ERR_ALIGNMENT, "append inputs must be 16-byte aligned");
  unsigned int* err = nullptr;
  cudaError_t e = device_info(nullptr, &err);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  AppendArgs a;
  a.cache = view_of(cache);
  a.a_k_out = cache->a_k;
  a.b_k_out = cache->b_k;
  a.a_v_out = cache->a_v;
  a.b_v_out = cache->b_v;
  a.seq_lens = cache->seq_lens;
  a.n_new = n_new;
  a.slots = slots;
  a.positions = positions;
  a.a_k = a_k;
  a.b_k = b_k;
  a.a_v = a_v;
  a.b_v = b_v;
  make_rope_table(cache->rope_base, cache->head_dim, &a.rope);
  a.err = err;
  e = launch_append(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return TPA_OK;
}
}  // namespace

tpa_status tpa_cache_append(const tpa_cache* cache, int32_t n_new, const int32_t* positions, const void* a_k,
                            const void* b_k, const void* a_v, const void* b_v, void* stream) {
  return write_factors(cache, n_new, nullptr, positions, a_k, b_k, a_v, b_v, stream);
}

tpa_status tpa_cache_write_slots(const tpa_cache* cache, int32_t n_new, const int32_t* slots,
                                 const int32_t* positions, const void* a_k, const void* b_k, const void* a_v,
                                 const void* b_v, void* stream) {
  if (n_new > 0 && !slots) return fail(TPA_ERR_NULL, "slots is NULL");
  return write_factors(cache, n_new, slots, positions, a_k, b_k, a_v, b_v, stream);
}

int32_t tpa_decode_default_splits(const tpa_cache* cache, int32_t max_len, int32_t kernel) {
  if (check_cache(cache) != TPA_OK || max_len < 0) return 0;
  int sms = 148;
  if (device_info(&sms, nullptr) != cudaSuccess) sms = 148;
  if (use_tensor_decode(cache, kernel)) return tensor_decode_default_ctas(sms, decode_variant(kernel));
  return plan_splits(cache, max_len, 0, sms).splits;
}

size_t tpa_decode_workspace_size(const tpa_cache* cache, int32_t max_len, int32_t num_splits, int32_t kernel) {
  if (check_cache(cache) != TPA_OK || max_len < 0) return 0;
  int sms = 148;
  if (device_info(&sms, nullptr) != cudaSuccess) sms = 148;
  if (use_tensor_decode(cache, kernel))
    return tensor_decode_workspace_bytes(
        cache->batch, num_splits > 0 ? num_splits : tensor_decode_default_ctas(sms, decode_variant(kernel)));
  const SplitPlan p = plan_splits(cache, max_len, num_splits, sms);
  return carve_decode_ws(nullptr, cache->batch, cache->heads, cache->head_dim, p.splits).bytes;
}

namespace {

// Decode with a dense query (r_q == 0) or a factorized one (a_q, q = B_Q, r_q >= 1); with
// `step`, the query's own token is appended and attended in the same launches.
tpa_status decode_impl(const tpa_cache* cache, const void* q, const void* a_q, int32_t r_q, const int32_t* q_pos,
                       float scale, float* out, int32_t max_len, int32_t num_splits, int32_t kernel, void* workspace,
                       size_t workspace_bytes, void* stream, const DecodeStepArgs* step = nullptr,
                       float* lse = nullptr, TensorDecodeArgs* bind = nullptr) {
  tpa_status s = check_cache(cache);
  if (s != TPA_OK) return s;
  if (!q || !q_pos || !out) return fail(TPA_ERR_NULL, "q, q_pos or out is NULL");
  if (max_len < 0) return fail(TPA_ERR_SHAPE, "max_len = %d < 0", max_len);
  if (max_len > cache->capacity) return fail(TPA_ERR_CAPACITY, "max_len %d > capacity %d", max_len, cache->capacity);
  if (num_splits < 0) return fail(TPA_ERR_SHAPE, "num_splits = %d < 0", num_splits);
  if (kernel != TPA_KERNEL_AUTO && kernel != TPA_KERNEL_SIMT && kernel != TPA_KERNEL_TENSOR &&
      kernel != TPA_KERNEL_TENSOR_SYNC)
    return fail(TPA_ERR_SHAPE, "kernel = %d", kernel);
  if ((kernel == TPA_KERNEL_TENSOR || kernel == TPA_KERNEL_TENSOR_SYNC) &&
      !tensor_decode_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v))
    return fail(TPA_ERR_UNSUPPORTED, "tensor-core decode needs bf16, heads 32, head_dim 128, r_k == r_v <= 2");
  if (!isfinite(scale)) return fail(TPA_ERR_SHAPE, "scale is not finite");
  if (!aligned16(q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(q_pos) & 3u))
    return fail(TPA_ERR_ALIGNMENT, "q and out must be 16-byte aligned");
  if (r_q > 0) {
    // the factorized query is formed inside the tcgen05 kernel only
    if (!a_q) return fail(TPA_ERR_NULL, "a_q is NULL");
    if (r_q > 8) return fail(TPA_ERR_UNSUPPORTED, "r_q = %d not in [1,8]", r_q);
    if (kernel == TPA_KERNEL_SIMT || kernel == TPA_KERNEL_TENSOR_SYNC ||
        !tensor_decode_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v) ||
        !tensor_decode_batch_ok(cache->batch))
      return fail(TPA_ERR_UNSUPPORTED,
                  "a factorized decode query needs the tcgen05 kernel: bf16, heads 32, head_dim 128, "
                  "r_k == r_v <= 2, batch <= 1024, kernel AUTO or TENSOR");
    if (reinterpret_cast<uintptr_t>(a_q) & 1u) return fail(TPA_ERR_ALIGNMENT, "a_q must be 2-byte aligned");
  }
  if (lse) {
    if (kernel == TPA_KERNEL_SIMT || kernel == TPA_KERNEL_TENSOR_SYNC ||
        !tensor_decode_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v) ||
        !tensor_decode_batch_ok(cache->batch))
      return fail(TPA_ERR_UNSUPPORTED,
                  "the log-sum-exp output needs the tcgen05 kernel: bf16, heads 32, head_dim 128, "
                  "r_k == r_v <= 2, batch <= 1024, kernel AUTO or TENSOR");
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return fail(TPA_ERR_ALIGNMENT, "lse must be 4-byte aligned");
  }
  if (step) {
    if (!step->a_k || !step->b_k || !step->a_v || !step->b_v)
      return fail(TPA_ERR_NULL, "a factor of the step's token is NULL");
    if (step->advance != 0 && step->advance != 1) return fail(TPA_ERR_SHAPE, "advance = %d", step->advance);
    if (kernel == TPA_KERNEL_SIMT || kernel == TPA_KERNEL_TENSOR_SYNC ||
        !tensor_decode_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v) ||
        !tensor_decode_batch_ok(cache->batch))
      return fail(TPA_ERR_UNSUPPORTED,
                  "a decode step needs the tcgen05 kernel: bf16, heads 32, head_dim 128, r_k == r_v <= 2, "
                  "batch <= 1024, kernel AUTO or TENSOR");
    if (!aligned16(step->a_k) || !aligned16(step->b_k) || !aligned16(step->a_v) || !aligned16(step->b_v))
      return fail(TPA_ERR_ALIGNMENT, "the step's factors must be 16-byte aligned");
  }
  int sms = 0;
  unsigned int* err = nullptr;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RopeTable rope;
  make_rope_table(cache->rope_base, cache->head_dim, &rope);
  if ((kernel == TPA_KERNEL_TENSOR || kernel == TPA_KERNEL_TENSOR_SYNC) && !tensor_decode_batch_ok(cache->batch))
    return fail(TPA_ERR_UNSUPPORTED, "tensor-core decode takes at most 1024 sequences per call");
  if (use_tensor_decode(cache, kernel)) {
    const int variant = decode_variant(kernel);
    const int grid = num_splits > 0 ? num_splits : tensor_decode_default_ctas(sms, variant);
    const size_t need = tensor_decode_workspace_bytes(cache->batch, grid);
    if (!workspace) return fail(TPA_ERR_WORKSPACE, "workspace is NULL, %zu bytes needed", need);
    if (workspace_bytes < need)
      return fail(TPA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
    if (!aligned256(workspace)) return fail(TPA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    TensorDecodeArgs a;
    a.cache = view_of(cache);
    a.q = q;
    a.a_q = a_q;
    a.r_q = r_q;
    a.q_pos = q_pos;
    a.scale = scale;
    a.max_len = max_len;
    a.grid = grid;
    a.out = out;
    a.workspace = workspace;
    a.rope = rope;
    a.err = err;
    a.variant = variant;
    a.step = step;
    a.lse = lse;
    if (bind) {  // a step plan: checked and prepared, launched later
      *bind = a;
      return TPA_OK;
    }
    e = launch_tensor_decode(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor decode launch");
    return TPA_OK;
  }
  if (bind) return fail(TPA_ERR_UNSUPPORTED, "a step plan needs the tcgen05 kernel");
  const SplitPlan plan = plan_splits(cache, max_len, num_splits, sms);
  DecodeWs ws = carve_decode_ws(workspace, cache->batch, cache->heads, cache->head_dim, plan.splits);
  if (ws.bytes > 0) {
    if (!workspace) return fail(TPA_ERR_WORKSPACE, "workspace is NULL, %zu bytes needed", ws.bytes);
    if (workspace_bytes < ws.bytes)
      return fail(TPA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, ws.bytes);
    if (!aligned256(workspace)) return fail(TPA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  }
  SimtArgs a;
  a.cache = view_of(cache);
  a.q = q;
  a.q_rotated_f32 = 0;
  a.q_pos = q_pos;
  a.q_per_seq = 1;
  a.causal = 0;
  a.scale = scale;
  a.max_len = max_len;
  a.plan = plan;
  a.out = out;
  a.ws_ml = ws.ml;
  a.ws_o = ws.o;
  a.rope = rope;
  a.err = err;
  e = launch_simt_attention(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if (plan.splits > 1) {
    MergeArgs m;
    m.n_queries = cache->batch;
    m.heads = cache->heads;
    m.head_dim = cache->head_dim;
    m.splits = plan.splits;
    m.ws_ml = ws.ml;
    m.ws_o = ws.o;
    m.out = out;
    m.use_pdl = 1;
    e = launch_merge(m, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return TPA_OK;
}

}  // namespace

tpa_status tpa_decode_attention(const tpa_cache* cache, const void* q, const int32_t* q_pos, float scale, float* out,
                                int32_t max_len, int32_t num_splits, int32_t kernel, void* workspace,
                                size_t workspace_bytes, void* stream) {
  return decode_impl(cache, q, nullptr, 0, q_pos, scale, out, max_len, num_splits, kernel, workspace,
                     workspace_bytes, stream);
}

tpa_status tpa_decode_attention_factored(const tpa_cache* cache, int32_t r_q, const void* a_q, const void* b_q,
                                         const int32_t* q_pos, float scale, float* out, int32_t max_len,
                                         int32_t num_splits, int32_t kernel, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (r_q < 1) return fail(TPA_ERR_SHAPE, "r_q = %d < 1", r_q);
  return decode_impl(cache, b_q, a_q, r_q, q_pos, scale, out, max_len, num_splits, kernel, workspace,
                     workspace_bytes, stream);
}

tpa_status tpa_decode_attention_lse(const tpa_cache* cache, const void* q, const int32_t* q_pos, float scale,
                                    float* out, float* lse, int32_t max_len, int32_t num_splits, int32_t kernel,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  if (!lse) return fail(TPA_ERR_NULL, "lse is NULL");
  return decode_impl(cache, q, nullptr, 0, q_pos, scale, out, max_len, num_splits, kernel, workspace,
                     workspace_bytes, stream, nullptr, lse);
}

tpa_status tpa_merge_lse(int32_t n_parts, int32_t rows, int32_t head_dim, const float* parts_out,
                         const float* parts_lse, float* out, float* lse_out, void* stream) {
  if (n_parts < 1 || rows < 0) return fail(TPA_ERR_SHAPE, "n_parts = %d (>= 1), rows = %d (>= 0)", n_parts, rows);
  if (head_dim < 4 || head_dim > 128 || head_dim % 4 != 0)
    return fail(TPA_ERR_UNSUPPORTED, "head_dim %d: a multiple of 4 in [4, 128]", head_dim);
  if (rows == 0) return TPA_OK;
  if (!parts_out || !parts_lse || !out) return fail(TPA_ERR_NULL, "parts_out, parts_lse or out is NULL");
  if (!aligned16(parts_out) || !aligned16(out) || (reinterpret_cast<uintptr_t>(parts_lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_out) & 3u))
    return fail(TPA_ERR_ALIGNMENT, "parts_out and out must be 16-byte aligned, the lse arrays 4-byte aligned");
  const cudaError_t e = launch_merge_lse(n_parts, rows, head_dim, parts_out, parts_lse, out, lse_out,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "lse merge launch");
  return TPA_OK;
}

tpa_status tpa_stage_async(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return TPA_OK;
  if (!dst || !src) return fail(TPA_ERR_NULL, "dst or src is NULL");
  const cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "input copy");
  return TPA_OK;
}

namespace {

constexpr uint32_t kStepPlanMagic = 0x54504153u;

// What a tpa_step_plan holds: the checked launch arguments of one decode step.
struct StepPlan {
  uint32_t magic;  // kStepPlanMagic once initialised
  int device;
  DecodeStepArgs step;
  TensorDecodeArgs args;  // args.step is pointed at `step` at each run (the plan may be copied)
  void* stage_dst;
  const void* stage_src;
  size_t stage_bytes;
};
static_assert(sizeof(StepPlan) <= sizeof(tpa_step_plan), "tpa_step_plan is too small");
static_assert(alignof(StepPlan) <= alignof(tpa_step_plan), "tpa_step_plan is under-aligned");

}  // namespace

tpa_status tpa_step_plan_init(tpa_step_plan* plan, const tpa_cache* cache, const int32_t* positions,
                              const void* a_k, const void* b_k, const void* a_v, const void* b_v, int32_t r_q,
                              const void* a_q, const void* q, float scale, float* out, int32_t max_len,
                              int32_t advance, int32_t num_splits, int32_t kernel, void* workspace,
                              size_t workspace_bytes, void* stage_dst, const void* stage_src, size_t stage_bytes) {
  if (!plan) return fail(TPA_ERR_NULL, "plan is NULL");
  memset(plan, 0, sizeof(*plan));
  StepPlan* sp = reinterpret_cast<StepPlan*>(plan);
  if (r_q < 0) return fail(TPA_ERR_SHAPE, "r_q = %d < 0", r_q);
  if (stage_bytes > 0 && (!stage_dst || !stage_src)) return fail(TPA_ERR_NULL, "stage_dst or stage_src is NULL");
  sp->step.a_k = a_k;
  sp->step.b_k = b_k;
  sp->step.a_v = a_v;
  sp->step.b_v = b_v;
  sp->step.advance = advance;
  const tpa_status s = decode_impl(cache, q, r_q > 0 ? a_q : nullptr, r_q, positions, scale, out, max_len,
                                   num_splits, kernel, workspace, workspace_bytes, nullptr, &sp->step, nullptr,
                                   &sp->args);
  if (s != TPA_OK) {
    memset(plan, 0, sizeof(*plan));
    return s;
  }
  const cudaError_t e = cudaGetDevice(&sp->device);
  if (e != cudaSuccess) {
    memset(plan, 0, sizeof(*plan));
    return cuda_fail(e, "device query");
  }
  if (stage_bytes > 0) {
    // the bound copy runs every step without further checks: its ends must be device memory of
    // this device and page-locked host memory
    cudaPointerAttributes ad, as;
    const bool dst_ok = cudaPointerGetAttributes(&ad, stage_dst) == cudaSuccess &&
                        (ad.type == cudaMemoryTypeDevice || ad.type == cudaMemoryTypeManaged) &&
                        ad.device == sp->device;
    const bool src_ok = cudaPointerGetAttributes(&as, stage_src) == cudaSuccess && as.type == cudaMemoryTypeHost;
    cudaGetLastError();  // a failed attribute query leaves no error behind
    if (!dst_ok || !src_ok) {
      memset(plan, 0, sizeof(*plan));
      return fail(TPA_ERR_UNSUPPORTED, "%s", !dst_ok ? "stage_dst is not device memory of the current device"
                                                     : "stage_src is not page-locked host memory");
    }
  }
  sp->stage_dst = stage_bytes > 0 ? stage_dst : nullptr;
  sp->stage_src = stage_bytes > 0 ? stage_src : nullptr;
  sp->stage_bytes = stage_bytes;
  sp->magic = kStepPlanMagic;
  return TPA_OK;
}

tpa_status tpa_step_plan_run(const tpa_step_plan* plan, void* stream) {
  if (!plan) return fail(TPA_ERR_NULL, "plan is NULL");
  const StepPlan* sp = reinterpret_cast<const StepPlan*>(plan);
  if (sp->magic != kStepPlanMagic) return fail(TPA_ERR_SHAPE, "the plan is not initialised");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  if (dev != sp->device) return fail(TPA_ERR_UNSUPPORTED, "the plan is for device %d, device %d is current", sp->device, dev);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sp->stage_bytes > 0) {
    e = cudaMemcpyAsync(sp->stage_dst, sp->stage_src, sp->stage_bytes, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "input copy");
  }
  TensorDecodeArgs a = sp->args;
  a.step = &sp->step;
  e = launch_tensor_decode(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "tensor decode launch");
  return TPA_OK;
}

tpa_status tpa_decode_step(const tpa_cache* cache, const int32_t* positions, const void* a_k, const void* b_k,
                           const void* a_v, const void* b_v, int32_t r_q, const void* a_q, const void* q, float scale,
                           float* out, int32_t max_len, int32_t advance, int32_t num_splits, int32_t kernel,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (r_q < 0) return fail(TPA_ERR_SHAPE, "r_q = %d < 0", r_q);
  DecodeStepArgs step;
  step.a_k = a_k;
  step.b_k = b_k;
  step.a_v = a_v;
  step.b_v = b_v;
  step.advance = advance;
  return decode_impl(cache, q, r_q > 0 ? a_q : nullptr, r_q, positions, scale, out, max_len, num_splits, kernel,
                     workspace, workspace_bytes, stream, &step);
}

size_t tpa_prefill_workspace_size(const tpa_cache* cache, int32_t n_tokens, int32_t r_q, int32_t kernel) {
  if (check_cache(cache) != TPA_OK || n_tokens < 0 || r_q < 1 || r_q > 8) return 0;
  if (kernel != TPA_KERNEL_SIMT &&
      tensor_prefill_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v, r_q))
    return tensor_prefill_workspace_bytes(cache->batch, cache->capacity, cache->r_k, n_tokens, r_q);
  return round256(static_cast<size_t>(cache->batch) * n_tokens * cache->heads * cache->head_dim * sizeof(float));
}

tpa_status tpa_prefill_attention(const tpa_cache* cache, int32_t n_tokens, int32_t r_q, const void* a_q,
                                 const void* b_q, const int32_t* q_pos, float scale, float* out, int32_t kernel,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  tpa_status s = check_cache(cache);
  if (s != TPA_OK) return s;
  if (n_tokens < 0 || n_tokens > cache->capacity)
    return fail(TPA_ERR_SHAPE, "n_tokens = %d outside [0, capacity]", n_tokens);
  if (r_q < 1 || r_q > 8) return fail(TPA_ERR_UNSUPPORTED, "r_q = %d not in [1,8]", r_q);
  if (kernel != TPA_KERNEL_AUTO && kernel != TPA_KERNEL_SIMT && kernel != TPA_KERNEL_TENSOR)
    return fail(TPA_ERR_SHAPE, "kernel = %d", kernel);
  const bool tensor_ok =
      tensor_prefill_supported(cache->dtype, cache->heads, cache->head_dim, cache->r_k, cache->r_v, r_q);
  if (kernel == TPA_KERNEL_TENSOR && !tensor_ok)
    return fail(TPA_ERR_UNSUPPORTED, "tensor-core prefill needs bf16, heads 32, head_dim 128, r_k == r_v <= 2");
  if (n_tokens == 0) return TPA_OK;
  if (!a_q || !b_q || !q_pos || !out) return fail(TPA_ERR_NULL, "a_q, b_q, q_pos or out is NULL");
  if (!isfinite(scale)) return fail(TPA_ERR_SHAPE, "scale is not finite");
  if (!aligned16(a_q) || !aligned16(b_q) || !aligned16(out) || (reinterpret_cast<uintptr_t>(q_pos) & 3u))
    return fail(TPA_ERR_ALIGNMENT, "a_q, b_q and out must be 16-byte aligned");
  const size_t need = tpa_prefill_workspace_size(cache, n_tokens, r_q, kernel);
  if (!workspace) return fail(TPA_ERR_WORKSPACE, "workspace is NULL, %zu bytes needed", need);
  if (workspace_bytes < need) return fail(TPA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
  if (!aligned256(workspace)) return fail(TPA_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  unsigned int* err = nullptr;
  int sms = 0;
  cudaError_t e = device_info(&sms, &err);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RopeTable rope;
  make_rope_table(cache->rope_base, cache->head_dim, &rope);
  if (kernel != TPA_KERNEL_SIMT && tensor_ok) {
    TensorPrefillArgs a;
    a.cache = view_of(cache);
    a.n_tokens = n_tokens;
    a.r_q = r_q;
    a.a_q = a_q;
    a.b_q = b_q;
    a.q_pos = q_pos;
    a.scale = scale;
    a.out = out;
    a.workspace = workspace;
    a.rope = rope;
    a.err = err;
    a.sms = sms;
    e = launch_tensor_prefill(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "tensor prefill launch");
    return TPA_OK;
  }
  PrefillQArgs qa;
  qa.batch = cache->batch;
  qa.n_tokens = n_tokens;
  qa.heads = cache->heads;
  qa.head_dim = cache->head_dim;
  qa.r_q = r_q;
  qa.dtype = cache->dtype;
  qa.a_q = a_q;
  qa.b_q = b_q;
  qa.q_pos = q_pos;
  qa.q_out = static_cast<float*>(workspace);
  qa.rope = rope;
  e = launch_prefill_q(qa, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill query launch");
  SimtArgs a;
  a.cache = view_of(cache);
  a.q = workspace;
  a.q_rotated_f32 = 1;
  a.q_pos = q_pos;
  a.q_per_seq = n_tokens;
  a.causal = 1;
  a.scale = scale;
  a.max_len = cache->capacity;
  a.plan.splits = 1;
  a.plan.chunk = cache->capacity;
  a.out = out;
  a.ws_ml = nullptr;
  a.ws_o = nullptr;
  a.rope = rope;
  a.err = err;
  e = launch_simt_attention(a, st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return TPA_OK;
}

tpa_status tpa_read_device_error(uint32_t* code_out, void* stream) {
  if (!code_out) return fail(TPA_ERR_NULL, "code_out is NULL");
  unsigned int* err = nullptr;
  cudaError_t e = device_info(nullptr, &err);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int v = 0;
  e = cudaMemcpy(&v, err, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  e = cudaMemset(err, 0, sizeof(unsigned int));
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  *code_out = v;
  return TPA_OK;
}

tpa_status tpa_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 10000000000ull) return fail(TPA_ERR_SHAPE, "limit_ns = %llu outside [1, 1e10]",
                                                              static_cast<unsigned long long>(limit_ns));
  unsigned int* err = nullptr;
  cudaError_t e = device_info(nullptr, &err);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  e = launch_wait_timeout_selftest(limit_ns, err, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return TPA_OK;
}

const char* tpa_status_string(tpa_status status) {
  switch (status) {
    case TPA_OK: return "TPA_OK";
    case TPA_ERR_NULL: return "TPA_ERR_NULL: a required pointer is NULL";
    case TPA_ERR_SHAPE: return "TPA_ERR_SHAPE: a size is out of range or inconsistent";
    case TPA_ERR_UNSUPPORTED: return "TPA_ERR_UNSUPPORTED: shape or dtype outside the supported set";
    case TPA_ERR_CAPACITY: return "TPA_ERR_CAPACITY: length exceeds the cache capacity";
    case TPA_ERR_WORKSPACE: return "TPA_ERR_WORKSPACE: workspace missing or too small";
    case TPA_ERR_ALIGNMENT: return "TPA_ERR_ALIGNMENT: pointer not aligned";
    case TPA_ERR_CUDA: return "TPA_ERR_CUDA: CUDA runtime error";
  }
  return "unknown tpa_status";
}

const char* tpa_last_error_message(void) { return t_last_error.c_str(); }

}  // extern "C"
