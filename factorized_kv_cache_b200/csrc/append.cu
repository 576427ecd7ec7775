// Cache append with RoPE on the key feature factor.
//
// Tensor Product Attention Is All You Need, section 关键设计 (the cache keeps
// A_K, B_K, A_V, B_V per token) and section RoPE 兼容性 / Theorem 3.1 (the
// rotation acts on B only).  Token j of sequence b lands in slot
// seq_lens[b] + j; B_K rows are rotated at positions[b][j]; afterwards
// seq_lens[b] grows by n_new.
//
// Write-bound: every byte is read once and written once with 16-byte vectors.
// Small appends (decode: a few tokens per sequence) run as one CTA per
// sequence that also bumps the length; large appends (prefill) spread tokens
// over many CTAs and bump the lengths in a second one-CTA launch, so no CTA
// ever reads a length another CTA has already advanced.
#include "device_common.cuh"
#include "ptx_sm100.cuh"
#include "tpa_internal.h"

namespace tpa {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kTokensPerCta = 8;
constexpr int kSingleCtaMaxTokens = 32;

// cos, sin of every (token, RoPE pair) this CTA writes, one double-precision
// evaluation per entry spread over the CTA: s_cs[jj][pair] for tokens
// j0 + jj, jj < n_tok.  Ends with __syncthreads.
__device__ void rope_table(const AppendArgs& a, int b, int j0, int n_tok, float2* s_cs) {
  const int pairs = a.cache.head_dim / 2;
  for (int e = threadIdx.x; e < n_tok * pairs; e += blockDim.x) {
    const int jj = e / pairs, pr = e % pairs;
    const int pos = a.positions[static_cast<size_t>(b) * a.n_new + j0 + jj];
    float c, s;
    rope_cos_sin(pos, a.rope.theta[pr], &c, &s);
    s_cs[jj * kMaxPairs + pr] = make_float2(c, s);
  }
  __syncthreads();
}

// Copy (A_K, A_V, B_V) or rotate (B_K) every 16-byte vector of token j of
// sequence b into `slot`, with 64 threads; cs = that token's cos/sin row.
template <typename T>
__device__ void append_token(const AppendArgs& a, int b, int j, int slot, const float2* cs) {
  constexpr int V = Vec16<T>::N;
  const int h = a.cache.heads, d = a.cache.head_dim;
  const int rk = a.cache.r_k, rv = a.cache.r_v;
  const size_t cap = a.cache.capacity;
  const size_t src_tok = static_cast<size_t>(b) * a.n_new + j;
  const size_t dst_tok = static_cast<size_t>(b) * cap + slot;
  // vectors per plane for this token
  const int n_ak = rk * h / V, n_bk = rk * d / V, n_av = rv * h / V, n_bv = rv * d / V;
  const int total = n_ak + n_bk + n_av + n_bv;
  for (int v = threadIdx.x % 64; v < total; v += 64) {
    if (v < n_ak) {
      const T* src = static_cast<const T*>(a.a_k) + src_tok * rk * h + v * V;
      T* dst = static_cast<T*>(a.a_k_out) + dst_tok * rk * h + v * V;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    } else if (v < n_ak + n_bk) {
      const int w = v - n_ak;
      const int e0 = (w * V) % d;  // first feature index of this vector within its rank row
      const T* src = static_cast<const T*>(a.b_k) + src_tok * rk * d + w * V;
      T* dst = static_cast<T*>(a.b_k_out) + dst_tok * rk * d + w * V;
      float x[V];
      load16_f32(src, x);
#pragma unroll
      for (int p = 0; p < V / 2; ++p) {
        const float2 r = cs[(e0 >> 1) + p];
        rope_pair(x[2 * p], x[2 * p + 1], r.x, r.y);
      }
      store16_from_f32(dst, x);
    } else if (v < n_ak + n_bk + n_av) {
      const int w = v - n_ak - n_bk;
      const T* src = static_cast<const T*>(a.a_v) + src_tok * rv * h + w * V;
      T* dst = static_cast<T*>(a.a_v_out) + dst_tok * rv * h + w * V;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    } else {
      const int w = v - n_ak - n_bk - n_av;
      const T* src = static_cast<const T*>(a.b_v) + src_tok * rv * d + w * V;
      T* dst = static_cast<T*>(a.b_v_out) + dst_tok * rv * d + w * V;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
    }
  }
}

// One CTA per sequence: read the length, write every token, bump the length.
template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_single_kernel(const __grid_constant__ AppendArgs a) {
  // a kernel launched after this one with programmatic dependent launch may start its own
  // set-up now; it waits for this grid before it reads anything written here
  ptx::pdl_launch_dependents();
  __shared__ int s_base;
  __shared__ float2 s_cs[kSingleCtaMaxTokens * kMaxPairs];
  const int b = blockIdx.x;
  if (threadIdx.x == 0) s_base = a.seq_lens[b];
  rope_table(a, b, 0, a.n_new, s_cs);  // ends with __syncthreads
  const int base = s_base;
  const bool fits = base >= 0 && base + a.n_new <= a.cache.capacity;
  for (int j = threadIdx.x / 64; j < a.n_new; j += kAppendThreads / 64) {
    const int slot = base + j;
    if (slot < 0 || slot >= a.cache.capacity) continue;
    append_token<T>(a, b, j, slot, s_cs + j * kMaxPairs);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (fits) {
      a.seq_lens[b] = base + a.n_new;
    } else {
      atomicOr(a.err, TPA_DEVERR_APPEND_OVERFLOW);
    }
  }
}

// Many CTAs per sequence; lengths are only read here.  With explicit slots
// the lengths are not touched at all.
template <typename T>
__global__ void __launch_bounds__(kAppendThreads) append_multi_kernel(const __grid_constant__ AppendArgs a) {
  ptx::pdl_launch_dependents();
  __shared__ float2 s_cs[kTokensPerCta * kMaxPairs];
  const int b = blockIdx.y;
  const int base = a.slots ? 0 : a.seq_lens[b];
  const int j0 = blockIdx.x * kTokensPerCta;
  rope_table(a, b, j0, min(kTokensPerCta, a.n_new - j0), s_cs);
  for (int jj = threadIdx.x / 64; jj < kTokensPerCta; jj += kAppendThreads / 64) {
    const int j = j0 + jj;
    if (j >= a.n_new) break;
    const int slot = a.slots ? a.slots[static_cast<size_t>(b) * a.n_new + j] : base + j;
    if (slot < 0 || slot >= a.cache.capacity) {
      if (a.slots && (threadIdx.x & 63) == 0) atomicOr(a.err, TPA_DEVERR_APPEND_OVERFLOW);
      continue;
    }
    append_token<T>(a, b, j, slot, s_cs + jj * kMaxPairs);
  }
}

__global__ void bump_lens_kernel(int32_t* seq_lens, int batch, int n_new, int capacity, unsigned int* err) {
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    const int base = seq_lens[b];
    if (base >= 0 && base + n_new <= capacity) {
      seq_lens[b] = base + n_new;
    } else {
      atomicOr(err, TPA_DEVERR_APPEND_OVERFLOW);
    }
  }
}

template <typename T>
cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t stream) {
  if (a.slots) {
    dim3 grid((a.n_new + kTokensPerCta - 1) / kTokensPerCta, a.cache.batch);
    append_multi_kernel<T><<<grid, kAppendThreads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  if (a.n_new <= kSingleCtaMaxTokens) {
    append_single_kernel<T><<<a.cache.batch, kAppendThreads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  dim3 grid((a.n_new + kTokensPerCta - 1) / kTokensPerCta, a.cache.batch);
  append_multi_kernel<T><<<grid, kAppendThreads, 0, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  bump_lens_kernel<<<1, 256, 0, stream>>>(a.seq_lens, a.cache.batch, a.n_new, a.cache.capacity, a.err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream) {
  if (a.cache.dtype == TPA_F32) return launch_append_t<float>(a, stream);
  return launch_append_t<__nv_bfloat16>(a, stream);
}

}  // namespace tpa
