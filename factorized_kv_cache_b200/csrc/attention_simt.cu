// CUDA-core attention over the factorized cache (fp32 FMA), every supported
// shape and both dtypes.  It serves the fp32 decode workload, the shapes the
// tensor-core kernels do not cover, and as the CUDA-core baseline.
//
// Per cached token s and head i (Tensor Product Attention Is All You Need,
// sections 关键设计 and FlashTPA; the factors are never expanded to K or V):
//   S'[r, i] = q~_i . B~_K[s, r]                       (rank-r feature dot)
//   z[i]     = scale * (1/R_K) sum_r A_K[s, r, i] S'[r, i]
//   online softmax over s (running max m, sum l; base-2 exponentials)
//   o_i     += p (1/R_V) sum_r A_V[s, r, i] B_V[s, r, :]   (rank-R_V update)
// A CTA owns one (query, split) pair.  Eight threads share a head, each
// holding d_h/8 features of q~ and of the accumulator; their partial dots are
// summed with three xor-shuffles.  Token groups inside the CTA stride over
// the split's tokens and are merged through shared memory at the end.
#include <math.h>

#include "device_common.cuh"
#include "tpa_internal.h"

namespace tpa {
namespace {

constexpr int kSimtThreads = 256;
constexpr int kSlices = 8;

template <typename T, int SL>
__device__ __forceinline__ void load_slice(const T* __restrict__ p, float* out) {
  constexpr int V = Vec16<T>::N;
  if constexpr (SL % V == 0) {
#pragma unroll
    for (int k = 0; k < SL; k += V) load16_f32(p + k, out + k);
  } else {
#pragma unroll
    for (int k = 0; k < SL; ++k) out[k] = to_f32(p[k]);
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads, 2) simt_attention_kernel(const __grid_constant__ SimtArgs a) {
  constexpr int SL = D / kSlices;
  const int h = a.cache.heads;
  const int rk = a.cache.r_k, rv = a.cache.r_v;
  const int group = kSlices * h;
  const int G = kSimtThreads / group;
  const int tid = threadIdx.x;
  const int g = tid / group;
  const bool lane_on = g < G;
  const int i = lane_on ? (tid % group) / kSlices : 0;
  const int c = tid % kSlices;

  const int qi = blockIdx.y;
  const int b = qi / a.q_per_seq;
  const int t = qi % a.q_per_seq;
  const int split = blockIdx.x;

  int len = a.cache.seq_lens[b];
  int limit;
  if (a.causal) {
    const int P = len - a.q_per_seq;
    if (len > a.cache.capacity || P < 0) {
      if (tid == 0 && split == 0) atomicOr(a.err, TPA_DEVERR_PREFILL_LEN);
      return;  // leave this query's output untouched
    }
    limit = P + t + 1;
  } else {
    if (len < 0 || len > a.cache.capacity || len > a.max_len) {
      if (tid == 0 && split == 0) atomicOr(a.err, TPA_DEVERR_LEN_RANGE);
      len = min(max(len, 0), min(a.cache.capacity, a.max_len));
    }
    limit = len;
  }
  const int s_begin = split * a.plan.chunk;
  const int s_end = min(limit, s_begin + a.plan.chunk);

  // q~ slice for head i, features [c*SL, c*SL+SL)
  float qv[SL];
  if (a.q_rotated_f32) {
    const float* qp = static_cast<const float*>(a.q) + (static_cast<size_t>(qi) * h + i) * D + c * SL;
#pragma unroll
    for (int k = 0; k < SL; ++k) qv[k] = qp[k];
  } else {
    const T* qp = static_cast<const T*>(a.q) + (static_cast<size_t>(b) * h + i) * D + c * SL;
    load_slice<T, SL>(qp, qv);
    const int pos = a.q_pos[b];
#pragma unroll
    for (int p = 0; p < SL / 2; ++p) {
      float cs, sn;
      rope_cos_sin(pos, a.rope.theta[(c * SL) / 2 + p], &cs, &sn);
      rope_pair(qv[2 * p], qv[2 * p + 1], cs, sn);
    }
  }

  const float zs = a.scale * kLog2e / static_cast<float>(rk);
  const float inv_rv = 1.0f / static_cast<float>(rv);
  const size_t cap = a.cache.capacity;
  const T* AK = static_cast<const T*>(a.cache.a_k) + static_cast<size_t>(b) * cap * rk * h;
  const T* BK = static_cast<const T*>(a.cache.b_k) + static_cast<size_t>(b) * cap * rk * D;
  const T* AV = static_cast<const T*>(a.cache.a_v) + static_cast<size_t>(b) * cap * rv * h;
  const T* BV = static_cast<const T*>(a.cache.b_v) + static_cast<size_t>(b) * cap * rv * D;

  float m = -INFINITY, l = 0.0f;
  float acc[SL];
#pragma unroll
  for (int k = 0; k < SL; ++k) acc[k] = 0.0f;

  // kU tokens per group per iteration; every load of the iteration is issued
  // before the arithmetic that consumes it, so kU * (R_K + R_V) row loads are
  // in flight per thread instead of one.
  constexpr int kU = 4;
  for (int base = s_begin; base < s_end; base += G * kU) {
    float z[kU];
    bool valid[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int s = base + u * G + g;
      valid[u] = lane_on && s < s_end;
      z[u] = 0.0f;
    }
    for (int r = 0; r < rk; ++r) {
      float kb[kU][SL];
      float av[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int s = base + u * G + g;
        av[u] = 0.0f;
        if (valid[u]) {
          load_slice<T, SL>(BK + (static_cast<size_t>(s) * rk + r) * D + c * SL, kb[u]);
          av[u] = to_f32(AK[(static_cast<size_t>(s) * rk + r) * h + i]);
        } else {
#pragma unroll
          for (int k = 0; k < SL; ++k) kb[u][k] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        float part = 0.0f;
#pragma unroll
        for (int k = 0; k < SL; ++k) part = fmaf(qv[k], kb[u][k], part);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        z[u] = fmaf(av[u], part, z[u]);
      }
    }
    float m_new = m;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      z[u] *= zs;
      if (valid[u]) m_new = fmaxf(m_new, z[u]);
    }
    if (m_new == -INFINITY) continue;  // no valid token for this thread in this iteration
    const float corr = exp2f(m - m_new);
    float p[kU];
    float psum = 0.0f;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      p[u] = valid[u] ? exp2f(z[u] - m_new) : 0.0f;
      psum += p[u];
    }
    l = fmaf(l, corr, psum);
#pragma unroll
    for (int k = 0; k < SL; ++k) acc[k] *= corr;
    for (int r = 0; r < rv; ++r) {
      float vb[kU][SL];
      float w[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int s = base + u * G + g;
        w[u] = 0.0f;
        if (valid[u]) {
          load_slice<T, SL>(BV + (static_cast<size_t>(s) * rv + r) * D + c * SL, vb[u]);
          w[u] = p[u] * inv_rv * to_f32(AV[(static_cast<size_t>(s) * rv + r) * h + i]);
        } else {
#pragma unroll
          for (int k = 0; k < SL; ++k) vb[u][k] = 0.0f;
        }
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
#pragma unroll
        for (int k = 0; k < SL; ++k) acc[k] = fmaf(w[u], vb[u][k], acc[k]);
      }
    }
    m = m_new;
  }

  // merge the token groups of this CTA
  __shared__ float s_m[kSimtThreads / kSlices];
  __shared__ float s_l[kSimtThreads / kSlices];
  __shared__ float s_o[kSimtThreads / kSlices][D];
  const int slot = g * h + i;  // < G*h <= 32
  if (lane_on) {
    if (c == 0) {
      s_m[slot] = m;
      s_l[slot] = l;
    }
#pragma unroll
    for (int k = 0; k < SL; ++k) s_o[slot][c * SL + k] = acc[k];
  }
  __syncthreads();
  if (!lane_on || g != 0) return;
  float M = -INFINITY;
  for (int gg = 0; gg < G; ++gg) M = fmaxf(M, s_m[gg * h + i]);
  float L = 0.0f;
  float O[SL];
#pragma unroll
  for (int k = 0; k < SL; ++k) O[k] = 0.0f;
  if (M != -INFINITY) {
    for (int gg = 0; gg < G; ++gg) {
      const float mg = s_m[gg * h + i];
      const float wgt = (mg == -INFINITY) ? 0.0f : exp2f(mg - M);
      L = fmaf(s_l[gg * h + i], wgt, L);
#pragma unroll
      for (int k = 0; k < SL; ++k) O[k] = fmaf(s_o[gg * h + i][c * SL + k], wgt, O[k]);
    }
  }
  if (a.plan.splits == 1) {
    float* op = a.out + (static_cast<size_t>(qi) * h + i) * D + c * SL;
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
#pragma unroll
    for (int k = 0; k < SL; ++k) op[k] = O[k] * inv;
  } else {
    const size_t part = (static_cast<size_t>(qi) * a.plan.splits + split) * h + i;
    if (c == 0) {
      a.ws_ml[2 * part] = M;
      a.ws_ml[2 * part + 1] = L;
    }
    float* op = a.ws_o + part * D + c * SL;
#pragma unroll
    for (int k = 0; k < SL; ++k) op[k] = O[k];
  }
}

template <typename T>
cudaError_t launch_simt_t(const SimtArgs& a, cudaStream_t stream) {
  dim3 grid(a.plan.splits, a.cache.batch * a.q_per_seq);
  switch (a.cache.head_dim) {
    case 16: simt_attention_kernel<T, 16><<<grid, kSimtThreads, 0, stream>>>(a); break;
    case 32: simt_attention_kernel<T, 32><<<grid, kSimtThreads, 0, stream>>>(a); break;
    case 64: simt_attention_kernel<T, 64><<<grid, kSimtThreads, 0, stream>>>(a); break;
    case 128: simt_attention_kernel<T, 128><<<grid, kSimtThreads, 0, stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// Log-sum-exp merge: M = max_j m_j, L = sum_j l_j 2^(m_j-M),
// o = sum_j o_j 2^(m_j-M) / L (m in base-2 units).  One CTA per (query, head);
// the split maxima and sums are reduced across the CTA, the features are
// accumulated with eight independent loads in flight per thread.
__device__ __forceinline__ float block_reduce(float v, bool is_max, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_red[warp] = v;
  __syncthreads();
  v = s_red[0];
  for (int k = 1; k < nw; ++k) v = is_max ? fmaxf(v, s_red[k]) : v + s_red[k];
  return v;
}

__global__ void __launch_bounds__(128) merge_kernel(const __grid_constant__ MergeArgs a) {
  // with programmatic dependent launch, wait here for the split kernel's writes
  if (a.use_pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float s_red[4];
  const int q = blockIdx.x, i = blockIdx.y;
  const size_t row = static_cast<size_t>(q) * a.splits;
  const float* ml = a.ws_ml + 2 * (row * a.heads + i);  // split j at ml[2 * j * heads]
  const size_t mstride = 2 * static_cast<size_t>(a.heads);
  float M = -INFINITY;
  for (int j = threadIdx.x; j < a.splits; j += blockDim.x) M = fmaxf(M, ml[j * mstride]);
  M = block_reduce(M, true, s_red);
  float L = 0.0f;
  if (M != -INFINITY) {
    for (int j = threadIdx.x; j < a.splits; j += blockDim.x) {
      const float mj = ml[j * mstride];
      if (mj != -INFINITY) L = fmaf(ml[j * mstride + 1], exp2f(mj - M), L);
    }
  }
  L = block_reduce(L, false, s_red);
  const float inv = L > 0.0f ? 1.0f / L : 0.0f;
  const size_t ostride = static_cast<size_t>(a.heads) * a.head_dim;
  const float* o0 = a.ws_o + (row * a.heads + i) * a.head_dim;
  for (int k = threadIdx.x; k < a.head_dim; k += blockDim.x) {
    float O = 0.0f;
    if (M != -INFINITY) {
      int j = 0;
      for (; j + 8 <= a.splits; j += 8) {
        float v[8], wgt[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          v[u] = o0[(j + u) * ostride + k];
          const float mj = ml[(j + u) * mstride];
          wgt[u] = mj == -INFINITY ? 0.0f : exp2f(mj - M);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) O = fmaf(v[u], wgt[u], O);
      }
      for (; j < a.splits; ++j) {
        const float mj = ml[j * mstride];
        if (mj != -INFINITY) O = fmaf(o0[j * ostride + k], exp2f(mj - M), O);
      }
    }
    a.out[(static_cast<size_t>(q) * a.heads + i) * a.head_dim + k] = O * inv;
  }
}

// Dense rotated prefill queries (fp32): Q[t][i] = (1/R_Q) sum_j A_Q[t,j,i] RoPE(B_Q[t,j], pos_t)
// (section 解决思路 for the Q factorization, Theorem 3.1 for RoPE on B_Q).
// kPrefillQTokens tokens per CTA: one cos/sin per (token, RoPE pair), the rotated B_Q rows and
// A_Q of those tokens staged in shared memory, then every output float4 computed from them and
// stored coalesced (the kernel is bound by writing the fp32 queries).
constexpr int kPrefillQTokens = 4;
constexpr int kPrefillQThreads = 256;

// kD, kHeads > 0: the shape fixed at compile time (index arithmetic by shifts); 0: taken from a.
template <typename T, int kD, int kHeads>
__global__ void __launch_bounds__(kPrefillQThreads) prefill_q_kernel(const __grid_constant__ PrefillQArgs a) {
  extern __shared__ float s_q[];
  const int d = kD > 0 ? kD : a.head_dim, h = kHeads > 0 ? kHeads : a.heads, rq = a.r_q;
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kPrefillQTokens;
  const int nt = min(kPrefillQTokens, a.n_tokens - t0);
  float2* s_cs = reinterpret_cast<float2*>(s_q);                  // [tokens][d/2]
  float* s_bq = s_q + kPrefillQTokens * d;                         // [tokens][r_q][d] rotated
  float* s_aq = s_bq + kPrefillQTokens * rq * d;                   // [tokens][r_q][h]
  const int pairs = d / 2;
  for (int e = threadIdx.x; e < nt * pairs; e += blockDim.x) {
    const int tt = e / pairs, pr = e % pairs;
    float c, sn;
    rope_cos_sin(a.q_pos[static_cast<size_t>(b) * a.n_tokens + t0 + tt], a.rope.theta[pr], &c, &sn);
    s_cs[tt * pairs + pr] = make_float2(c, sn);
  }
  const size_t tok0 = static_cast<size_t>(b) * a.n_tokens + t0;
  const T* aq = static_cast<const T*>(a.a_q) + tok0 * rq * h;
  for (int e = threadIdx.x; e < nt * rq * h; e += blockDim.x) s_aq[e] = to_f32(aq[e]);
  __syncthreads();
  const T* bq = static_cast<const T*>(a.b_q) + tok0 * rq * d;
  for (int e = threadIdx.x; e < nt * rq * pairs; e += blockDim.x) {
    const int tt = e / (rq * pairs), pr = e % pairs;
    float x = to_f32(bq[2 * e]), y = to_f32(bq[2 * e + 1]);
    const float2 r = s_cs[tt * pairs + pr];
    rope_pair(x, y, r.x, r.y);
    s_bq[2 * e] = x;
    s_bq[2 * e + 1] = y;
  }
  __syncthreads();
  const float inv_rq = 1.0f / static_cast<float>(rq);
  float4* qo = reinterpret_cast<float4*>(a.q_out + tok0 * h * d);
  const int per_tok = h * d / 4;
  for (int e = threadIdx.x; e < nt * per_tok; e += blockDim.x) {
    const int tt = e / per_tok, r4 = e % per_tok;
    const int i = (4 * r4) / d, k = (4 * r4) % d;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < rq; ++j) {
      const float w = s_aq[(tt * rq + j) * h + i];
      const float4 v = *reinterpret_cast<const float4*>(s_bq + (tt * rq + j) * d + k);
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    qo[e] = make_float4(acc.x * inv_rq, acc.y * inv_rq, acc.z * inv_rq, acc.w * inv_rq);
  }
}

}  // namespace

cudaError_t launch_simt_attention(const SimtArgs& a, cudaStream_t stream) {
  if (a.cache.dtype == TPA_F32) return launch_simt_t<float>(a, stream);
  return launch_simt_t<__nv_bfloat16>(a, stream);
}

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream) {
  dim3 grid(a.n_queries, a.heads);
  const int threads = 128;
  if (!a.use_pdl) {
    merge_kernel<<<grid, threads, 0, stream>>>(a);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel, a);
}

cudaError_t launch_prefill_q(const PrefillQArgs& a, cudaStream_t stream) {
  dim3 grid((a.n_tokens + kPrefillQTokens - 1) / kPrefillQTokens, a.batch);
  const size_t smem = sizeof(float) * kPrefillQTokens *
                      (static_cast<size_t>(a.head_dim) + static_cast<size_t>(a.r_q) * (a.head_dim + a.heads));
  const bool fixed = a.head_dim == 128 && a.heads == 32;
  if (a.dtype == TPA_F32) {
    if (fixed)
      prefill_q_kernel<float, 128, 32><<<grid, kPrefillQThreads, smem, stream>>>(a);
    else
      prefill_q_kernel<float, 0, 0><<<grid, kPrefillQThreads, smem, stream>>>(a);
  } else {
    if (fixed)
      prefill_q_kernel<__nv_bfloat16, 128, 32><<<grid, kPrefillQThreads, smem, stream>>>(a);
    else
      prefill_q_kernel<__nv_bfloat16, 0, 0><<<grid, kPrefillQThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace tpa
