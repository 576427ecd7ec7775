// Attention over disjoint token sets from each set's result: the reduction of a
// decode whose token range is split across devices (or any other split).
//
// Tensor Product Attention Is All You Need, section FlashTPA: attention is the
// softmax over every cached token.  Over a union of disjoint sets r with
// results (o_r, lse_r), lse_r = log sum_{s in r} exp(z_s):
//   lse = log sum_r exp(lse_r),   o = sum_r exp(lse_r - lse) o_r,
// so the sets merge exactly; a set without tokens (lse_r = -inf) drops out.
//
// One warp per output row (a sequence and head): lane l holds features
// 4l .. 4l + 3.  The parts are read in order with four rows' loads in flight.
#include <math.h>

#include "tpa_internal.h"

namespace tpa {
namespace {

constexpr int kWarps = 8;

__global__ void __launch_bounds__(kWarps * 32) merge_lse_kernel(int n_parts, int rows, int head_dim,
                                                                 const float* __restrict__ parts_out,
                                                                 const float* __restrict__ parts_lse,
                                                                 float* __restrict__ out, float* __restrict__ lse_out) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int n4 = head_dim / 4;
  float top = -INFINITY;
  for (int r = lane; r < n_parts; r += 32) top = fmaxf(top, parts_lse[static_cast<size_t>(r) * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) top = fmaxf(top, __shfl_xor_sync(0xffffffffu, top, o));
  const float base = top == -INFINITY ? 0.f : top;
  float tot = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (int r = 0; r < n_parts; ++r) {
    const size_t pr = static_cast<size_t>(r) * rows + row;
    const float l = parts_lse[pr];
    const float w = l == -INFINITY ? 0.f : expf(l - base);
    tot += w;
    if (lane < n4 && w != 0.f) {
      const float4 v = reinterpret_cast<const float4*>(parts_out + pr * head_dim)[lane];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
  }
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  if (lane < n4)
    reinterpret_cast<float4*>(out + static_cast<size_t>(row) * head_dim)[lane] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lse_out && lane == 0) lse_out[row] = tot > 0.f ? base + logf(tot) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge_lse(int n_parts, int rows, int head_dim, const float* parts_out, const float* parts_lse,
                             float* out, float* lse_out, cudaStream_t stream) {
  const int blocks = (rows + kWarps - 1) / kWarps;
  merge_lse_kernel<<<blocks, kWarps * 32, 0, stream>>>(n_parts, rows, head_dim, parts_out, parts_lse, out, lse_out);
  return cudaGetLastError();
}

}  // namespace tpa
