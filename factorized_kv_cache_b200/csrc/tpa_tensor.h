// Internal interface of the tensor-core kernels (decode and causal prefill).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "tpa_internal.h"

namespace tpa {

// ---- decode (bf16, h = 32, d_h = 128, R_K == R_V in {1, 2}, batch <= 1024)
// The grid is `grid` CTAs sharing the batch's tiles evenly (see decode_tensor.cu).
// Two kernels share the partition, the workspace layout and the merge:
// kDecodeUmma (tcgen05, TMEM accumulators, one CTA per SM) and kDecodeSync
// (warp-level mma.sync, two CTAs per SM).
constexpr int kDecodeUmma = 0;
constexpr int kDecodeSync = 1;
bool tensor_decode_supported(int dtype, int heads, int head_dim, int r_k, int r_v);
bool tensor_decode_batch_ok(int batch);
int tensor_decode_default_ctas(int sms, int variant);
size_t tensor_decode_workspace_bytes(int batch, int grid);

// A decode step: the token being generated is stored at slot seq_lens[b] and attended by its
// own query (tcgen05 kernel only; the query position is that token's position).
struct DecodeStepArgs {
  const void* a_k;  // [B][R_K][h] bf16
  const void* b_k;  // [B][R_K][d_h] bf16, unrotated
  const void* a_v;  // [B][R_V][h]
  const void* b_v;  // [B][R_V][d_h]
  int advance;      // 1: seq_lens[b] += 1 after the step
};

struct TensorDecodeArgs {
  CacheView cache;
  const void* q;       // dense query [B][h][d_h], or B_Q [B][r_q][d_h] when r_q > 0
  const void* a_q;     // A_Q [B][r_q][h] when r_q > 0 (tcgen05 kernel only)
  int r_q;
  const int32_t* q_pos;
  float scale;
  int max_len;
  int grid;
  float* out;
  void* workspace;  // tensor_decode_workspace_bytes(batch, grid) bytes, 256-byte aligned
  RopeTable rope;
  unsigned int* err;
  int variant;  // kDecodeUmma or kDecodeSync
  const DecodeStepArgs* step;  // null for a plain decode
  float* lse;                  // [B][h] natural-log log-sum-exp of the scaled scores, or null
};
cudaError_t launch_tensor_decode(const TensorDecodeArgs& a, cudaStream_t stream);

// ---- causal prefill (bf16, h = 32, d_h = 128, R_K == R_V in {1, 2}, R_Q <= 8)
bool tensor_prefill_supported(int dtype, int heads, int head_dim, int r_k, int r_v, int r_q);
// fp16 copies of the cache's B_K and B_V planes and of the chunk's rotated B_Q rank rows
size_t tensor_prefill_workspace_bytes(int batch, int capacity, int r, int n_tokens, int r_q);

struct TensorPrefillArgs {
  CacheView cache;
  int n_tokens;
  int r_q;
  const void* a_q;
  const void* b_q;
  const int32_t* q_pos;
  float scale;
  float* out;
  void* workspace;
  RopeTable rope;
  unsigned int* err;
  int sms;
};
cudaError_t launch_tensor_prefill(const TensorPrefillArgs& a, cudaStream_t stream);

}  // namespace tpa
