// Internal launch interface between the C ABI (tpa_api.cu) and the kernels.
// Host-side only: plain structs of pointers and sizes.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tpa.h"

namespace tpa {

constexpr int kMaxPairs = 64;  // head_dim <= 128

// theta_j = base^(-2j/d_h) for j < d_h/2, computed once on the host in double.
struct RopeTable {
  double theta[kMaxPairs];
};

void make_rope_table(double base, int head_dim, RopeTable* t);

// Sets the text tpa_last_error_message() returns on this host thread.
void set_last_error_message(const char* fmt, ...) __attribute__((format(printf, 1, 2)));

struct CacheView {
  int batch, capacity, heads, head_dim, r_k, r_v, dtype;
  const void* a_k;
  const void* b_k;
  const void* a_v;
  const void* b_v;
  const int32_t* seq_lens;
};

struct AppendArgs {
  CacheView cache;
  void* a_k_out;
  void* b_k_out;
  void* a_v_out;
  void* b_v_out;
  int32_t* seq_lens;  // mutable view of cache.seq_lens
  int n_new;
  const int32_t* slots;  // [B][n_new] explicit destination slots, or nullptr to append at seq_lens[b]
  const int32_t* positions;
  const void* a_k;
  const void* b_k;
  const void* a_v;
  const void* b_v;
  RopeTable rope;
  unsigned int* err;
};
cudaError_t launch_append(const AppendArgs& a, cudaStream_t stream);

// Split plan shared by every decode kernel: split j of sequence b covers
// tokens [j*chunk, min((j+1)*chunk, len_b)).
struct SplitPlan {
  int splits;
  int chunk;
};

// Queries handled by the CUDA-core attention kernel.  Decode: one query per
// sequence (q_per_seq = 1) attending the whole cache.  Prefill: q_per_seq
// queries per sequence, query t attending slots 0 .. len_b - q_per_seq + t.
struct SimtArgs {
  CacheView cache;
  const void* q;          // decode: [B][h][d] cache dtype, unrotated; prefill: [B][T][h][d] fp32, rotated
  int q_rotated_f32;      // 1 for the prefill form
  const int32_t* q_pos;   // decode: [B] (used when q is unrotated)
  int q_per_seq;          // 1 for decode
  int causal;             // prefill: limit each query to its own slot
  float scale;
  int max_len;
  SplitPlan plan;
  float* out;             // [B][q_per_seq][h][d]
  float* ws_ml;           // [B*q_per_seq][splits][h][2] (when splits > 1)
  float* ws_o;            // [B*q_per_seq][splits][h][d]
  RopeTable rope;
  unsigned int* err;
};
cudaError_t launch_simt_attention(const SimtArgs& a, cudaStream_t stream);

// Log-sum-exp merge of split partials into out.
struct MergeArgs {
  int n_queries, heads, head_dim, splits;
  const float* ws_ml;
  const float* ws_o;
  float* out;
  int use_pdl;
};
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t stream);

// Attention over disjoint token sets from each set's (o, lse) (lse_merge.cu): parts_out
// [n_parts][rows][head_dim], parts_lse [n_parts][rows] -> out [rows][head_dim], lse_out [rows]
// (may be null); head_dim a multiple of 4, at most 128.
cudaError_t launch_merge_lse(int n_parts, int rows, int head_dim, const float* parts_out, const float* parts_lse,
                             float* out, float* lse_out, cudaStream_t stream);

// Dense rotated queries for the CUDA-core prefill: Q[b][t][i][:] (fp32).
struct PrefillQArgs {
  int batch, n_tokens, heads, head_dim, r_q, dtype;
  const void* a_q;
  const void* b_q;
  const int32_t* q_pos;
  float* q_out;
  RopeTable rope;
};
cudaError_t launch_prefill_q(const PrefillQArgs& a, cudaStream_t stream);

// one CTA waiting on a shared-memory barrier that nothing completes, for limit_ns
cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, unsigned int* err, cudaStream_t stream);

}  // namespace tpa
