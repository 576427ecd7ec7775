// Pieces shared by the two tensor-core decode kernels (decode_tensor.cu,
// decode_umma.cu): kernel parameters and the balanced tile partition.
//
// The tiles of all sequences (TOK tokens each) are laid end to end,
// sequence-major, and CTA c of a grid of G takes tiles
// [ceil(c NT / G), ceil((c+1) NT / G)).  Only the first and the last sequence
// of a CTA's range can be shared with other CTAs; their partial softmax
// states go to workspace slots 2c and 2c+1, so the merge needs 2G slots
// whatever the batch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tpa_internal.h"

namespace tpa {
namespace dec {

constexpr int kH = 32;
constexpr int kD = 128;
constexpr int kMaxBatch = 1024;

struct DecodeTcParams {
  const int32_t* seq_lens;
  const void* q;           // [B][32][128] bf16, unrotated; with r_q > 0: B_Q [B][r_q][128]
  const void* a_q;         // A_Q [B][r_q][32] bf16 when the query is factorized (r_q > 0)
  int r_q;                 // 0: dense query
  float inv_rq;            // 1 / r_q
  const int32_t* q_pos;
  int batch, capacity, max_len, grid;
  double inv_grid;         // 1 / grid
  float zs;                // scale * log2(e) / R_K
  float inv_rv;            // 1 / R_V
  float* out;              // [B][32][128]
  int32_t* ws_prefix;      // [B + 1]
  float* ws_ml;            // [2G][32][2]
  float* ws_o;             // [2G][32][128]
  // A decode step (append + attend, see decode_tensor.cu): CTA 0 records the lengths it saw
  // (-1: out of range) for the merge kernel, which adds the step's own token.
  int32_t* ws_len;         // [B], or null when no step follows
  // A decode step, or a decode that also returns each head's log-sum-exp: a sequence finished
  // inside one CTA leaves its (m, l) per head beside its normalised output.
  float* whole_ml;         // [B][32][2], or null
  unsigned int* err;
  RopeTable rope;
};

// CTA that owns tile t: floor(t grid / nt).  The quotient is formed in
// double precision, which is exact here: the product is an integer below
// 2^53, and a quotient that is not an integer sits at least 1/nt away from
// one, far above the 2^-53 relative rounding (64-bit integer division would
// cost a long instruction sequence at kernel start).
__device__ __forceinline__ int owner_of(int t, int nt, int grid) {
  return static_cast<int>(floor(static_cast<double>(t) * grid / nt));
}

// First tile of CTA c: ceil(c nt / grid), exact for the same reason.
__device__ __forceinline__ int first_tile(int c, int nt, int grid) {
  return static_cast<int>(ceil(static_cast<double>(c) * nt / grid));
}

// ceil(c nt / grid) from a precomputed 1/grid: the double product is within one
// of the quotient, and one 64-bit integer step each way makes it exact (a
// multiply instead of the division sequence at the start of every CTA).
__device__ __forceinline__ int first_tile_fast(int c, int nt, int grid, double inv_grid) {
  const long long num = static_cast<long long>(c) * nt;
  long long q = static_cast<long long>(static_cast<double>(num) * inv_grid);
  if (q * grid < num) ++q;                    // q >= num / grid
  if ((q - 1) * grid >= num && q > 0) --q;    // q - 1 < num / grid
  return static_cast<int>(q);
}

// Exclusive prefix of per-sequence tile counts into s_pref[0..B] and the
// clamped lengths into s_len, computed by all NT_ threads of the CTA.  A
// length outside [0, min(capacity, max_len)] is clamped and flagged.  Ends
// with __syncthreads.
template <int TOK, int NT_>
__device__ void build_prefix(const DecodeTcParams& p, int32_t* s_pref, int32_t* s_len, int32_t* s_tmp) {
  const int B = p.batch;
  const int tid = threadIdx.x;
  const int per = (B + NT_ - 1) / NT_;
  const int b0 = tid * per;
  int local = 0;
  for (int b = b0; b < min(B, b0 + per); ++b) {
    int L = p.seq_lens[b];
    if (L < 0 || L > p.capacity || L > p.max_len) {
      if (blockIdx.x == 0) atomicOr(p.err, TPA_DEVERR_LEN_RANGE);
      L = min(max(L, 0), min(p.capacity, p.max_len));
    }
    s_len[b] = L;
    local += (L + TOK - 1) / TOK;
  }
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_tmp[warp] = incl;
  __syncthreads();
  int warp_off = 0;
  for (int w = 0; w < warp; ++w) warp_off += s_tmp[w];
  int run = warp_off + incl - local;
  for (int b = b0; b < min(B, b0 + per); ++b) {
    s_pref[b] = run;
    run += (s_len[b] + TOK - 1) / TOK;
  }
  if (tid == NT_ - 1) s_pref[B] = warp_off + incl;
  __syncthreads();
}

// Largest b with s_pref[b] <= t and s_pref[b + 1] > t (the sequence holding tile t).
__device__ __forceinline__ int sequence_of_tile(const int32_t* s_pref, int B, int t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= t) lo = mid; else hi = mid - 1;
  }
  while (lo < B && s_pref[lo + 1] <= t) ++lo;
  return lo;
}

}  // namespace dec

// The tcgen05 decode kernel (decode_umma.cu) on its default grid p.grid.
cudaError_t launch_decode_umma(const dec::DecodeTcParams& p, const CacheView& cv, cudaStream_t stream);

}  // namespace tpa
