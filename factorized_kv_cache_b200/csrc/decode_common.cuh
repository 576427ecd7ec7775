// Pieces shared by the two tensor-core decode kernels (decode_tensor.cu,
// decode_umma.cu): kernel parameters and the balanced tile partition.
//
// The tiles of all sequences (TOK tokens each) are laid end to end,
// sequence-major, as units of work, and CTA c of a grid of G takes units
// [ceil(c NT / G), ceil((c+1) NT / G)).  A non-empty sequence may start with
// `setup` extra units before its tiles: they stand for the time a CTA spends
// on a sequence's query before its first score (the query stage), so a CTA
// that starts a new sequence inside its range is given that much less
// streaming, and the CTAs end together.  Only the first and the last sequence
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
  int setup;               // set-up units per non-empty sequence, when charged (build_prefix)
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

// Exclusive prefix of per-sequence unit counts into s_pref[0..B] and the
// clamped lengths into s_len, computed by all NT_ threads of the CTA.  A
// length outside [0, min(capacity, max_len)] is clamped and flagged.  The
// set-up units are charged (p.setup per non-empty sequence) only when they
// leave the largest share, ceil(units / grid), where the tiles alone put it:
// the partition is whole tiles, and a set-up unit that pushed every CTA's
// share up by a tile would cost more than the query stage it stands for.
// Returns the set-up units charged per sequence (the same in every CTA).  Ends
// with __syncthreads.
template <int TOK, int NT_>
__device__ int build_prefix(const DecodeTcParams& p, int32_t* s_pref, int32_t* s_len, int32_t* s_tmp) {
  static_assert(NT_ <= 16 * 32, "two scans share s_tmp[32]");
  const int B = p.batch;
  const int tid = threadIdx.x;
  const int per = (B + NT_ - 1) / NT_;
  const int b0 = tid * per;
  int local = 0, local_n = 0;  // tiles, non-empty sequences
  for (int b = b0; b < min(B, b0 + per); ++b) {
    int L = p.seq_lens[b];
    if (L < 0 || L > p.capacity || L > p.max_len) {
      if (blockIdx.x == 0) atomicOr(p.err, TPA_DEVERR_LEN_RANGE);
      L = min(max(L, 0), min(p.capacity, p.max_len));
    }
    s_len[b] = L;
    const int tiles = (L + TOK - 1) / TOK;
    local += tiles;
    local_n += tiles > 0 ? 1 : 0;
  }
  const int lane = tid & 31, warp = tid >> 5;
  int incl = local, incl_n = local_n;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    const int vn = __shfl_up_sync(0xffffffffu, incl_n, o);
    if (lane >= o) {
      incl += v;
      incl_n += vn;
    }
  }
  if (lane == 31) {
    s_tmp[warp] = incl;
    s_tmp[16 + warp] = incl_n;
  }
  __syncthreads();
  // the warps' totals: lane w of every warp holds warp w's, so one reduction each gives this
  // warp's offset and the CTA's total
  constexpr int kWarps = NT_ / 32;
  const int wt = lane < kWarps ? s_tmp[lane] : 0;
  const int wn = lane < kWarps ? s_tmp[16 + lane] : 0;
  const int warp_off = __reduce_add_sync(0xffffffffu, lane < warp ? wt : 0);
  const int warp_off_n = __reduce_add_sync(0xffffffffu, lane < warp ? wn : 0);
  const unsigned tiles_all = static_cast<unsigned>(__reduce_add_sync(0xffffffffu, wt));
  const unsigned nonempty = static_cast<unsigned>(__reduce_add_sync(0xffffffffu, wn));
  const unsigned g = static_cast<unsigned>(p.grid);
  const int setup = (p.setup > 0 && tiles_all > 0 &&
                     (tiles_all + nonempty * static_cast<unsigned>(p.setup) + g - 1) / g == (tiles_all + g - 1) / g)
                        ? p.setup
                        : 0;
  int run = warp_off + incl - local, run_n = warp_off_n + incl_n - local_n;
  for (int b = b0; b < min(B, b0 + per); ++b) {
    s_pref[b] = run + setup * run_n;
    const int tiles = (s_len[b] + TOK - 1) / TOK;
    run += tiles;
    run_n += tiles > 0 ? 1 : 0;
  }
  if (tid == NT_ - 1) s_pref[B] = tiles_all + setup * nonempty;
  __syncthreads();
  return setup;
}

// First tile unit of sequence b (past its set-up units; s_pref[b + 1] when it has no tiles).
__device__ __forceinline__ int first_work(const int32_t* s_pref, int b, int setup) {
  return s_pref[b + 1] > s_pref[b] ? s_pref[b] + setup : s_pref[b];
}

// Largest b with s_pref[b] <= t and s_pref[b + 1] > t (the sequence holding unit t).
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
