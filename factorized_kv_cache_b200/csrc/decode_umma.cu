// Decode attention on the 5th-generation tensor cores (tcgen05: TMEM
// accumulators, shared-memory operands fed by TMA), bf16, h = 32,
// d_h = 128, R_K = R_V = R in {1, 2}.
//
// What it computes (Tensor Product Attention Is All You Need, sections
// 关键设计 and FlashTPA; K and V are never expanded): for the cached rows
// (s, r) of a sequence and head i,
//   S[(s,r), i] = B~_K[s, r] . q~_i                           (tensor cores)
//   z[s, i]     = scale/R_K sum_r A_K[s, r, i] S[(s,r), i]
//   online softmax over s per head: p[s, i] = 2^(z log2e - m_i)
//   W[(s,r), i] = p[s, i] A_V[s, r, i] / R_V
//   O^T[:, i]  += sum_(s,r) B_V[s, r, :] W[(s,r), i]          (tensor cores)
// Cache rows are the M = 128 dimension of both MMAs: the score MMA is
// B_K tile (128 rows x 128 features, K-major) times the query (N = 64:
// the 32 heads' bf16 high parts, then their low parts), the value MMA is
// B_V^T (M = 128 features, MN-major straight from the cache tile) times W
// (K = 128 rows, N = 64: W's bf16 high parts, then its low parts).  Both
// splits keep ~16 bits: one bf16 rounding of W costs up to ~3e-3 relative
// error on the decode workloads, above their 2e-3 budget.
//
// Roles (320 threads, one CTA per SM): warp 0 streams tiles with TMA
// (no multicast) into a K ring {B_K, A_K} and a V ring {B_V, A_V}, two
// 40 KB slots each, the K loads running one tile ahead of the V loads;
// warp 1 owns 256 TMEM columns and one of its threads issues the MMAs;
// warps 2-9 run the softmax.  TMEM lane quadrant q (warps q + 2 and q + 6)
// holds cache rows 32q .. 32q + 31 of S and features 32q .. 32q + 31 of
// O^T; warps 2-5 take heads 0-15 of their rows, warps 6-9 heads 16-31, so
// every sub-partition runs two softmax warps.
// Per tile j: S(j) goes to TMEM columns [64 (j % 2), +64), so the score MMA
// of tile j + 1 overlaps the softmax of tile j; W(j) goes to one of two
// shared-memory buffers; O^T sits in columns [128, 192).  The K slot is
// released once the score MMA has completed and the softmax has read A_K;
// the V slot once the value MMA has completed.
//
// Softmax: every thread holds 16 scores of its row.  The running maxima m_i
// are shared by the CTA and move lazily: one barrier-with-OR per tile asks
// whether any score exceeds its head's maximum by more than 2^8; only then
// is the tile maximum reduced (warp reduce-scatter plus a 4-quadrant
// exchange) and O^T, l rescaled.  The row sums l_i stay per thread and are
// reduced at the end of a sequence segment.
//
// Scheduling, partials and the merge follow the balanced tile partition in
// decode_common.cuh (shared with the warp-level kernel in decode_tensor.cu).
// The kernel is launched with programmatic dependent launch: barriers, TMEM
// and the tensor maps are set up before it waits for the preceding kernel.
//
// Every wait is bounded (2 s): on a timeout the waiting thread sets the error
// word and an abort flag; the softmax warps leave their loop together at the
// next barrier, the MMA thread waits for its MMAs before TMEM is released, and
// the TMA thread for its loads in flight.
#include <cuda.h>
#include <math.h>

#include <mutex>

#include "decode_common.cuh"
#include "device_common.cuh"
#include "ptx_sm100.cuh"
#include "tma_host.h"
#include "tpa_internal.h"
#include "tpa_tensor.h"

namespace tpa {
namespace {

using dec::DecodeTcParams;
using dec::kD;
using dec::kH;
using dec::kMaxBatch;

constexpr int kRows = 128;                   // cache rows per tile
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kThreads = 64 + kSoftmaxThreads;
constexpr int kHalf = kH / 2;                // heads per softmax thread
constexpr int kBox = kRows * 128;            // 64 features x 128 rows, bf16: 16 KB
constexpr int kBBytes = 2 * kBox;            // one B tile
constexpr int kABytes = kRows * kH * 2;      // one A tile: 8 KB
constexpr int kSlotBytes = kBBytes + kABytes;
constexpr int kWBytes = kRows * 64 * 2;      // W: 128 rows x (32 hi + 32 lo) bf16
constexpr int kQBox = 64 * 128;              // query: 64 rows x 64 features, bf16
constexpr int kOffK = 0;                     // K ring: 2 slots {B_K, A_K}
constexpr int kOffV = kOffK + 2 * kSlotBytes;  // V ring: 2 slots {B_V, A_V}
constexpr int kOffW = kOffV + 2 * kSlotBytes;  // two W buffers
constexpr int kOffQ = kOffW + 2 * kWBytes;     // query hi/lo, two 64-feature boxes
constexpr int kOffRed = kOffQ + 2 * kQBox;     // float [4 quadrants][32 heads]
constexpr int kOffCs = kOffRed + 4 * 32 * 4;   // float [64][2]: cos, sin of the query position
constexpr int kOffBar = kOffCs + 64 * 2 * 4;
// kfull[2], kempty[2], vfull[2], vempty[2], sfull[2], wready[2], wfree[2], qready, fin
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;  // TMEM address, abort flag, scan scratch [32]
constexpr int kOffPref = kOffMisc + 8 + 32 * 4;
constexpr int kOffLen = kOffPref + (kMaxBatch + 1) * 4;
constexpr size_t kSmemBytes = 1024 + kOffLen + kMaxBatch * 4;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kSlotBytes % 1024 == 0 && kWBytes % 1024 == 0 && kQBox % 1024 == 0, "swizzle atoms stay aligned");
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;
constexpr unsigned kErrTimeout = 0x8u;
constexpr float kLazy = 8.f;  // rescale only when a score exceeds its head's maximum by 2^8

// kind::f16 instruction descriptors: D fp32, A and B bf16, M = 128, N = 64.
constexpr uint32_t kIdescScore = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
// value MMA: A (B_V^T) and B (W) both MN-major
constexpr uint32_t kIdescValue = kIdescScore | (1u << 15) | (1u << 16);

// Reduce 16 per-head values over the 32 lanes of a warp; afterwards lanes k
// and k + 16 hold the result for head k (four halving exchange steps, then
// one across the two half-warps: 16 shuffles).
template <bool kMax>
__device__ __forceinline__ float reduce_scatter16(float (&v)[kHalf], int lane) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  const float other = __shfl_xor_sync(0xffffffffu, v[0], 16);
  return kMax ? fmaxf(v[0], other) : v[0] + other;
}

// Heads 16 hh .. 16 hh + 15 of row `row` of a 128-row A tile (32 bf16 =
// 64 bytes per row, 64-byte swizzle) as fp32.
__device__ __forceinline__ void load_a_half(const uint8_t* tile, int row, int hh, float* f) {
  const uint8_t* base = tile + row * 64;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(base + (((2 * hh + c) ^ ((row >> 1) & 3)) << 4));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[8 * c + 2 * k] = ptx::bf16_lo(w[k]);
      f[8 * c + 2 * k + 1] = ptx::bf16_hi(w[k]);
    }
  }
}

// Sum over the four TMEM lane quadrants of the per-quadrant head values in
// s_red[quad][32], for heads 16 hh .. 16 hh + 15.
template <bool kMax>
__device__ __forceinline__ void combine_quadrants(const float* s_red, int hh, float (&out)[kHalf]) {
#pragma unroll
  for (int h4 = 0; h4 < kHalf / 4; ++h4) {
    const float4 x0 = reinterpret_cast<const float4*>(s_red + 16 * hh)[h4];
    const float4 x1 = reinterpret_cast<const float4*>(s_red + 32 + 16 * hh)[h4];
    const float4 x2 = reinterpret_cast<const float4*>(s_red + 64 + 16 * hh)[h4];
    const float4 x3 = reinterpret_cast<const float4*>(s_red + 96 + 16 * hh)[h4];
    if (kMax) {
      out[4 * h4] = fmaxf(fmaxf(x0.x, x1.x), fmaxf(x2.x, x3.x));
      out[4 * h4 + 1] = fmaxf(fmaxf(x0.y, x1.y), fmaxf(x2.y, x3.y));
      out[4 * h4 + 2] = fmaxf(fmaxf(x0.z, x1.z), fmaxf(x2.z, x3.z));
      out[4 * h4 + 3] = fmaxf(fmaxf(x0.w, x1.w), fmaxf(x2.w, x3.w));
    } else {
      out[4 * h4] = (x0.x + x1.x) + (x2.x + x3.x);
      out[4 * h4 + 1] = (x0.y + x1.y) + (x2.y + x3.y);
      out[4 * h4 + 2] = (x0.z + x1.z) + (x2.z + x3.z);
      out[4 * h4 + 3] = (x0.w + x1.w) + (x2.w + x3.w);
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    decode_umma_kernel(const __grid_constant__ DecodeTcParams p, const __grid_constant__ CUtensorMap tm_bk,
                       const __grid_constant__ CUtensorMap tm_bv, const __grid_constant__ CUtensorMap tm_ak,
                       const __grid_constant__ CUtensorMap tm_av) {
  constexpr int TOK = kRows / R;  // tokens per tile
  extern __shared__ uint8_t smem_raw[];

  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  float* s_red = reinterpret_cast<float*>(gbase + kOffRed);
  float* s_cs = reinterpret_cast<float*>(gbase + kOffCs);
  // a query in TPA form: its raw rank rows [r_q][128] bf16 and A_Q / R_Q [r_q][32] staged in the W
  // buffers, which are idle whenever a sequence segment starts
  __nv_bfloat16* s_bqr = reinterpret_cast<__nv_bfloat16*>(gbase + kOffW);
  float* s_aq = reinterpret_cast<float*>(gbase + kOffW + 8 * kD * 2);
  const uint32_t bar0 = sbase + kOffBar;
  auto kfull = [&](int s) { return bar0 + 8 * s; };
  auto kempty = [&](int s) { return bar0 + 8 * (2 + s); };
  auto vfull = [&](int s) { return bar0 + 8 * (4 + s); };
  auto vempty = [&](int s) { return bar0 + 8 * (6 + s); };
  auto sfull = [&](int s) { return bar0 + 8 * (8 + s); };
  auto wready = [&](int s) { return bar0 + 8 * (10 + s); };
  auto wfree = [&](int s) { return bar0 + 8 * (12 + s); };
  const uint32_t qready = bar0 + 8 * 14;
  const uint32_t fin = bar0 + 8 * 15;
  volatile uint32_t* s_taddr = reinterpret_cast<volatile uint32_t*>(gbase + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);
  int32_t* s_tmp = reinterpret_cast<int32_t*>(gbase + kOffMisc + 8);
  int32_t* s_pref = reinterpret_cast<int32_t*>(gbase + kOffPref);
  int32_t* s_len = reinterpret_cast<int32_t*>(gbase + kOffLen);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Set-up that touches no global memory runs before the wait on the preceding kernel
  // (programmatic dependent launch): barriers, TMEM, tensor-map prefetch.
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(kfull(s), 1);
      ptx::mbar_init(kempty(s), 1 + kSoftmaxWarps);  // score-MMA commit + the softmax warps (A_K read)
      ptx::mbar_init(vfull(s), 1);
      ptx::mbar_init(vempty(s), 1);
      ptx::mbar_init(sfull(s), 1);
      ptx::mbar_init(wready(s), kSoftmaxWarps);
      ptx::mbar_init(wfree(s), 1);
    }
    ptx::mbar_init(qready, kSoftmaxWarps);
    ptx::mbar_init(fin, 1);
    *s_abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + kOffMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  if (tid == 0) {
    ptx::prefetch_tmap(&tm_bk);
    ptx::prefetch_tmap(&tm_bv);
    ptx::prefetch_tmap(&tm_ak);
    ptx::prefetch_tmap(&tm_av);
  }
  ptx::tc_fence_before();
  __syncwarp();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *s_taddr;
  ptx::pdl_wait();  // the cache, the lengths and the query are written by earlier work
  // The merge kernel may be scheduled from here on: every CTA has passed its wait, so all
  // work before this grid is complete and the merge may read the step's inputs at once
  // (it waits for this grid before it reads anything written here).
  ptx::pdl_launch_dependents();

  const int setup = dec::build_prefix<TOK, kThreads>(p, s_pref, s_len, s_tmp);  // ends with __syncthreads
  const int B = p.batch;
  const int NT = s_pref[B];
  if (blockIdx.x == 0) {
    for (int b = tid; b <= B; b += kThreads) p.ws_prefix[b] = s_pref[b];
    if (tid == 0) p.ws_prefix[B + 1] = setup;  // for the merge
  }
  const int c = blockIdx.x;
  const int t_begin = NT == 0 ? 0 : dec::first_tile_fast(c, NT, p.grid, p.inv_grid);
  const int t_end = NT == 0 ? 0 : dec::first_tile_fast(c + 1, NT, p.grid, p.inv_grid);
  // the lengths this grid saw, -1 where out of range, for the merge of a decode step
  auto record_lengths = [&](int first, int step) {
    for (int b = first; b < B; b += step) p.ws_len[b] = p.seq_lens[b] == s_len[b] ? s_len[b] : -1;
  };
  if (t_begin >= t_end) {  // uniform: no tiles for this CTA
    if (warp == 1 && blockIdx.x == 0 && p.ws_len) record_lengths(lane, 32);
    if (warp == 1) ptx::tmem_dealloc(tbase, kTmemCols);
    return;
  }
  const int b_first = dec::sequence_of_tile(s_pref, B, t_begin);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Load order K0, K1, V0, K2, V1, K3, ...: the score MMA of a tile needs only its K
    // slot, and the softmax reaches for A_V (the V slot) last.
    if (lane == 0) {
      // the CTA's tiles in order: units [t_begin, t_end) without the set-up units
      int n = 0;
      for (int b = b_first; b < B && s_pref[b] < t_end; ++b)
        n += max(0, min(t_end, s_pref[b + 1]) - max(t_begin, dec::first_work(s_pref, b, setup)));
      // cursors (sequence, unit) of the K and V streams: each call moves one to the next tile
      // (units past a sequence's set-up units) and returns the tile's first cache row
      int k_seq = b_first, k_unit = t_begin - 1, v_seq = b_first, v_unit = t_begin - 1;
      auto next_row = [&](int& cb, int& ct) {
        ++ct;
        while (cb < B) {
          const int w0 = dec::first_work(s_pref, cb, setup);
          if (ct < w0) ct = w0;
          if (ct < s_pref[cb + 1]) break;
          ++cb;
        }
        return (cb * p.capacity + (ct - dec::first_work(s_pref, cb, setup)) * TOK) * R;
      };
      auto load_k = [&](int j) -> bool {
        const int s = j & 1;
        if (j >= 2 && !ptx::mbar_wait_bounded(kempty(s), ((j >> 1) & 1) ^ 1)) return false;
        const int row0 = next_row(k_seq, k_unit);
        const uint32_t kb = sbase + kOffK + s * kSlotBytes;
        ptx::mbar_arrive_expect_tx(kfull(s), kSlotBytes);
        ptx::tma_load_2d(kb, &tm_bk, 0, row0, kfull(s));
        ptx::tma_load_2d(kb + kBox, &tm_bk, 64, row0, kfull(s));
        ptx::tma_load_2d(kb + kBBytes, &tm_ak, 0, row0, kfull(s));
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j & 1;
        if (j >= 2 && !ptx::mbar_wait_bounded(vempty(s), ((j >> 1) & 1) ^ 1)) return false;
        const int row0 = next_row(v_seq, v_unit);
        const uint32_t vb = sbase + kOffV + s * kSlotBytes;
        ptx::mbar_arrive_expect_tx(vfull(s), kSlotBytes);
        ptx::tma_load_2d(vb, &tm_bv, 0, row0, vfull(s));
        ptx::tma_load_2d(vb + kBox, &tm_bv, 64, row0, vfull(s));
        ptx::tma_load_2d(vb + kBBytes, &tm_av, 0, row0, vfull(s));
        return true;
      };
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (; k_issued < min(2, n); ++k_issued) load_k(k_issued);
      while (ok && v_issued < n) {
        if (*s_abort) {
          ok = false;
          break;
        }
        if (!(ok = load_v(v_issued))) break;
        ++v_issued;
        if (k_issued < n) {
          if (!(ok = load_k(k_issued))) break;
          ++k_issued;
        }
      }
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
        // every load already issued lands before the CTA can exit
        for (int k = max(0, k_issued - 2); k < k_issued; ++k) ptx::mbar_wait_bounded(kfull(k & 1), (k >> 1) & 1);
        for (int k = max(0, v_issued - 2); k < v_issued; ++k) ptx::mbar_wait_bounded(vfull(k & 1), (k >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Order per tile j: score MMA of j, then the value MMA of j - 1 (whose W the
    // softmax is finishing meanwhile).  At the first tile of a sequence segment the
    // pending value MMA goes first: the softmax warps must finish the previous
    // segment before they can write the next query.
    if (lane == 0) {
      auto value_mma = [&](int j, bool first) -> bool {
        if (!ptx::mbar_wait_bounded(wready(j & 1), (j >> 1) & 1)) return false;
        if (!ptx::mbar_wait_bounded(vfull(j & 1), (j >> 1) & 1)) return false;
        ptx::tc_fence_after();
        const uint32_t vb = sbase + kOffV + (j & 1) * kSlotBytes;
        const uint32_t wb = sbase + kOffW + (j & 1) * kWBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 cache rows in steps of 16
          const uint64_t da = ptx::umma_desc_sw128(vb + kk * 2048, kBox, 1024);
          const uint64_t db = ptx::umma_desc_sw128(wb + kk * 2048, kBox, 1024);
          ptx::umma_ss(tbase + kColO, da, db, kIdescValue, (!first || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(wfree(j & 1));
        ptx::umma_commit(vempty(j & 1));
        return true;
      };
      int it = 0, seg = 0, pend = -1;
      bool pend_first = false, ok = true;
      for (int b = b_first; b < B && s_pref[b] < t_end && ok; ++b) {
        const int ta = max(t_begin, dec::first_work(s_pref, b, setup)), tb = min(t_end, s_pref[b + 1]);
        if (ta >= tb) continue;
        for (int t = ta; t < tb; ++t, ++it) {
          if (*s_abort) {
            ok = false;
            break;
          }
          const bool first = t == ta;
          if (first) {
            if (pend >= 0 && !(ok = value_mma(pend, pend_first))) break;
            pend = -1;
            if (!(ok = ptx::mbar_wait_bounded(qready, seg & 1))) break;
          }
          if (!(ok = ptx::mbar_wait_bounded(kfull(it & 1), (it >> 1) & 1))) break;
          ptx::tc_fence_after();
          const uint32_t kb = sbase + kOffK + (it & 1) * kSlotBytes;
#pragma unroll
          for (int k = 0; k < 8; ++k) {  // K = 128 features in steps of 16
            const uint64_t da = ptx::umma_desc_sw128(kb + (k >> 2) * kBox + (k & 3) * 32, 16, 1024);
            const uint64_t db = ptx::umma_desc_sw128(sbase + kOffQ + (k >> 2) * kQBox + (k & 3) * 32, 16, 1024);
            ptx::umma_ss(tbase + 64u * (it & 1), da, db, kIdescScore, k > 0 ? 1u : 0u);
          }
          ptx::umma_commit(sfull(it & 1));
          ptx::umma_commit(kempty(it & 1));
          if (pend >= 0 && !(ok = value_mma(pend, pend_first))) break;
          pend = it;
          pend_first = first;
        }
        ++seg;
      }
      if (ok && pend >= 0) ok = value_mma(pend, pend_first);
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      // every MMA issued by this thread completes before TMEM can be released; TMEM is released
      // after the time limit all the same, with the error recorded
      ptx::umma_commit(fin);
      if (!ptx::mbar_wait_bounded(fin, 0)) atomicOr(p.err, kErrTimeout);
    } else if (blockIdx.x == 0 && p.ws_len) {
      record_lengths(lane - 1, 31);  // the other lanes of the MMA warp are idle
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quad = warp & 3;                // TMEM lanes 32 quad .. 32 quad + 31
    const int hh = (warp - 2) >> 2;           // heads 16 hh .. 16 hh + 15
    const int row = quad * 32 + lane;         // tile row for the scores, feature for O^T
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int wt = tid - 64;                  // 0 .. 255
    int it = 0;
    bool aborted = false;
    for (int b = b_first; b < B && s_pref[b] < t_end; ++b) {
      const int w0 = dec::first_work(s_pref, b, setup);
      const int ta = max(t_begin, w0), tb = min(t_end, s_pref[b + 1]);
      if (ta >= tb) continue;
      const int len_b = s_len[b];
      // ---- rotated query as bf16 hi (rows 0..31) and lo (rows 32..63), K-major, 128-byte swizzle.
      // This thread's 16 features of one head and the position are loaded together, first.  A
      // factorized query (section 解决思路: q = (1/R_Q) A_Q^T B_Q, RoPE on the B factor) is
      // combined from its unrotated rank rows in fp32 first and rotated once after, as a dense
      // query is: RoPE is linear, so RoPE((1/R_Q) sum_j A_Q[j] B_Q[j]) equals
      // (1/R_Q) sum_j A_Q[j] RoPE(B_Q[j]) (the same rounding count, in another order).
      {
        const int head = wt >> 3, f0 = (wt & 7) * 16;
        uint32_t hi[8], lo[8];
        float qf[16];
        uint4 qv[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};  // a dense query, raw until after the barrier
        if (p.r_q == 0) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) +
                                                            (static_cast<size_t>(b) * kH + head) * kD + f0);
          qv[0] = src[0];
          qv[1] = src[1];
        } else {
          // the rank rows are shared by all heads: each is loaded once, by 16 threads, as raw bf16
          // into the (idle) W buffers, A_Q / R_Q beside them
          const int jr = wt >> 4, c8 = (wt & 15) * 8;  // rank row, first feature of 8
          if (jr < p.r_q)
            reinterpret_cast<uint4*>(s_bqr + jr * kD)[c8 / 8] = *reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(p.q) + (static_cast<size_t>(b) * p.r_q + jr) * kD + c8);
          const int ja = wt >> 5;                       // A_Q: rank row ja, head (wt & 31)
          if (ja < p.r_q)
            s_aq[ja * kH + (wt & 31)] =
                __bfloat162float(static_cast<const __nv_bfloat16*>(p.a_q)[(static_cast<size_t>(b) * p.r_q + ja) * kH +
                                                                          (wt & 31)]) * p.inv_rq;
        }
        if (wt < kD / 2) {
          float cs, sn;
          rope_cos_sin(p.q_pos[b], p.rope.theta[wt], &cs, &sn);
          s_cs[2 * wt] = cs;
          s_cs[2 * wt + 1] = sn;
        }
        ptx::named_barrier(1, kSoftmaxThreads);
        if (p.r_q == 0) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const uint32_t w[4] = {qv[v].x, qv[v].y, qv[v].z, qv[v].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              qf[8 * v + 2 * k] = ptx::bf16_lo(w[k]);
              qf[8 * v + 2 * k + 1] = ptx::bf16_hi(w[k]);
            }
          }
        } else {
          // this thread's 16 features of its head: (1/R_Q) sum_j A_Q[j] B_Q[j], unrotated
#pragma unroll
          for (int e = 0; e < 16; ++e) qf[e] = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < p.r_q) {
              const float wq = s_aq[j * kH + head];
              const uint4* src = reinterpret_cast<const uint4*>(s_bqr + j * kD + f0);
#pragma unroll
              for (int v = 0; v < 2; ++v) {
                const uint4 rv = src[v];
                const uint32_t w[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  qf[8 * v + 2 * k] = fmaf(wq, ptx::bf16_lo(w[k]), qf[8 * v + 2 * k]);
                  qf[8 * v + 2 * k + 1] = fmaf(wq, ptx::bf16_hi(w[k]), qf[8 * v + 2 * k + 1]);
                }
              }
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int jp = f0 / 2 + e;  // RoPE pair (features 2 jp, 2 jp + 1)
          float x = qf[2 * e], y = qf[2 * e + 1];
          rope_pair(x, y, s_cs[2 * jp], s_cs[2 * jp + 1]);
          hi[e] = ptx::pack_bf16(x, y);
          lo[e] = ptx::pack_bf16(x - ptx::bf16_lo(hi[e]), y - ptx::bf16_hi(hi[e]));
        }
        uint8_t* qb = gbase + kOffQ + (f0 >> 6) * kQBox;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int chunk = ((f0 & 63) >> 3) + cc;
          const int sw = (chunk ^ (head & 7)) << 4;  // rows head and 32 + head share (row & 7)
          *reinterpret_cast<uint4*>(qb + head * 128 + sw) =
              make_uint4(hi[4 * cc], hi[4 * cc + 1], hi[4 * cc + 2], hi[4 * cc + 3]);
          *reinterpret_cast<uint4*>(qb + (32 + head) * 128 + sw) =
              make_uint4(lo[4 * cc], lo[4 * cc + 1], lo[4 * cc + 2], lo[4 * cc + 3]);
        }
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(qready);

      float m[kHalf], lsum[kHalf];
#pragma unroll
      for (int h = 0; h < kHalf; ++h) {
        m[h] = -INFINITY;
        lsum[h] = 0.f;
      }
      for (int t = ta; t < tb; ++t, ++it) {
        const int j = it, s = j & 1;
        bool fail = !ptx::mbar_wait_bounded(sfull(s), (j >> 1) & 1);
        if (!fail) fail = !ptx::mbar_wait_bounded(kfull(s), (j >> 1) & 1);
        if (fail) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
        ptx::tc_fence_after();
        const int tok0 = (t - w0) * TOK;
        const int valid_rows = min(kRows, (len_b - tok0) * R);
        const bool valid = row < valid_rows;
        // ---- 16 scores of this row: z[i] = (S_hi + S_lo) A_K scale/R_K, log2 units
        float z[kHalf];
        {
          float ak[kHalf];
          load_a_half(gbase + kOffK + s * kSlotBytes + kBBytes, row, hh, ak);
          uint32_t sh[kHalf], sl[kHalf];
          ptx::tmem_ld16(tbase + lane_off + 64u * s + kHalf * hh, sh);
          ptx::tmem_ld16(tbase + lane_off + 64u * s + 32 + kHalf * hh, sl);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHalf; ++h) z[h] = (__uint_as_float(sh[h]) + __uint_as_float(sl[h])) * ak[h];
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(kempty(s));  // A_K read, S(j) read
        if (R == 2) {
#pragma unroll
          for (int h = 0; h < kHalf; ++h) z[h] += __shfl_xor_sync(0xffffffffu, z[h], 1);  // ranks of one token
        }
        bool need = false;
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
          z[h] = valid ? z[h] * p.zs : -INFINITY;
          need |= z[h] > m[h] + kLazy;
        }
        const bool stop = fail || *s_abort != 0;
        if (ptx::named_barrier_or(1, kSoftmaxThreads, need || stop)) {
          if (ptx::named_barrier_or(2, kSoftmaxThreads, stop)) {
            aborted = true;
            break;  // every softmax thread leaves here together
          }
          // ---- new maxima: tile maximum per head over the CTA
          float v[kHalf];
#pragma unroll
          for (int h = 0; h < kHalf; ++h) v[h] = z[h];
          const float wmax = reduce_scatter16<true>(v, lane);
          if (lane < kHalf) s_red[quad * 32 + kHalf * hh + lane] = wmax;
          ptx::named_barrier(2, kSoftmaxThreads);
          float tmax[kHalf];
          combine_quadrants<true>(s_red, hh, tmax);
          float alpha[kHalf];
#pragma unroll
          for (int h = 0; h < kHalf; ++h) {
            const float mn = fmaxf(m[h], tmax[h]);
            alpha[h] = (m[h] == -INFINITY) ? 0.f : exp2f(m[h] - mn);
            m[h] = mn;
            lsum[h] *= alpha[h];
          }
          if (t > ta) {
            // O^T (this thread's feature lane, its 16 head columns of each half) by alpha,
            // once the value MMA of tile j - 1 has finished accumulating
            bool okw = ptx::mbar_wait_bounded(wfree((j - 1) & 1), ((j - 1) >> 1) & 1);
            if (__all_sync(0xffffffffu, okw)) {
              ptx::tc_fence_after();
#pragma unroll
              for (int part = 0; part < 2; ++part) {
                uint32_t o[kHalf];
                const uint32_t col = tbase + lane_off + kColO + 32 * part + kHalf * hh;
                ptx::tmem_ld16(col, o);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < kHalf; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
                ptx::tmem_st16(col, o);
              }
              ptx::tmem_wait_st();
            } else {
              atomicOr(p.err, kErrTimeout);
              *s_abort = 1;
            }
          }
        }
        // ---- W = p A_V / R_V as bf16 hi | lo into this row of W buffer s (MN-major, 128-byte
        // swizzle), once the V tile has landed and the value MMA of tile j - 2 has read the buffer
        {
          bool okv = ptx::mbar_wait_bounded(vfull(s), (j >> 1) & 1);
          if (okv && j >= 2) okv = ptx::mbar_wait_bounded(wfree(s), ((j >> 1) - 1) & 1);
          if (!okv) {
            atomicOr(p.err, kErrTimeout);
            *s_abort = 1;
          }
          float av[kHalf];
          load_a_half(gbase + kOffV + s * kSlotBytes + kBBytes, row, hh, av);
          uint32_t whi[kHalf / 2], wlo[kHalf / 2];
#pragma unroll
          for (int e = 0; e < kHalf / 2; ++e) {
            const int h0 = 2 * e, h1 = 2 * e + 1;
            const float p0 = exp2f(z[h0] - m[h0]);
            const float p1 = exp2f(z[h1] - m[h1]);
            lsum[h0] += p0;
            lsum[h1] += p1;
            const float w0 = valid ? p0 * av[h0] * p.inv_rv : 0.f;
            const float w1 = valid ? p1 * av[h1] * p.inv_rv : 0.f;
            whi[e] = ptx::pack_bf16(w0, w1);
            wlo[e] = ptx::pack_bf16(w0 - ptx::bf16_lo(whi[e]), w1 - ptx::bf16_hi(whi[e]));
          }
          uint8_t* wrow = gbase + kOffW + s * kWBytes + row * 128;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int chi = 2 * hh + cc, clo = 4 + 2 * hh + cc;
            *reinterpret_cast<uint4*>(wrow + ((chi ^ (row & 7)) << 4)) =
                make_uint4(whi[4 * cc], whi[4 * cc + 1], whi[4 * cc + 2], whi[4 * cc + 3]);
            *reinterpret_cast<uint4*>(wrow + ((clo ^ (row & 7)) << 4)) =
                make_uint4(wlo[4 * cc], wlo[4 * cc + 1], wlo[4 * cc + 2], wlo[4 * cc + 3]);
          }
          if (!valid) {
            // a B_V row past the sequence end may hold NaN, and 0 * NaN would reach every
            // feature: each of the row's two threads zeroes one 64-feature box of it
            uint8_t* vrow = gbase + kOffV + s * kSlotBytes + hh * kBox + row * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) *reinterpret_cast<uint4*>(vrow + cc * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(wready(s));
      }
      if (aborted) break;
      // ---- end of the segment: l per head over the CTA, then O^T / l or the partial state
      const float inv_r = 1.f / static_cast<float>(R);  // each token's p was added once per rank row
      const float lw = reduce_scatter16<false>(lsum, lane);
      ptx::named_barrier(1, kSoftmaxThreads);  // the last tile's maxima exchange has finished reading s_red
      if (lane < kHalf) s_red[quad * 32 + kHalf * hh + lane] = lw;
      ptx::named_barrier(1, kSoftmaxThreads);
      float l[kHalf];
      combine_quadrants<false>(s_red, hh, l);
#pragma unroll
      for (int h = 0; h < kHalf; ++h) l[h] *= inv_r;
      const int jl = it - 1;  // last tile of the segment
      const bool okf = ptx::mbar_wait_bounded(wfree(jl & 1), (jl >> 1) & 1);
      if (!__all_sync(0xffffffffu, okf)) {
        atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
        continue;  // the next tile barrier (or the kernel end) takes every warp out
      }
      ptx::tc_fence_after();
      uint32_t o0[kHalf], o1[kHalf];
      ptx::tmem_ld16(tbase + lane_off + kColO + kHalf * hh, o0);
      ptx::tmem_ld16(tbase + lane_off + kColO + 32 + kHalf * hh, o1);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      const bool whole = dec::owner_of(w0, NT, p.grid) == dec::owner_of(s_pref[b + 1] - 1, NT, p.grid);
      const int d = row;
      if (whole) {
        float* op = p.out + (static_cast<size_t>(b) * kH + kHalf * hh) * kD + d;
#pragma unroll
        for (int h = 0; h < kHalf; ++h) {
          const float o = __uint_as_float(o0[h]) + __uint_as_float(o1[h]);
          op[h * kD] = l[h] > 0.f ? o / l[h] : 0.f;
        }
        if (p.whole_ml && quad == 0 && lane < kHalf) {  // for the merge kernel: a step's token, or the lse
          float mk = m[0], lk = l[0];
#pragma unroll
          for (int h = 1; h < kHalf; ++h) {
            mk = lane == h ? m[h] : mk;
            lk = lane == h ? l[h] : lk;
          }
          const size_t e = (static_cast<size_t>(b) * kH + kHalf * hh + lane) * 2;
          p.whole_ml[e] = mk;
          p.whole_ml[e + 1] = lk;
        }
      } else {
        const int slot = 2 * c + (b == b_first ? 0 : 1);  // a shared sequence is the first or the last one
        float* op = p.ws_o + (static_cast<size_t>(slot) * kH + kHalf * hh) * kD + d;
#pragma unroll
        for (int h = 0; h < kHalf; ++h) op[h * kD] = __uint_as_float(o0[h]) + __uint_as_float(o1[h]);
        if (quad == 0 && lane < kHalf) {
          float mk = m[0], lk = l[0];
#pragma unroll
          for (int h = 1; h < kHalf; ++h) {
            mk = lane == h ? m[h] : mk;
            lk = lane == h ? l[h] : lk;
          }
          const size_t e = (static_cast<size_t>(slot) * kH + kHalf * hh + lane) * 2;
          p.ws_ml[e] = mk;
          p.ws_ml[e + 1] = lk;
        }
      }
    }
    ptx::tc_fence_before();
  }
  // The TMA and MMA warps ran their loops on lane 0 alone: reconverge them first, so that the
  // CTA barrier counts every thread and TMEM is released only after every role is done.
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tbase, kTmemCols);
  }
}

cudaError_t set_smem_once(int r) {
  static std::once_flag once[64][2];
  static cudaError_t status[64][2];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int k = r == 1 ? 0 : 1;
  std::call_once(once[dev][k], [dev, k]() {
    auto kern = k == 0 ? decode_umma_kernel<1> : decode_umma_kernel<2>;
    status[dev][k] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  });
  return status[dev][k];
}

}  // namespace

cudaError_t launch_decode_umma(const dec::DecodeTcParams& p, const CacheView& cv, cudaStream_t stream) {
  const uint64_t rows_k = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_k;
  const uint64_t rows_v = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_v;
  CUtensorMap tbk, tbv, tak, tav;
  cudaError_t e;
  if ((e = encode_bf16_2d(&tbk, cv.b_k, kD, rows_k, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tbv, cv.b_v, kD, rows_v, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tak, cv.a_k, kH, rows_k, kH, kRows, 64)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tav, cv.a_v, kH, rows_v, kH, kRows, 64)) != cudaSuccess) return e;
  if ((e = set_smem_once(cv.r_k)) != cudaSuccess) return e;
  auto kern = cv.r_k == 1 ? decode_umma_kernel<1> : decode_umma_kernel<2>;
  // programmatic dependent launch: the CTAs start (barriers, TMEM, tensor maps) while the
  // preceding kernel drains; the kernel waits for it before its first global access
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p, tbk, tbv, tak, tav);
}

}  // namespace tpa
