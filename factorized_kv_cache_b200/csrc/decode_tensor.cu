// Tensor-core decode attention over the factorized cache (bf16, h = 32,
// d_h = 128, R_K = R_V = R in {1, 2}).
//
// What it computes (Tensor Product Attention Is All You Need, sections
// 关键设计 and FlashTPA; K and V are never expanded): for each cached token s
// and head i,
//   S'[i, (s, r)] = q~_i . B~_K[s, r]                        (tensor cores)
//   z[i, s]       = scale/R_K * sum_r A_K[s, r, i] S'[i, (s, r)]
//   online softmax over s, p[i, s] = 2^(z log2e - m)
//   W[i, (s, r)]  = p[i, s] A_V[s, r, i] / R_V
//   O[i, :]      += sum_(s, r) W[i, (s, r)] B_V[s, r, :]     (tensor cores)
// The score contraction treats B_K rows as the shared "keys" of all 32 heads
// (M = heads, N = token rows, K = d_h); the value contraction uses W as the
// A operand (M = heads, K = token rows, N = d_h).  Both the rotated query
// and W are split into a bf16 high part and a bf16 remainder (two MMAs
// each), so they keep about 16 bits: a single bf16 rounding of W costs up to
// ~3e-3 relative error, and of the query as much once scores grow beyond the
// synthetic workloads' magnitude, against a 2e-3 budget.
//
// Data movement: one elected producer thread streams 64-row tiles of the
// four cache planes with TMA (cp.async.bulk.tensor, no multicast) into a
// 4-stage shared-memory ring guarded by mbarriers.  B tiles use the 128-byte
// swizzle and A tiles the 64-byte swizzle, which makes every ldmatrix of the
// consumers bank-conflict free.  Four consumer warps split each tile as
// 2 head halves x 2 row halves; their softmax states merge through shared
// memory whenever a sequence segment ends.
//
// Scheduling: the grid has G CTAs (one per SM by default).  The tiles of all
// sequences are laid end to end (sequence-major) and CTA c takes tiles
// [ceil(c NT / G), ceil((c+1) NT / G)): every CTA gets the same number of
// tiles to within one, whatever the length mix.  A sequence whose tiles all
// belong to one CTA is normalised and written directly.  Only the first and
// the last sequence of a CTA's range can be shared with other CTAs; their
// partial states (m, l, o) go to slots 2c and 2c+1, so the partials need
// 2G slots whatever the batch size.  A small merge kernel, launched with
// programmatic dependent launch, combines the partials of every other
// sequence by log-sum-exp.
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
using dec::owner_of;

constexpr int kRows = 64;                          // cache-plane rows per tile
constexpr int kStages = 2;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kBoxBytes = kRows * 128;             // 64 features x kRows rows, bf16
constexpr int kBBytes = 2 * kBoxBytes;             // one B tile (128 features)
constexpr int kABytes = kRows * kH * 2;            // one A tile
constexpr int kStageBytes = 2 * kBBytes + 2 * kABytes;
// Per-segment scratch: the rotated query as bf16 high and low parts
// ([2][32][128], 16 KB, swizzled for ldmatrix) while tiles are processed,
// then the row-half merge buffers (O[2][16][128] and (m, l)[2][16]) at the
// end of the segment.
constexpr int kMergeFloats = 2 * 16 * kD + 2 * 16 * 2;
constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + kMergeFloats * 4 + 2 * kStages * 8 +
                              (kMaxBatch + 1) * 4 + kMaxBatch * 4 + 64 * 4 + 64 * 2 * 4;
static_assert(2 * (kSmemBytes + 1024) <= 228 * 1024, "two CTAs per SM");
static_assert(2 * kH * kD * 2 <= 2 * 16 * kD * 4, "query hi + lo fit in the merge buffer");
constexpr unsigned kErrTimeout = 0x8u;

template <int R>
__global__ void __maxnreg__(168)  // 168 x 32 x 3 warps fit one SM sub-partition: two CTAs per SM
    decode_tc_kernel(const __grid_constant__ DecodeTcParams p, const __grid_constant__ CUtensorMap tm_bk,
                     const __grid_constant__ CUtensorMap tm_bv, const __grid_constant__ CUtensorMap tm_ak,
                     const __grid_constant__ CUtensorMap tm_av) {
  constexpr int TOK = kRows / R;  // tokens per tile
  extern __shared__ uint8_t smem_raw[];
  // the merge kernel may be scheduled now; it waits for this grid before reading
  ptx::pdl_launch_dependents();

  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  float* s_merge_o = reinterpret_cast<float*>(gbase + kStages * kStageBytes);  // [2][16][128]
  const uint32_t s_q = sbase + kStages * kStageBytes;  // rotated query, aliases s_merge_o during a segment
  float* s_merge_ml = s_merge_o + 2 * 16 * kD;                                  // [2][16][2]
  uint64_t* s_bar = reinterpret_cast<uint64_t*>(s_merge_ml + 2 * 16 * 2);      // full[kStages], empty[kStages]
  int32_t* s_pref = reinterpret_cast<int32_t*>(s_bar + 2 * kStages);           // [kMaxBatch + 1]
  int32_t* s_len = s_pref + kMaxBatch + 1;                                     // [kMaxBatch]
  int32_t* s_tmp = s_len + kMaxBatch;                                          // [32] scan scratch
  volatile int* s_abort = s_tmp + 32;                                          // set by a warp that timed out
  float* s_cs = reinterpret_cast<float*>(s_tmp + 64);                          // [64][2] cos, sin of the query
  const uint32_t bar_full = ptx::smem_u32(s_bar);
  const uint32_t bar_empty = bar_full + 8 * kStages;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(bar_full + 8 * s, 1);
      ptx::mbar_init(bar_empty + 8 * s, kConsumerWarps);
    }
    *s_abort = 0;
    ptx::fence_barrier_init();
  }
  dec::build_prefix<TOK, kThreads>(p, s_pref, s_len, s_tmp);  // ends with __syncthreads
  const int B = p.batch;
  const int NT = s_pref[B];
  if (blockIdx.x == 0)
    for (int b = tid; b <= B; b += kThreads) p.ws_prefix[b] = s_pref[b];
  if (NT == 0) return;
  const int c = blockIdx.x;
  const int t_begin = dec::first_tile(c, NT, p.grid);
  const int t_end = dec::first_tile(c + 1, NT, p.grid);
  if (t_begin >= t_end) return;
  // first sequence with tiles in [t_begin, ...): largest b with s_pref[b] <= t_begin and s_pref[b+1] > t_begin
  const int b_first = dec::sequence_of_tile(s_pref, B, t_begin);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_bk);
      ptx::prefetch_tmap(&tm_bv);
      ptx::prefetch_tmap(&tm_ak);
      ptx::prefetch_tmap(&tm_av);
      int it = 0;
      bool ok = true;
      for (int b = b_first; b < B && s_pref[b] < t_end && ok; ++b) {
        const int ta = max(t_begin, s_pref[b]), tb = min(t_end, s_pref[b + 1]);
        for (int t = ta; t < tb; ++t, ++it) {
          const int stage = it % kStages;
          const uint32_t par = ((it / kStages) & 1) ^ 1;
          if (!ptx::mbar_wait_bounded(bar_empty + 8 * stage, par)) {
            atomicOr(p.err, kErrTimeout);
            ok = false;
            break;
          }
          const int row0 = (b * p.capacity + (t - s_pref[b]) * TOK) * R;
          const uint32_t st = sbase + stage * kStageBytes;
          const uint32_t fb = bar_full + 8 * stage;
          ptx::mbar_arrive_expect_tx(fb, kStageBytes);
          ptx::tma_load_2d(st, &tm_bk, 0, row0, fb);
          ptx::tma_load_2d(st + kBoxBytes, &tm_bk, 64, row0, fb);
          ptx::tma_load_2d(st + kBBytes, &tm_bv, 0, row0, fb);
          ptx::tma_load_2d(st + kBBytes + kBoxBytes, &tm_bv, 64, row0, fb);
          ptx::tma_load_2d(st + 2 * kBBytes, &tm_ak, 0, row0, fb);
          ptx::tma_load_2d(st + 2 * kBBytes + kABytes, &tm_av, 0, row0, fb);
        }
      }
      if (!ok) {
        // drain: let every load already issued land before the CTA can exit
        for (int k = max(0, it - kStages); k < it; ++k)
          ptx::mbar_wait_bounded(bar_full + 8 * (k % kStages), (k / kStages) & 1);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int hh = warp & 1;   // head half: heads 16*hh .. 16*hh+15
  const int rh = warp >> 1;  // row half: rows 32*rh .. 32*rh+31 of every tile
  const int g = lane >> 2, q4 = lane & 3;
  const int r0 = rh * 32;
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: matrix index, row within matrix
  int it = 0;

  for (int b = b_first; b < B && s_pref[b] < t_end; ++b) {
    const int ta = max(t_begin, s_pref[b]), tb = min(t_end, s_pref[b + 1]);
    if (ta >= tb) continue;
    const int len_b = s_len[b];
    // ---- rotated query fragments for this sequence (bf16, A operand of the score MMA)
    if (tid < kD / 2) {
      float cs, sn;
      rope_cos_sin(p.q_pos[b], p.rope.theta[tid], &cs, &sn);
      s_cs[2 * tid] = cs;
      s_cs[2 * tid + 1] = sn;
    }
    ptx::named_barrier(1, kConsumerWarps * 32);
    {
      // q~ = hi + lo, each as bf16 rows of 256 B with 16-byte chunks XOR-swizzled by (row & 7)
      // within each 128-byte half; the lo plane follows the hi plane (8 KB)
      const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) + static_cast<size_t>(b) * kH * kD;
      uint8_t* sq = gbase + kStages * kStageBytes;
      for (int e = tid; e < kH * kD / 2; e += kConsumerWarps * 32) {
        const int head = e / (kD / 2), j = e % (kD / 2);  // RoPE pair j = features (2j, 2j+1)
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(qb + head * kD + 2 * j);
        float x = __bfloat162float(v.x), y = __bfloat162float(v.y);
        rope_pair(x, y, s_cs[2 * j], s_cs[2 * j + 1]);
        const int c = j >> 2;
        const int pc = (c & 8) | ((c & 7) ^ (head & 7));
        const uint32_t hi = ptx::pack_bf16(x, y);
        const uint32_t lo = ptx::pack_bf16(x - ptx::bf16_lo(hi), y - ptx::bf16_hi(hi));
        *reinterpret_cast<uint32_t*>(sq + head * 256 + pc * 16 + (j & 3) * 4) = hi;
        *reinterpret_cast<uint32_t*>(sq + kH * kD * 2 + head * 256 + pc * 16 + (j & 3) * 4) = lo;
      }
    }
    ptx::named_barrier(1, kConsumerWarps * 32);
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    float O[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) O[n][0] = O[n][1] = O[n][2] = O[n][3] = 0.f;

    for (int t = ta; t < tb; ++t, ++it) {
      const int stage = it % kStages;
      if (*s_abort) break;
      if (!ptx::mbar_wait_bounded(bar_full + 8 * stage, (it / kStages) & 1)) {
        if (lane == 0) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
        break;
      }
      const uint32_t st = sbase + stage * kStageBytes;
      const uint32_t s_bk = st, s_bv = st + kBBytes, s_ak = st + 2 * kBBytes, s_av = s_ak + kABytes;
      const int tok0 = (t - s_pref[b]) * TOK;        // first token of the tile
      const int valid_rows = min(kRows, (len_b - tok0) * R);
      const bool partial = valid_rows < kRows;

      // ---- scores S'[head][row] for the warp's 32 rows (4 n-tiles of 8)
      float S[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
#pragma unroll
      for (int kk2 = 0; kk2 < 4; ++kk2) {
        const int box = kk2 >> 1;
        const int chunk = (kk2 & 1) * 4 + mi;
        uint32_t bf[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          const int row = r0 + nt * 8 + rr;
          const uint32_t addr = s_bk + box * kBoxBytes + row * 128 + ((chunk ^ (row & 7)) << 4);
          ptx::ldsm_x4(addr, bf[nt][0], bf[nt][1], bf[nt][2], bf[nt][3]);
        }
        // query fragments of k-steps 2*kk2 and 2*kk2+1 (A operand: heads x 16 features), high then
        // low plane; four independent accumulators between two MMAs into the same one
#pragma unroll
        for (int plane = 0; plane < 2; ++plane) {
          uint32_t qa[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int qrow = hh * 16 + (mi & 1) * 8 + rr;
            const int c = (2 * kk2 + u) * 2 + (mi >> 1);
            const int pc = (c & 8) | ((c & 7) ^ (qrow & 7));
            ptx::ldsm_x4(s_q + plane * (kH * kD * 2) + qrow * 256 + pc * 16, qa[u][0], qa[u][1], qa[u][2], qa[u][3]);
          }
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) ptx::mma_bf16(S[nt], qa[0], bf[nt][0], bf[nt][1]);
#pragma unroll
          for (int nt = 0; nt < 4; ++nt) ptx::mma_bf16(S[nt], qa[1], bf[nt][2], bf[nt][3]);
        }
      }
      // ---- head factors A_K, A_V in the accumulator layout (ldmatrix.trans)
      uint32_t akf[4][2], avf[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int row = r0 + np * 16 + (mi >> 1) * 8 + rr;
        const int chunk = 2 * hh + (mi & 1);
        const uint32_t off = row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4);
        ptx::ldsm_x4_t(s_ak + off, akf[2 * np][0], akf[2 * np][1], akf[2 * np + 1][0], akf[2 * np + 1][1]);
        ptx::ldsm_x4_t(s_av + off, avf[2 * np][0], avf[2 * np][1], avf[2 * np + 1][0], avf[2 * np + 1][1]);
      }
      // ---- z = scale/R_K * sum_r A_K S' (log2 units), masked past the sequence end
      // R == 1: z[nt][j] j = 0,1 head g (rows 2q4+j), j = 2,3 head g+8
      // R == 2: z[nt][0] head g, z[nt][2] head g+8 (one token per n-tile)
      float z[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const int rowc = r0 + nt * 8 + 2 * q4;  // plane row of column 2*q4
        if (R == 1) {
          z[nt][0] = S[nt][0] * ptx::bf16_lo(akf[nt][0]) * p.zs;
          z[nt][1] = S[nt][1] * ptx::bf16_hi(akf[nt][0]) * p.zs;
          z[nt][2] = S[nt][2] * ptx::bf16_lo(akf[nt][1]) * p.zs;
          z[nt][3] = S[nt][3] * ptx::bf16_hi(akf[nt][1]) * p.zs;
          if (partial) {
            if (rowc >= valid_rows) z[nt][0] = z[nt][2] = -INFINITY;
            if (rowc + 1 >= valid_rows) z[nt][1] = z[nt][3] = -INFINITY;
          }
        } else {
          z[nt][0] = (S[nt][0] * ptx::bf16_lo(akf[nt][0]) + S[nt][1] * ptx::bf16_hi(akf[nt][0])) * p.zs;
          z[nt][2] = (S[nt][2] * ptx::bf16_lo(akf[nt][1]) + S[nt][3] * ptx::bf16_hi(akf[nt][1])) * p.zs;
          if (partial && rowc >= valid_rows) z[nt][0] = z[nt][2] = -INFINITY;
          z[nt][1] = z[nt][0];
          z[nt][3] = z[nt][2];
        }
      }
      // ---- online softmax per head row (the quad of lanes sharing g holds one head)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        mx[0] = fmaxf(mx[0], fmaxf(z[nt][0], z[nt][1]));
        mx[1] = fmaxf(mx[1], fmaxf(z[nt][2], z[nt][3]));
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 1));
        mx[hr] = fmaxf(mx[hr], __shfl_xor_sync(0xffffffffu, mx[hr], 2));
      }
      float alpha[2], mn[2];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        mn[hr] = fmaxf(m[hr], mx[hr]);
        alpha[hr] = (mn[hr] == -INFINITY) ? 1.f : exp2f(m[hr] - mn[hr]);
        m[hr] = mn[hr];
        l[hr] *= alpha[hr];
      }
      if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          O[n][0] *= alpha[0];
          O[n][1] *= alpha[0];
          O[n][2] *= alpha[1];
          O[n][3] *= alpha[1];
        }
      }
      // ---- W = p A_V / R_V as hi + lo bf16 pairs (A operand of the value MMA)
      float w[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        const float p0 = (mn[0] == -INFINITY) ? 0.f : exp2f(z[nt][0] - mn[0]);
        const float p2 = (mn[1] == -INFINITY) ? 0.f : exp2f(z[nt][2] - mn[1]);
        if (R == 1) {
          const float p1 = (mn[0] == -INFINITY) ? 0.f : exp2f(z[nt][1] - mn[0]);
          const float p3 = (mn[1] == -INFINITY) ? 0.f : exp2f(z[nt][3] - mn[1]);
          l[0] += p0 + p1;
          l[1] += p2 + p3;
          w[nt][0] = p0 * ptx::bf16_lo(avf[nt][0]);
          w[nt][1] = p1 * ptx::bf16_hi(avf[nt][0]);
          w[nt][2] = p2 * ptx::bf16_lo(avf[nt][1]);
          w[nt][3] = p3 * ptx::bf16_hi(avf[nt][1]);
          if (partial) {
            const int rowc = r0 + nt * 8 + 2 * q4;
            if (rowc >= valid_rows) w[nt][0] = w[nt][2] = 0.f;
            if (rowc + 1 >= valid_rows) w[nt][1] = w[nt][3] = 0.f;
          }
        } else {
          l[0] += p0;
          l[1] += p2;
          w[nt][0] = 0.5f * p0 * ptx::bf16_lo(avf[nt][0]);
          w[nt][1] = 0.5f * p0 * ptx::bf16_hi(avf[nt][0]);
          w[nt][2] = 0.5f * p2 * ptx::bf16_lo(avf[nt][1]);
          w[nt][3] = 0.5f * p2 * ptx::bf16_hi(avf[nt][1]);
          if (partial && r0 + nt * 8 + 2 * q4 >= valid_rows) w[nt][0] = w[nt][1] = w[nt][2] = w[nt][3] = 0.f;
        }
      }
      // ---- O += W B_V over the warp's 32 rows (two k-chunks of 16 rows)
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
        uint32_t ahi[4], alo[4];
        {
          const float* w0 = w[2 * kc];
          const float* w1 = w[2 * kc + 1];
          ahi[0] = ptx::pack_bf16(w0[0], w0[1]);
          ahi[1] = ptx::pack_bf16(w0[2], w0[3]);
          ahi[2] = ptx::pack_bf16(w1[0], w1[1]);
          ahi[3] = ptx::pack_bf16(w1[2], w1[3]);
          alo[0] = ptx::pack_bf16(w0[0] - ptx::bf16_lo(ahi[0]), w0[1] - ptx::bf16_hi(ahi[0]));
          alo[1] = ptx::pack_bf16(w0[2] - ptx::bf16_lo(ahi[1]), w0[3] - ptx::bf16_hi(ahi[1]));
          alo[2] = ptx::pack_bf16(w1[0] - ptx::bf16_lo(ahi[2]), w1[1] - ptx::bf16_hi(ahi[2]));
          alo[3] = ptx::pack_bf16(w1[2] - ptx::bf16_lo(ahi[3]), w1[3] - ptx::bf16_hi(ahi[3]));
        }
        const int krow = r0 + kc * 16;
        // rows of this lane's B fragment elements (for masking a partial tile)
        const int vr0 = krow + 2 * q4, vr1 = krow + 8 + 2 * q4;
        // zero B_V elements of rows past the end (they may hold NaN; 0 * NaN would poison O)
        const uint32_t m0 = partial ? ((vr0 < valid_rows ? 0x0000ffffu : 0u) | (vr0 + 1 < valid_rows ? 0xffff0000u : 0u))
                                    : 0xffffffffu;
        const uint32_t m1 = partial ? ((vr1 < valid_rows ? 0x0000ffffu : 0u) | (vr1 + 1 < valid_rows ? 0xffff0000u : 0u))
                                    : 0xffffffffu;
#pragma unroll
        for (int g4 = 0; g4 < 2; ++g4) {
          uint32_t v[4][4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int nd2 = g4 * 4 + u;
            const int row = krow + (mi & 1) * 8 + rr;
            const int d0 = nd2 * 16 + (mi >> 1) * 8;
            const uint32_t addr = s_bv + (d0 >> 6) * kBoxBytes + row * 128 + ((((d0 & 63) >> 3) ^ (row & 7)) << 4);
            ptx::ldsm_x4_t(addr, v[u][0], v[u][1], v[u][2], v[u][3]);
            v[u][0] &= m0;
            v[u][2] &= m0;
            v[u][1] &= m1;
            v[u][3] &= m1;
          }
          // eight independent accumulators between the hi and the lo MMA of each
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ptx::mma_bf16(O[2 * (g4 * 4 + u)], ahi, v[u][0], v[u][1]);
            ptx::mma_bf16(O[2 * (g4 * 4 + u) + 1], ahi, v[u][2], v[u][3]);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            ptx::mma_bf16(O[2 * (g4 * 4 + u)], alo, v[u][0], v[u][1]);
            ptx::mma_bf16(O[2 * (g4 * 4 + u) + 1], alo, v[u][2], v[u][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_empty + 8 * stage);
    }

    // ---- end of this sequence's segment: merge row halves, write the result
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      l[hr] += __shfl_xor_sync(0xffffffffu, l[hr], 1);
      l[hr] += __shfl_xor_sync(0xffffffffu, l[hr], 2);
    }
    float* mo = s_merge_o + hh * 16 * kD;
    float* mml = s_merge_ml + hh * 32;
    ptx::named_barrier(1, kConsumerWarps * 32);  // every warp is done with the query (same bytes)
    if (rh == 1) {
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const int d = n * 8 + 2 * q4;
        *reinterpret_cast<float2*>(mo + g * kD + d) = make_float2(O[n][0], O[n][1]);
        *reinterpret_cast<float2*>(mo + (g + 8) * kD + d) = make_float2(O[n][2], O[n][3]);
      }
      if (q4 == 0) {
        mml[2 * g] = m[0];
        mml[2 * g + 1] = l[0];
        mml[2 * (g + 8)] = m[1];
        mml[2 * (g + 8) + 1] = l[1];
      }
    }
    ptx::named_barrier(1, kConsumerWarps * 32);
    if (rh == 0) {
      float M[2], Lt[2], f0[2], f1[2];
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int hrow = g + 8 * hr;
        const float m1 = mml[2 * hrow], l1 = mml[2 * hrow + 1];
        M[hr] = fmaxf(m[hr], m1);
        f0[hr] = (m[hr] == -INFINITY) ? 0.f : exp2f(m[hr] - M[hr]);
        f1[hr] = (m1 == -INFINITY) ? 0.f : exp2f(m1 - M[hr]);
        Lt[hr] = l[hr] * f0[hr] + l1 * f1[hr];
      }
      const bool whole = owner_of(s_pref[b], NT, p.grid) == owner_of(s_pref[b + 1] - 1, NT, p.grid);
      const int slot = 2 * c + (b == b_first ? 0 : 1);  // a shared sequence is the first or the last one
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        const int d = n * 8 + 2 * q4;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int hrow = g + 8 * hr;
          const float2 o1 = *reinterpret_cast<const float2*>(mo + hrow * kD + d);
          float x = O[n][2 * hr] * f0[hr] + o1.x * f1[hr];
          float y = O[n][2 * hr + 1] * f0[hr] + o1.y * f1[hr];
          const int head = hh * 16 + hrow;
          if (whole) {
            const float inv = Lt[hr] > 0.f ? 1.f / Lt[hr] : 0.f;
            *reinterpret_cast<float2*>(p.out + (static_cast<size_t>(b) * kH + head) * kD + d) =
                make_float2(x * inv, y * inv);
          } else {
            *reinterpret_cast<float2*>(p.ws_o + (static_cast<size_t>(slot) * kH + head) * kD + d) =
                make_float2(x, y);
          }
        }
      }
      if (!whole && q4 == 0) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int head = hh * 16 + g + 8 * hr;
          p.ws_ml[(static_cast<size_t>(slot) * kH + head) * 2] = M[hr];
          p.ws_ml[(static_cast<size_t>(slot) * kH + head) * 2 + 1] = Lt[hr];
        }
      }
    }
    ptx::named_barrier(1, kConsumerWarps * 32);  // merge buffer free for the next segment
    if (*s_abort) break;  // every consumer warp sees the same flag after the barrier
  }
}

// LSE merge of the partials of every sequence split across CTAs.  One CTA per
// (sequence, head).  The touched CTAs of sequence b are cs..ce; when every CTA
// owns at least one tile (G <= NT) they all touched b, b is the first sequence
// of each of them but possibly cs, and only cs needs a division.  The (m, l)
// pairs are reduced across the CTA; the features are then summed by partial
// groups of 32 threads (one float4 column per thread), each thread with
// kMergeBatch partial loads in flight at once: 8 groups of 4 for 256 threads,
// and for a batch of one or two sequences (each split over ~150 CTAs) 32 groups
// of 5, so that all of a long sequence's partials arrive in one L2 round trip.
//
// Decode step (kStep): the token being generated (its factors and its query,
// section 解决思路: Q_t, K_t, V_t all come from x_t) is appended and attended
// in the same two launches.  It enters the log-sum-exp as one more partial
// state (m = its own score z_t, l = 1, o = V_t), so the split kernel reads only
// the tokens cached before the step and never waits on the new slot.  Its score
// and value are formed here before the wait on the split kernel, from inputs
// that earlier work wrote (the split kernel lets this grid start only once all
// of its CTAs are past their own wait): the new B_K row and the query are
// rotated at the step's position (Theorem 3.1), the row rounded to bf16 exactly
// as an append stores it.  After the wait the (sequence, head 0) CTA stores the
// token in slot L = the length the split kernel saw and, if asked, sets the
// length to L + 1.  These CTAs start as the split kernel's CTAs leave their SMs,
// so the work before the wait mostly overlaps the split kernel's tail.
struct TcStepParams {
  const int32_t* pos;             // [B] position of the step's token (its key and its query)
  const __nv_bfloat16* a_k;       // new token [B][R][32], B_K [B][R][128] unrotated, A_V, B_V
  const __nv_bfloat16* b_k;
  const __nv_bfloat16* a_v;
  const __nv_bfloat16* b_v;
  const __nv_bfloat16* q;         // dense query [B][32][128], or B_Q [B][r_q][128]
  const __nv_bfloat16* a_q;       // A_Q [B][r_q][32] when r_q > 0
  int r_q;
  float inv_rq;
  int r;                          // R_K = R_V
  float zs;                       // scale * log2(e) / R_K
  float inv_rv;
  int capacity;
  int advance;
  const int32_t* ws_len;          // lengths the split kernel saw (-1: out of range)
  __nv_bfloat16* c_ak;            // the cache planes and lengths
  __nv_bfloat16* c_bk;
  __nv_bfloat16* c_av;
  __nv_bfloat16* c_bv;
  int32_t* seq_lens;
  unsigned int* err;
  RopeTable rope;
};

struct TcMergeParams {
  int batch, grid;
  int setup;               // set-up units before each non-empty sequence's tiles (the split kernel's)
  const int32_t* prefix;
  const float* ws_ml;
  const float* ws_o;
  float* out;
  float* lse;              // [B][32] natural-log log-sum-exp of the scaled scores, or null
  const float* whole_ml;   // (m, l) of the sequences the split kernel finished inside one CTA
  TcStepParams st;         // read only by the step variant
};

constexpr float kLn2 = 0.6931471805599453f;

// Threads of a merge CTA: 256 for most batches; 1024 when a batch of one or two sequences
// spreads each over ~150 CTAs of the split kernel, so that one pass loads every partial.
constexpr int kMergeThreadsSmallBatch = 1024;
constexpr int kMergeMax = 1024;  // partials per pass

// Block-wide max or sum over NT / 32 warps.  The warps' values meet in s_red and every warp
// reduces them itself, so the result reaches all threads after one barrier past the write.
template <int NT>
__device__ __forceinline__ float merge_reduce(float v, bool is_max, float* s_red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, w) : v + w;
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
  __syncthreads();
  if constexpr (NT <= 256) {  // a few warps: read their values in turn
    v = s_red[0];
#pragma unroll
    for (int k = 1; k < NT / 32; ++k) v = is_max ? fmaxf(v, s_red[k]) : v + s_red[k];
  } else {  // up to 32 warps: one value per lane, then a shuffle tree
    const int lane = threadIdx.x & 31;
    v = lane < NT / 32 ? s_red[lane] : (is_max ? -INFINITY : 0.f);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float w = __shfl_xor_sync(0xffffffffu, v, o);
      v = is_max ? fmaxf(v, w) : v + w;
    }
  }
  return v;
}

template <bool kStep, int kMergeThreads>
__global__ void __launch_bounds__(kMergeThreads) decode_tc_merge_kernel(const __grid_constant__ TcMergeParams p) {
  constexpr int kMergeGroups = kMergeThreads / 32;
  constexpr int kMergeBatch = kMergeThreads >= 1024 ? 5 : 4;  // 32 x 5 partials in one pass
  // the next decode may start its set-up on SMs this grid frees; it waits for this grid to
  // complete before it touches memory
  ptx::pdl_launch_dependents();
  __shared__ float s_w[kMergeMax];
  __shared__ int s_slot[kMergeMax];
  __shared__ float s_red[kMergeThreads / 32];
  __shared__ float4 s_acc[kMergeGroups][32];
  const int b = blockIdx.x, i = blockIdx.y, tid = threadIdx.x;
  const int f4 = tid & 31, grp = tid >> 5;  // float4 column, partial group

  // ---- the step's token for head i: score z_t (log2 units, warps 0-1) and value V_t (columns
  // 4 f4 .. 4 f4 + 3, warp kVnWarp), both chains' loads issued at once
  constexpr int kVnWarp = 2;
  const bool vn_warp = (tid >> 5) == kVnWarp;
  float zn = 0.f;
  float4 vn = make_float4(0.f, 0.f, 0.f, 0.f);
  uint32_t bkr[2] = {0u, 0u};  // rotated B_K pair 2 tid, 2 tid + 1 of rank rows 0, 1 (bf16 x 2), tid < 64
  uint32_t word = 0u;          // one 4-byte word of the token's A_K | A_V | B_V, head-0 CTA, tid >= 64
  __shared__ float s_dot[2];
  if constexpr (kStep) {
    const TcStepParams& st = p.st;
    const int R = st.r;
    if (tid < 64) {
      float ak[2] = {0.f, 0.f};
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (r < R) ak[r] = __bfloat162float(st.a_k[(static_cast<size_t>(b) * R + r) * kH + i]);
      const int pos = st.pos[b];
      __nv_bfloat162 kk[2], qq[8];
      float aq[8];
#pragma unroll
      for (int r = 0; r < 2; ++r)
        if (r < R) kk[r] = reinterpret_cast<const __nv_bfloat162*>(st.b_k + (static_cast<size_t>(b) * R + r) * kD)[tid];
      if (st.r_q == 0) {
        qq[0] = reinterpret_cast<const __nv_bfloat162*>(st.q + (static_cast<size_t>(b) * kH + i) * kD)[tid];
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < st.r_q) {
            const size_t row = static_cast<size_t>(b) * st.r_q + j;
            qq[j] = reinterpret_cast<const __nv_bfloat162*>(st.q + row * kD)[tid];
            aq[j] = __bfloat162float(st.a_q[row * kH + i]);
          }
        }
      }
      float c, sn;
      rope_cos_sin(pos, st.rope.theta[tid], &c, &sn);
      float qx = 0.f, qy = 0.f;
      if (st.r_q == 0) {
        qx = __low2float(qq[0]);
        qy = __high2float(qq[0]);
        rope_pair(qx, qy, c, sn);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < st.r_q) {
            float x = __low2float(qq[j]), y = __high2float(qq[j]);
            rope_pair(x, y, c, sn);
            qx = fmaf(aq[j], x, qx);
            qy = fmaf(aq[j], y, qy);
          }
        }
        qx *= st.inv_rq;
        qy *= st.inv_rq;
      }
      float dot = 0.f;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r < R) {
          float x = __low2float(kk[r]), y = __high2float(kk[r]);
          rope_pair(x, y, c, sn);
          __nv_bfloat162 kr = __floats2bfloat162_rn(x, y);  // the stored row
          bkr[r] = *reinterpret_cast<uint32_t*>(&kr);
          dot = fmaf(ak[r], fmaf(qx, __low2float(kr), qy * __high2float(kr)), dot);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      if ((tid & 31) == 0) s_dot[tid >> 5] = dot;
    } else if (vn_warp) {
      float av[2] = {0.f, 0.f};
      uint2 raw[2] = {make_uint2(0u, 0u), make_uint2(0u, 0u)};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r < R) {
          const size_t row = static_cast<size_t>(b) * R + r;
          av[r] = __bfloat162float(st.a_v[row * kH + i]);
          raw[r] = reinterpret_cast<const uint2*>(st.b_v + row * kD)[f4];
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        if (r < R) {
          const float a = av[r] * st.inv_rv;
          const __nv_bfloat162 v01 = *reinterpret_cast<const __nv_bfloat162*>(&raw[r].x);
          const __nv_bfloat162 v23 = *reinterpret_cast<const __nv_bfloat162*>(&raw[r].y);
          vn.x = fmaf(a, __low2float(v01), vn.x);
          vn.y = fmaf(a, __high2float(v01), vn.y);
          vn.z = fmaf(a, __low2float(v23), vn.z);
          vn.w = fmaf(a, __high2float(v23), vn.w);
        }
      }
    }
    if (blockIdx.y == 0 && tid >= 64) {
      const int w = tid - 64, na = R * kH / 2, nb = R * kD / 2;  // 4-byte words per plane
      if (w < na) word = reinterpret_cast<const uint32_t*>(st.a_k + static_cast<size_t>(b) * R * kH)[w];
      else if (w < 2 * na) word = reinterpret_cast<const uint32_t*>(st.a_v + static_cast<size_t>(b) * R * kH)[w - na];
      else if (w < 2 * na + nb)
        word = reinterpret_cast<const uint32_t*>(st.b_v + static_cast<size_t>(b) * R * kD)[w - 2 * na];
    }
    __syncthreads();
    zn = (s_dot[0] + s_dot[1]) * st.zs;
  }

  ptx::pdl_wait();  // the split kernel's partials, outputs and recorded lengths

  // everything the merge reads first, loaded together
  const int NT = p.prefix[p.batch];
  const int t0 = p.prefix[b], t1 = p.prefix[b + 1];
  bool nv = false;  // the step's token is attended
  if constexpr (kStep) {
    const TcStepParams& st = p.st;
    const int R = st.r;
    const int L = st.ws_len[b];
    nv = L >= 0 && L < st.capacity;
    if (blockIdx.y == 0) {
      if (nv) {
        const size_t tok = (static_cast<size_t>(b) * st.capacity + L) * R;  // first rank row of slot L
        if (tid < 64) {
          for (int r = 0; r < R; ++r) reinterpret_cast<uint32_t*>(st.c_bk + (tok + r) * kD)[tid] = bkr[r];
        } else {
          const int w = tid - 64, na = R * kH / 2, nb = R * kD / 2;
          if (w < na) reinterpret_cast<uint32_t*>(st.c_ak + tok * kH)[w] = word;
          else if (w < 2 * na) reinterpret_cast<uint32_t*>(st.c_av + tok * kH)[w - na] = word;
          else if (w < 2 * na + nb) reinterpret_cast<uint32_t*>(st.c_bv + tok * kD)[w - 2 * na] = word;
        }
        if (tid == 0 && st.advance) st.seq_lens[b] = L + 1;
      } else if (tid == 0 && L >= 0) {
        atomicOr(st.err, TPA_DEVERR_APPEND_OVERFLOW);  // the cache is full: the token is neither stored nor attended
      }
    }
  }

  float* o = p.out + (static_cast<size_t>(b) * kH + i) * kD;
  float* lse = p.lse ? p.lse + static_cast<size_t>(b) * kH + i : nullptr;
  // natural-log log-sum-exp from a maximum and a sum in log2 units
  auto write_lse = [&](float m2, float l) {
    if (lse && tid == 0) *lse = l > 0.f ? (m2 + log2f(l)) * kLn2 : -INFINITY;
  };
  if (t1 <= t0) {  // nothing cached: the step's token alone, or zeros
    if (vn_warp) reinterpret_cast<float4*>(o)[f4] = nv ? vn : make_float4(0.f, 0.f, 0.f, 0.f);
    write_lse(nv ? zn : 0.f, nv ? 1.f : 0.f);
    return;
  }
  const int setup = p.setup > 0 ? p.prefix[p.batch + 1] : 0;  // the set-up units the split kernel charged
  const int w0 = t0 + setup;  // the sequence's first tile unit (it is not empty here)
  const int cs = owner_of(w0, NT, p.grid), ce = owner_of(t1 - 1, NT, p.grid);
  if (cs == ce) {  // finished by the split kernel
    if (nv || lse) {
      const float2 ml = reinterpret_cast<const float2*>(p.whole_ml)[static_cast<size_t>(b) * kH + i];
      const float M = nv ? fmaxf(ml.x, zn) : ml.x;
      const float wo = (ml.x == -INFINITY ? 0.f : exp2f(ml.x - M)) * ml.y;
      const float wn = nv ? exp2f(zn - M) : 0.f;
      if (nv && vn_warp) {
        const float4 on = reinterpret_cast<const float4*>(o)[f4];
        const float inv = 1.f / (wo + wn);
        reinterpret_cast<float4*>(o)[f4] = make_float4((on.x * wo + vn.x * wn) * inv, (on.y * wo + vn.y * wn) * inv,
                                                        (on.z * wo + vn.z * wn) * inv, (on.w * wo + vn.w * wn) * inv);
      }
      write_lse(M, wo + wn);
    }
    return;
  }
  const int n = ce - cs + 1;
  const bool dense = p.grid <= NT;
  const bool cs_first = dec::first_tile(cs, NT, p.grid) >= t0;
  // slot (in units of [slot][head]) of CTA cs + u for this sequence, -1 if it did not touch it
  auto slot_of = [&](int u) -> int {
    const int cc = cs + u;
    if (dense) return (2 * cc + ((u > 0 || cs_first) ? 0 : 1)) * kH + i;
    const int a = dec::first_tile(cc, NT, p.grid), e = dec::first_tile(cc + 1, NT, p.grid);
    if (!(a < e && a < t1 && e > w0)) return -1;
    return (2 * cc + (a >= t0 ? 0 : 1)) * kH + i;
  };
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float M;  // the maximum of the partials' maxima (and the step token's score), log2 units
  if (n <= kMergeGroups * kMergeBatch) {
    // one pass: every partial's features and (m, l) are loaded at once, before the maximum is known
    float4 v[kMergeBatch];
    bool has[kMergeBatch];
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const int u = grp + kMergeGroups * k;
      const int sl = u < n ? slot_of(u) : -1;  // never read a partial this sequence did not write
      has[k] = sl >= 0;
      v[k] = has[k] ? reinterpret_cast<const float4*>(p.ws_o + static_cast<size_t>(sl) * kD)[f4]
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int my = tid < n ? slot_of(tid) : -1;
    const float2 ml = my >= 0 ? *reinterpret_cast<const float2*>(p.ws_ml + 2 * static_cast<size_t>(my))
                              : make_float2(-INFINITY, 0.f);
    M = merge_reduce<kMergeThreads>(ml.x, true, s_red);
    if (nv) M = fmaxf(M, zn);
    const float w = ml.x == -INFINITY ? 0.f : exp2f(ml.x - M);
    if (tid < n) s_w[tid] = w;
    L = merge_reduce<kMergeThreads>(ml.y * w, false, s_red);  // ends with a barrier: s_w visible
#pragma unroll
    for (int k = 0; k < kMergeBatch; ++k) {
      const float wk = has[k] ? s_w[grp + kMergeGroups * k] : 0.f;
      acc.x = fmaf(v[k].x, wk, acc.x);
      acc.y = fmaf(v[k].y, wk, acc.y);
      acc.z = fmaf(v[k].z, wk, acc.z);
      acc.w = fmaf(v[k].w, wk, acc.w);
    }
  } else {
    M = -INFINITY;
    for (int u = tid; u < n; u += kMergeThreads) {
      const int sl = slot_of(u);
      if (sl >= 0) M = fmaxf(M, p.ws_ml[2 * static_cast<size_t>(sl)]);
    }
    M = merge_reduce<kMergeThreads>(M, true, s_red);
    if (nv) M = fmaxf(M, zn);
    for (int c0 = 0; c0 < n; c0 += kMergeMax) {
      const int cn = min(kMergeMax, n - c0);
      float lpart = 0.f;
      for (int u = tid; u < cn; u += kMergeThreads) {
        const int sl = slot_of(c0 + u);
        float w = 0.f;
        if (sl >= 0) {
          const float mj = p.ws_ml[2 * static_cast<size_t>(sl)];
          w = mj == -INFINITY ? 0.f : exp2f(mj - M);
          lpart = fmaf(p.ws_ml[2 * static_cast<size_t>(sl) + 1], w, lpart);
        }
        s_w[u] = w;
        s_slot[u] = sl;
      }
      L += merge_reduce<kMergeThreads>(lpart, false, s_red);  // ends with a barrier: s_w, s_slot visible
      for (int u0 = grp; u0 < cn; u0 += kMergeGroups * kMergeBatch) {
        float4 v[kMergeBatch];
        float wv[kMergeBatch];
#pragma unroll
        for (int k = 0; k < kMergeBatch; ++k) {
          const int u = u0 + kMergeGroups * k;
          const int sl = u < cn ? s_slot[u] : -1;  // never read a partial this sequence did not write
          wv[k] = sl >= 0 ? s_w[u] : 0.f;
          v[k] = sl >= 0 ? reinterpret_cast<const float4*>(p.ws_o + static_cast<size_t>(sl) * kD)[f4]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kMergeBatch; ++k) {
          acc.x = fmaf(v[k].x, wv[k], acc.x);
          acc.y = fmaf(v[k].y, wv[k], acc.y);
          acc.z = fmaf(v[k].z, wv[k], acc.z);
          acc.w = fmaf(v[k].w, wv[k], acc.w);
        }
      }
      __syncthreads();  // s_w, s_slot are rewritten by the next pass
    }
  }
  if (nv) {  // the step's token: one more partial (z_t, 1, V_t), added once (warp kVnWarp holds V_t)
    const float wn = exp2f(zn - M);
    L += wn;
    if (vn_warp) {
      acc.x = fmaf(vn.x, wn, acc.x);
      acc.y = fmaf(vn.y, wn, acc.y);
      acc.z = fmaf(vn.z, wn, acc.z);
      acc.w = fmaf(vn.w, wn, acc.w);
    }
  }
  s_acc[grp][f4] = acc;
  __syncthreads();
  if constexpr (kMergeGroups > 8) {  // fold the groups to 8 first, in parallel
    if (tid < 8 * 32) {
      float4 r = s_acc[grp][f4];
#pragma unroll
      for (int g2 = grp + 8; g2 < kMergeGroups; g2 += 8) {
        r.x += s_acc[g2][f4].x;
        r.y += s_acc[g2][f4].y;
        r.z += s_acc[g2][f4].z;
        r.w += s_acc[g2][f4].w;
      }
      s_acc[grp][f4] = r;
    }
    __syncthreads();
  }
  if (tid < 32) {
    float4 r = s_acc[0][tid];
#pragma unroll
    for (int g2 = 1; g2 < (kMergeGroups < 8 ? kMergeGroups : 8); ++g2) {
      r.x += s_acc[g2][tid].x;
      r.y += s_acc[g2][tid].y;
      r.z += s_acc[g2][tid].z;
      r.w += s_acc[g2][tid].w;
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    reinterpret_cast<float4*>(o)[tid] = make_float4(r.x * inv, r.y * inv, r.z * inv, r.w * inv);
  }
  write_lse(M, L);
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// The dynamic shared-memory opt-in, once per (device, rank variant).
cudaError_t set_smem_once(int r) {
  static std::once_flag once[64][2];
  static cudaError_t status[64][2];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int k = r == 1 ? 0 : 1;
  std::call_once(once[dev][k], [dev, k]() {
    auto kern = k == 0 ? decode_tc_kernel<1> : decode_tc_kernel<2>;
    cudaError_t e2 = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(kSmemBytes));
    if (e2 == cudaSuccess)
      e2 = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    status[dev][k] = e2;
  });
  return status[dev][k];
}

// CTAs of the decode kernel resident per SM (queried once per device).
int ctas_per_sm() {
  static std::once_flag once[64];
  static int occ[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::call_once(once[dev], [dev]() {
    int n = 1;
    if (set_smem_once(1) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_tc_kernel<1>, kThreads, kSmemBytes) != cudaSuccess)
      n = 1;
    occ[dev] = n < 1 ? 1 : n;
  });
  return occ[dev];
}

struct TcWorkspace {
  int32_t* prefix;
  float* ml;
  float* o;
  int32_t* len;     // decode step: lengths the split kernel saw
  float* step_ml;   // decode step: (m, l) of sequences finished inside one CTA
  size_t bytes;
};

// [prefix: B + 2 int32 (the tile prefix, then the set-up units charged)][ml: 2G x 32 x 2 f32][o: 2G x 32 x 128 f32][len: B int32][step ml: B x 32 x 2 f32],
// each section 256-byte aligned.
TcWorkspace carve(void* base, int batch, int grid) {
  TcWorkspace w;
  const size_t slots = 2 * static_cast<size_t>(grid);
  const size_t pb = round256((static_cast<size_t>(batch) + 2) * 4);
  const size_t mlb = round256(slots * kH * 2 * 4);
  const size_t ob = round256(slots * kH * kD * 4);
  const size_t lb = round256(static_cast<size_t>(batch) * 4);
  const size_t sb = round256(static_cast<size_t>(batch) * kH * 2 * 4);
  char* c = static_cast<char*>(base);
  w.prefix = reinterpret_cast<int32_t*>(c);
  w.ml = reinterpret_cast<float*>(c ? c + pb : nullptr);
  w.o = reinterpret_cast<float*>(c ? c + pb + mlb : nullptr);
  w.len = reinterpret_cast<int32_t*>(c ? c + pb + mlb + ob : nullptr);
  w.step_ml = reinterpret_cast<float*>(c ? c + pb + mlb + ob + lb : nullptr);
  w.bytes = pb + mlb + ob + lb + sb;
  return w;
}

}  // namespace

bool tensor_decode_supported(int dtype, int heads, int head_dim, int r_k, int r_v) {
  return dtype == TPA_BF16 && heads == kH && head_dim == kD && r_k == r_v && (r_k == 1 || r_k == 2);
}

bool tensor_decode_batch_ok(int batch) { return batch >= 1 && batch <= kMaxBatch; }

// One wave: every resident CTA slot of the GPU (the tcgen05 kernel holds one SM per CTA).
int tensor_decode_default_ctas(int sms, int variant) {
  return (variant == kDecodeUmma ? 1 : ctas_per_sm()) * (sms > 0 ? sms : 148);
}

size_t tensor_decode_workspace_bytes(int batch, int grid) { return carve(nullptr, batch, grid).bytes; }

cudaError_t launch_tensor_decode(const TensorDecodeArgs& a, cudaStream_t stream) {
  const CacheView& cv = a.cache;
  cudaError_t e;
  TcWorkspace ws = carve(a.workspace, cv.batch, a.grid);
  DecodeTcParams p;
  p.seq_lens = cv.seq_lens;
  p.q = a.q;
  p.a_q = a.a_q;
  p.r_q = a.r_q;
  p.inv_rq = a.r_q > 0 ? 1.f / static_cast<float>(a.r_q) : 1.f;
  p.q_pos = a.q_pos;
  p.batch = cv.batch;
  p.capacity = cv.capacity;
  p.max_len = a.max_len;
  p.grid = a.grid;
  p.inv_grid = 1.0 / static_cast<double>(a.grid);
  p.zs = a.scale * kLog2e / static_cast<float>(cv.r_k);
  p.inv_rv = 1.f / static_cast<float>(cv.r_v);
  p.out = a.out;
  p.ws_prefix = ws.prefix;
  p.ws_ml = ws.ml;
  p.ws_o = ws.o;
  p.ws_len = a.step ? ws.len : nullptr;
  p.whole_ml = (a.step || a.lse) ? ws.step_ml : nullptr;
  p.err = a.err;
  p.rope = a.rope;
  // a sequence's query stage costs a tcgen05 CTA about one tile of streaming; the warp-level
  // kernel's partition counts tiles only
  p.setup = a.variant == kDecodeUmma ? 1 : 0;
  if (a.variant == kDecodeUmma) {
    e = launch_decode_umma(p, cv, stream);
  } else {
    const uint64_t rows_k = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_k;
    const uint64_t rows_v = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_v;
    CUtensorMap tbk, tbv, tak, tav;
    if ((e = encode_bf16_2d(&tbk, cv.b_k, kD, rows_k, 64, kRows, 128)) != cudaSuccess) return e;
    if ((e = encode_bf16_2d(&tbv, cv.b_v, kD, rows_v, 64, kRows, 128)) != cudaSuccess) return e;
    if ((e = encode_bf16_2d(&tak, cv.a_k, kH, rows_k, kH, kRows, 64)) != cudaSuccess) return e;
    if ((e = encode_bf16_2d(&tav, cv.a_v, kH, rows_v, kH, kRows, 64)) != cudaSuccess) return e;
    auto kern = cv.r_k == 1 ? decode_tc_kernel<1> : decode_tc_kernel<2>;
    if ((e = set_smem_once(cv.r_k)) != cudaSuccess) return e;
    kern<<<a.grid, kThreads, kSmemBytes, stream>>>(p, tbk, tbv, tak, tav);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  TcMergeParams mp;
  mp.batch = cv.batch;
  mp.grid = a.grid;
  mp.setup = p.setup;
  mp.prefix = ws.prefix;
  mp.ws_ml = ws.ml;
  mp.ws_o = ws.o;
  mp.out = a.out;
  mp.lse = a.lse;
  mp.whole_ml = ws.step_ml;
  if (a.step) {
    TcStepParams& st = mp.st;
    st.pos = a.q_pos;
    st.a_k = static_cast<const __nv_bfloat16*>(a.step->a_k);
    st.b_k = static_cast<const __nv_bfloat16*>(a.step->b_k);
    st.a_v = static_cast<const __nv_bfloat16*>(a.step->a_v);
    st.b_v = static_cast<const __nv_bfloat16*>(a.step->b_v);
    st.q = static_cast<const __nv_bfloat16*>(a.q);
    st.a_q = static_cast<const __nv_bfloat16*>(a.a_q);
    st.r_q = a.r_q;
    st.inv_rq = p.inv_rq;
    st.r = cv.r_k;
    st.zs = p.zs;
    st.inv_rv = p.inv_rv;
    st.capacity = cv.capacity;
    st.advance = a.step->advance;
    st.ws_len = ws.len;
    st.c_ak = static_cast<__nv_bfloat16*>(const_cast<void*>(cv.a_k));
    st.c_bk = static_cast<__nv_bfloat16*>(const_cast<void*>(cv.b_k));
    st.c_av = static_cast<__nv_bfloat16*>(const_cast<void*>(cv.a_v));
    st.c_bv = static_cast<__nv_bfloat16*>(const_cast<void*>(cv.b_v));
    st.seq_lens = const_cast<int32_t*>(cv.seq_lens);
    st.err = a.err;
    st.rope = a.rope;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cv.batch, kH);
  const bool small_batch = cv.batch <= 2;
  cfg.blockDim = dim3(small_batch ? kMergeThreadsSmallBatch : 256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (small_batch) {
    if (a.step) return cudaLaunchKernelEx(&cfg, decode_tc_merge_kernel<true, kMergeThreadsSmallBatch>, mp);
    return cudaLaunchKernelEx(&cfg, decode_tc_merge_kernel<false, kMergeThreadsSmallBatch>, mp);
  }
  if (a.step) return cudaLaunchKernelEx(&cfg, decode_tc_merge_kernel<true, 256>, mp);
  return cudaLaunchKernelEx(&cfg, decode_tc_merge_kernel<false, 256>, mp);
}

}  // namespace tpa
