// Causal prefill on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA), bf16, h = 32, d_h = 128, R_K = R_V = R in {1, 2}, R_Q <= 8.
//
// What it computes (Tensor Product Attention Is All You Need, sections
// 解决思路 for Q_t = (1/R_Q) A_Q^T B_Q, 关键设计 for the K/V factors,
// RoPE 兼容性 for RoPE on the B factors, FlashTPA for attention on factors):
// for query t of a chunk (cache slot P + t) and head i,
//   q_{t,i}     = (1/R_Q) sum_j A_Q[t, j, i] RoPE(B_Q[t, j], pos_t)
//   S[t, (s,r)] = q_{t,i} . B~_K[s, r]                       (tensor cores)
//   z[t, s]     = scale/R_K sum_r A_K[s, r, i] S[t, (s, r)],  s <= P + t
//   W[t, (s,r)] = softmax_s(z)[t, s] A_V[s, r, i] / R_V
//   O[t, i, :]  = sum_(s,r) W[t, (s,r)] B_V[s, r, :]         (tensor cores)
// The dense per-head query is the only thing expanded: it is built once per
// chunk in fp32 by prefill_q_kernel, then each softmax thread splits its own
// query row into bf16 high and low parts in TMEM.  Keys and values stay
// factorized: the score MMA contracts the query with B_K rows, and the value
// MMA contracts the softmax weights with B_V rows.  Putting the head factors
// on the query side of the MMA (a dense Q tile per head) costs 2 h d_h R_K
// tensor flops per (query, key) pair and almost no CUDA-core work; contracting
// B_Q with B_K first would save tensor flops but needs ~h R_Q R_K CUDA-core
// FMAs per pair to apply A_Q and A_K, which is slower on this machine.
//
// CTA = (sequence, head, tile of 128 queries); heavy (late) query tiles are
// dispatched first.  Roles: warp 0 issues TMA loads (a 2-stage ring of
// {B_K, B_V, A_K, A_V} tiles of 128 cache rows); warp 1 allocates 512 TMEM
// columns and one of its threads issues the MMAs; warps 2-5 (one TMEM lane =
// one query row per thread) stage the query and run the softmax.
// Per key tile j: S = (Q_hi + Q_lo) B_K^T (M = 128 queries, N = 128 rows,
// K = 128; A from TMEM columns [384, 512)) into TMEM columns
// [128 (j % 2), +128), so the score MMA of tile j + 1 runs while the softmax
// works on tile j; the softmax reads S, applies A_K, the causal mask
// and the online softmax, rescales O in TMEM when the running maximum grows
// by more than 2^8, and writes W as bf16 hi and lo halves into the first and
// second 64 columns of the same buffer (over S); then O += W_hi B_V + W_lo B_V
// (A from TMEM, B_V as an MN-major operand) into columns [256, 384).  Both the
// query and W are split into two bf16 parts, which keeps them to ~16 bits: one
// bf16 rounding of either costs ~3.5e-3 relative error on the prefill
// workload, above its 2e-3 budget.
#include <cuda.h>
#include <math.h>

#include <mutex>

#include "device_common.cuh"
#include "ptx_sm100.cuh"
#include "tma_host.h"
#include "tpa_internal.h"
#include "tpa_tensor.h"

namespace tpa {
namespace {

constexpr int kH = 32;
constexpr int kD = 128;
constexpr int kQ = 128;                 // queries per CTA
constexpr int kKRows = 128;             // cache rows per key tile
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kBox = kKRows * 128;      // 16 KB: one 64-feature box of a B tile
constexpr int kBTile = 2 * kBox;
constexpr int kATile = kKRows * kH * 2; // 8 KB
constexpr int kStageBytes = 2 * kBTile + 2 * kATile;
constexpr int kOffStages = 0;
constexpr int kOffAf = kOffStages + kStages * kStageBytes;  // fp32 A_K, A_V of the head: [2 stages][2][128]
constexpr int kOffBar = kOffAf + kStages * 2 * kKRows * 4;
constexpr int kNumBars = 2 * kStages + 7;  // full[2], empty[2], q_ready, s_full[2], w_ready, o_done, final, staged
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr size_t kSmemBytes = 1024 + kOffMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemCols = 512;
constexpr unsigned kErrTimeout = 0x8u;

// instruction descriptors, kind::f16: D fp32, A and B bf16, M = 128, N = 128
constexpr uint32_t kIdescSS = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescTS = kIdescSS | (1u << 16);  // B (= B_V tile) MN-major

struct PrefillTcParams {
  const int32_t* seq_lens;
  int batch, capacity, n_tokens, n_qtiles;
  float zs;       // scale * log2(e) / R_K
  float inv_rv;   // 1 / R_V
  const float* q;  // [B][T][32][128] fp32 rotated queries
  float* out;      // [B][T][32][128]
  unsigned int* err;
};

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillTcParams p,
                      const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                      const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_av) {
  constexpr int TOK = kKRows / R;  // tokens per key tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  float* s_af = reinterpret_cast<float*>(gbase + kOffAf);
  const uint32_t bar0 = sbase + kOffBar;
  auto bar_full = [&](int s) { return bar0 + 8 * s; };
  auto bar_empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  const uint32_t bar_q = bar0 + 8 * (2 * kStages);
  auto bar_s = [&](int buf) { return bar_q + 8 + 8 * buf; };  // S buffer `buf` holds a tile's scores
  const uint32_t bar_w = bar_q + 24, bar_o = bar_q + 32, bar_fin = bar_q + 40;
  const uint32_t bar_a = bar_q + 48;  // the four softmax warps have staged this tile's A_K, A_V
  volatile uint32_t* s_taddr = reinterpret_cast<volatile uint32_t*>(gbase + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // heavy query tiles first: blockIdx.y runs over query tiles from the last one down
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.y);
  const int i = blockIdx.x % kH;
  const int b = blockIdx.x / kH;
  const int q0 = qt * kQ;
  const int len = p.seq_lens[b];
  const int P = len - p.n_tokens;
  if (len > p.capacity || P < 0) {
    if (tid == 0 && i == 0 && qt == 0) atomicOr(p.err, TPA_DEVERR_PREFILL_LEN);
    return;
  }
  const int q_hi = min(q0 + kQ, p.n_tokens);          // queries [q0, q_hi) are real
  const int key_end = P + q_hi;                       // keys [0, key_end) are needed
  const int nk = (key_end + TOK - 1) / TOK;

  if (tid == 0) {
    // W, the query and the staged head factors: one arrival per softmax warp
    for (int s = 0; s < kNumBars; ++s) {
      const uint32_t bar = bar0 + 8 * s;
      ptx::mbar_init(bar, (bar == bar_w || bar == bar_q || bar == bar_a) ? 4 : 1);
    }
    *s_abort = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(sbase + kOffMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *s_taddr;
  // S of tile j in columns [128 (j % 2), +128): scores, then W hi (first 64) and W lo (next 64)
  auto t_s = [&](int j) { return tbase + 128u * static_cast<uint32_t>(j & 1); };
  const uint32_t t_o = tbase + 256;    // O
  const uint32_t t_q = tbase + 384;    // query hi (cols 384..447) and lo (448..511)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_bk);
      ptx::prefetch_tmap(&tm_bv);
      int issued = 0;
      for (int j = 0; j < nk; ++j) {
        const int st = j % kStages;
        if (*s_abort) break;
        if (!ptx::mbar_wait_bounded(bar_empty(st), ((j / kStages) & 1) ^ 1)) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
          break;
        }
        const int row0 = (b * p.capacity + j * TOK) * R;
        const uint32_t sb = sbase + kOffStages + st * kStageBytes;
        const uint32_t fb = bar_full(st);
        ptx::mbar_arrive_expect_tx(fb, kStageBytes);
        ptx::tma_load_2d(sb, &tm_bk, 0, row0, fb);
        ptx::tma_load_2d(sb + kBox, &tm_bk, 64, row0, fb);
        ptx::tma_load_2d(sb + kBTile, &tm_bv, 0, row0, fb);
        ptx::tma_load_2d(sb + kBTile + kBox, &tm_bv, 64, row0, fb);
        ptx::tma_load_2d(sb + 2 * kBTile, &tm_ak, 0, row0, fb);
        ptx::tma_load_2d(sb + 2 * kBTile + kATile, &tm_av, 0, row0, fb);
        ++issued;
      }
      // every issued load has landed before this CTA can finish
      for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j)
        ptx::mbar_wait_bounded(bar_full(j % kStages), (j / kStages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S(0); then for each tile j: S(j+1) into the other buffer (after the value MMA
    // of tile j-1 has consumed the W stored there), then O += W(j) B_V once the softmax of
    // tile j is done.  The score MMA of tile j+1 thus runs while the softmax works on tile j.
    if (lane == 0) {
      auto scores = [&](int j) {
        const uint32_t sb = sbase + kOffStages + (j % kStages) * kStageBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // query hi, then query lo
#pragma unroll
          for (int k = 0; k < 8; ++k) {         // K = 128 features in steps of 16
            const uint64_t db = ptx::umma_desc_sw128(sb + (k >> 2) * kBox + (k & 3) * 32, 16, 1024);
            ptx::umma_ts(t_s(j), t_q + half * 64 + k * 8, db, kIdescSS, (half > 0 || k > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(bar_s(j & 1));
      };
      bool ok = ptx::mbar_wait_bounded(bar_q, 0) && ptx::mbar_wait_bounded(bar_full(0), 0);
      if (ok) {
        ptx::tc_fence_after();
        scores(0);
      }
      for (int j = 0; j < nk && ok; ++j) {
        if (*s_abort) break;
        if (j + 1 < nk) {
          ok = ptx::mbar_wait_bounded(bar_full((j + 1) % kStages), ((j + 1) / kStages) & 1);
          if (ok && j > 0) ok = ptx::mbar_wait_bounded(bar_o, (j - 1) & 1);
          if (!ok) break;
          ptx::tc_fence_after();
          scores(j + 1);
        }
        ok = ptx::mbar_wait_bounded(bar_w, j & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t bv = sbase + kOffStages + (j % kStages) * kStageBytes + kBTile;
#pragma unroll
        for (int half = 0; half < 2; ++half) {    // W hi, then W lo
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {        // K = 128 cache rows in steps of 16
            const uint64_t db = ptx::umma_desc_sw128(bv + kk * 2048, kBox, 1024);
            ptx::umma_ts(t_o, t_s(j) + half * 64 + kk * 8, db, kIdescTS, (j > 0 || half > 0 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(bar_o);
        ptx::umma_commit(bar_empty(j % kStages));
      }
      if (!ok) {
        atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      // all MMAs issued by this thread complete before TMEM can be released
      ptx::umma_commit(bar_fin);
      ptx::mbar_wait_bounded(bar_fin, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;          // query row within the tile = key-tile row this thread stages
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tq = q0 + row;                   // query index in the chunk
    const int qslot = P + tq;                  // its cache slot: keys s <= qslot
    // stage this thread's query row as bf16 hi + lo into TMEM (zeros past the chunk)
    {
      const float* qr = p.q + ((static_cast<size_t>(b) * p.n_tokens + tq) * kH + i) * kD;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t hi[32], lo[32];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (tq < p.n_tokens) v = *reinterpret_cast<const float4*>(qr + c2 * 64 + 2 * e);
          hi[e] = ptx::pack_bf16(v.x, v.y);
          hi[e + 1] = ptx::pack_bf16(v.z, v.w);
          lo[e] = ptx::pack_bf16(v.x - ptx::bf16_lo(hi[e]), v.y - ptx::bf16_hi(hi[e]));
          lo[e + 1] = ptx::pack_bf16(v.z - ptx::bf16_lo(hi[e + 1]), v.w - ptx::bf16_hi(hi[e + 1]));
        }
        ptx::tmem_st32(t_q + lane_off + c2 * 32, hi);
        ptx::tmem_st32(t_q + lane_off + 64 + c2 * 32, lo);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_q);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int st = j % kStages;
      bool fail = *s_abort != 0;
      if (!fail) fail = !ptx::mbar_wait_bounded(bar_full(st), (j / kStages) & 1) || !ptx::mbar_wait_bounded(bar_s(j & 1), (j >> 1) & 1);
      ptx::tc_fence_after();
      const uint8_t* sb = gbase + kOffStages + st * kStageBytes;
      const int tok0 = j * TOK;
      const int valid_rows = min(kKRows, (len - tok0) * R);  // rows of real keys in this tile
      // this thread stages row `row` of the key tile: A_K[., i], A_V[., i] as fp32 (64-byte swizzled rows)
      if (!fail) {
        const int chunk = (i >> 3) ^ ((row >> 1) & 3);
        const int off = row * 64 + chunk * 16 + (i & 7) * 2;
        const float ak = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sb + 2 * kBTile + off));
        const float av = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(sb + 2 * kBTile + kATile + off));
        s_af[(st * 2 + 0) * kKRows + row] = ak;
        s_af[(st * 2 + 1) * kKRows + row] = av;
      }
      if (!fail && valid_rows < kKRows && row >= valid_rows) {
        // zero the B_V row past the sequence end (may hold NaN; 0 * NaN would reach every O row)
        uint4* vrow0 = reinterpret_cast<uint4*>(const_cast<uint8_t*>(sb) + kBTile + row * 128);
        uint4* vrow1 = reinterpret_cast<uint4*>(const_cast<uint8_t*>(sb) + kBTile + kBox + row * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          vrow0[c] = make_uint4(0, 0, 0, 0);
          vrow1[c] = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
      }
      // rendezvous of the four softmax warps (a bounded wait): the staged A_K, A_V of this tile
      // are visible afterwards; a warp that timed out raises the abort flag before arriving
      if (fail) {
        atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_a);
      if (!ptx::mbar_wait_bounded(bar_a, j & 1)) {
        atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      if (__any_sync(0xffffffffu, *s_abort != 0)) {
        ok = false;
        break;
      }
      const float* akf = s_af + (st * 2 + 0) * kKRows;
      const float* avf = s_af + (st * 2 + 1) * kKRows;
      // ---- scores: z[s] for the TOK tokens of the tile (log2 units)
      float z[TOK];
      const bool need_mask = (tok0 + TOK - 1 > P + q0) || (tok0 + TOK > len);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t sv[32];
        ptx::tmem_ld32(t_s(j) + lane_off + c4 * 32, sv);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32 / R; ++e) {
          const int rr = c4 * 32 + e * R;
          float acc = 0.f;
#pragma unroll
          for (int r = 0; r < R; ++r) acc = fmaf(akf[rr + r], __uint_as_float(sv[e * R + r]), acc);
          const int s = c4 * (32 / R) + e;
          z[s] = acc * p.zs;
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int s = 0; s < TOK; ++s) {
        if (need_mask) {
          const int slot = tok0 + s;
          if (slot > qslot || slot >= len) z[s] = -INFINITY;
        }
        mx = fmaxf(mx, z[s]);
      }
      // ---- online softmax with a lazily rescaled maximum; the TMEM rescale of O is a
      // warp-wide operation, so the whole warp runs it when any of its rows needs it
      const bool grow = mx > m + 8.f || (m == -INFINITY && mx != -INFINITY);
      const float alpha = !grow ? 1.f : (m == -INFINITY ? 0.f : exp2f(m - mx));
      if (grow) {
        l *= alpha;
        m = mx;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // the value MMA of tile j-1 may still be accumulating into O
        const bool o_prev = ptx::mbar_wait_bounded(bar_o, (j - 1) & 1);
        if (!__all_sync(0xffffffffu, o_prev)) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
          ok = false;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t ov[32];
          ptx::tmem_ld32(t_o + lane_off + c4 * 32, ov);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          ptx::tmem_st32(t_o + lane_off + c4 * 32, ov);
        }
      }
      // ---- W = p A_V / R_V as bf16 hi + lo, packed two rows per TMEM column
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {        // 64 cache rows per chunk -> 32 columns
        uint32_t whi[32], wlo[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int rr0 = c2 * 64 + 2 * e;    // cache rows rr0, rr0 + 1
          float w2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int rr = rr0 + u;
            const int s = rr / R;
            const float pz = (z[s] == -INFINITY) ? 0.f : exp2f(z[s] - m);
            w2[u] = (z[s] == -INFINITY) ? 0.f : pz * avf[rr] * p.inv_rv;
            if (rr % R == 0) l += pz;
          }
          whi[e] = ptx::pack_bf16(w2[0], w2[1]);
          wlo[e] = ptx::pack_bf16(w2[0] - ptx::bf16_lo(whi[e]), w2[1] - ptx::bf16_hi(whi[e]));
        }
        ptx::tmem_st32(t_s(j) + lane_off + c2 * 32, whi);
        ptx::tmem_st32(t_s(j) + lane_off + 64 + c2 * 32, wlo);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_w);
    }
    // ---- epilogue: O / l to out[b][t][i][:].  It waits on the issuer's final commit, not on
    // the parity of the value barrier: with two score buffers that barrier can still be two
    // phases behind here, where its parity alone cannot tell the last phase from an earlier one.
    const bool o_ready = ok && ptx::mbar_wait_bounded(bar_fin, 0);
    if (__all_sync(0xffffffffu, o_ready)) {  // the TMEM loads below are warp-wide
      ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* op = p.out + ((static_cast<size_t>(b) * p.n_tokens + tq) * kH + i) * kD;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t ov[32];
        ptx::tmem_ld32(t_o + lane_off + c4 * 32, ov);
        ptx::tmem_wait_ld();
        if (tq < p.n_tokens) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            *reinterpret_cast<float4*>(op + c4 * 32 + e) =
                make_float4(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv,
                            __uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
          }
        }
      }
    } else if (ok) {
      atomicOr(p.err, kErrTimeout);
      *s_abort = 1;
    }
    ptx::tc_fence_before();
  }
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
    auto kern = k == 0 ? prefill_tc_kernel<1> : prefill_tc_kernel<2>;
    status[dev][k] =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
  });
  return status[dev][k];
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

}  // namespace

bool tensor_prefill_supported(int dtype, int heads, int head_dim, int r_k, int r_v, int r_q) {
  return dtype == TPA_BF16 && heads == kH && head_dim == kD && r_k == r_v && (r_k == 1 || r_k == 2) && r_q >= 1 &&
         r_q <= 8;
}

size_t tensor_prefill_workspace_bytes(int batch, int n_tokens, int heads, int head_dim) {
  return round256(static_cast<size_t>(batch) * heads * n_tokens * head_dim * 4);  // fp32 rotated queries
}

cudaError_t launch_tensor_prefill(const TensorPrefillArgs& a, cudaStream_t stream) {
  const CacheView& cv = a.cache;
  const int T = a.n_tokens;
  float* qws = static_cast<float*>(a.workspace);
  PrefillQArgs qa;
  qa.batch = cv.batch;
  qa.n_tokens = T;
  qa.heads = cv.heads;
  qa.head_dim = cv.head_dim;
  qa.r_q = a.r_q;
  qa.dtype = cv.dtype;
  qa.a_q = a.a_q;
  qa.b_q = a.b_q;
  qa.q_pos = a.q_pos;
  qa.q_out = qws;
  qa.rope = a.rope;
  cudaError_t e = launch_prefill_q(qa, stream);
  if (e != cudaSuccess) return e;
  const uint64_t rows_k = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_k;
  const uint64_t rows_v = static_cast<uint64_t>(cv.batch) * cv.capacity * cv.r_v;
  CUtensorMap tbk, tbv, tak, tav;
  if ((e = encode_bf16_2d(&tbk, cv.b_k, kD, rows_k, 64, kKRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tbv, cv.b_v, kD, rows_v, 64, kKRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tak, cv.a_k, kH, rows_k, kH, kKRows, 64)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tav, cv.a_v, kH, rows_v, kH, kKRows, 64)) != cudaSuccess) return e;
  if ((e = set_smem_once(cv.r_k)) != cudaSuccess) return e;
  PrefillTcParams p;
  p.seq_lens = cv.seq_lens;
  p.batch = cv.batch;
  p.capacity = cv.capacity;
  p.n_tokens = T;
  p.n_qtiles = (T + kQ - 1) / kQ;
  p.zs = a.scale * kLog2e / static_cast<float>(cv.r_k);
  p.inv_rv = 1.f / static_cast<float>(cv.r_v);
  p.q = qws;
  p.out = a.out;
  p.err = a.err;
  dim3 grid(cv.batch * kH, p.n_qtiles);
  auto kern = cv.r_k == 1 ? prefill_tc_kernel<1> : prefill_tc_kernel<2>;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(p, tbk, tbv, tak, tav);
  return cudaGetLastError();
}

}  // namespace tpa
