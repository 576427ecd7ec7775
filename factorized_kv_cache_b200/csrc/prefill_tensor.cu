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
// chunk in fp32 by prefill_q_kernel and split by the softmax threads into
// bf16 high and low parts in shared memory.  Keys and values stay
// factorized: the score MMA contracts the query with B_K rows, and the value
// MMA contracts the softmax weights with B_V rows.  Putting the head factors
// on the query side of the MMA (a dense Q tile per head) costs 2 h d_h R_K
// tensor flops per (query, key) pair and little CUDA-core work; contracting
// B_Q with B_K first would save tensor flops but needs ~h R_Q R_K CUDA-core
// FMAs per pair to apply A_Q and A_K, which is slower on this machine.
//
// CTA = (sequence, pair of heads, tile of 128 queries); heavy (late) query
// tiles are dispatched first.  The two heads share every key/value tile and
// take turns on the tensor cores while the other one runs its softmax.
// Roles (352 threads): warp 0 issues TMA loads of 64-row key tiles {B_K, the
// 8-head slice of A_K holding both heads} into a 3-slot ring and value tiles
// {B_V, A_V slice} into a 2-slot ring; warp 1 allocates all 512 TMEM columns
// and one of its threads issues the MMAs; warps 2-5 (head 0) and 6-9
// (head 1) own one query row each (one TMEM lane); warp 10 stages both
// heads' A_K, A_V of a tile as fp32 (scale folded in) and zeroes B_V rows
// past the sequence end, which may hold NaN.
// TMEM per head h: S double-buffered in columns [256 h + 64 b, +64), then
// overwritten in place by W as bf16 hi (first 32 columns) and lo (next 32);
// O in [256 h + 128, +128).  Per key tile j and head:
//   S = (Q_hi + Q_lo) B_K^T  (M = 128 queries, N = 64 rows, K = 128; both
//       operands in shared memory, K-major, 128-byte swizzle);
//   softmax: A_K weighting, causal mask, online softmax with a lazily
//       rescaled maximum (only when it grows by more than 2^8), W = p A_V;
//   O += W_hi B_V + W_lo B_V  (A from TMEM, B_V MN-major).
// Both the query and W are split into two bf16 parts, which keeps them to
// ~16 bits: one bf16 rounding of either costs ~3.5e-3 relative error on the
// prefill workload, above its 2e-3 budget.  Every wait is bounded (2 s);
// a timeout sets the error word and an abort flag, and TMEM is released
// only after the MMA thread's last commit.
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
constexpr int kRows = 64;               // cache rows per key tile
constexpr int kKSlots = 3;
constexpr int kVSlots = 2;
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (3 + kSoftmaxWarps) * 32;
constexpr int kStagerWarp = 2 + kSoftmaxWarps;
constexpr int kBBox = kRows * 128;        // 64 features x 64 rows, bf16: 8 KB
constexpr int kBBytes = 2 * kBBox;        // one B tile
constexpr int kASlice = 8;                // heads in the A slice a tile carries (16 bytes per row)
constexpr int kABytes = kRows * kASlice * 2;
constexpr int kSlotBytes = kBBytes + kABytes;  // 17 KB
constexpr int kQBox = kQ * 128;           // 128 queries x 64 features, bf16: 16 KB
constexpr int kQHead = 4 * kQBox;         // hi (2 boxes) then lo (2 boxes)
constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKSlots * kSlotBytes;
constexpr int kOffQ = kOffV + kVSlots * kSlotBytes;
constexpr int kOffA = kOffQ + 2 * kQHead;  // fp32 [2 buffers][4: A_K h0, A_K h1, A_V h0, A_V h1][64]
constexpr int kOffBar = kOffA + 2 * 4 * kRows * 4;
// kfull[3], kempty[3], vfull[2], vempty[2], sfull[2 heads][2], wready[2][2], odone[2], staged[2], qready, fin
constexpr int kNumBars = 2 * kKSlots + 2 * kVSlots + 4 + 4 + 2 + 2 + 1 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr size_t kSmemBytes = 1024 + kOffMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kSlotBytes % 1024 == 0 && kQBox % 1024 == 0 && kOffQ % 1024 == 0, "swizzle atoms stay aligned");
constexpr uint32_t kTmemCols = 512;
constexpr unsigned kErrTimeout = 0x8u;

// kind::f16 instruction descriptors, D fp32, A and B bf16, M = 128:
// score MMA N = 64 (both K-major); value MMA N = 128 with B (the B_V tile) MN-major.
constexpr uint32_t kIdescScore = (1u << 4) | (1u << 7) | (1u << 10) | ((64u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescValue =
    (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

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
  constexpr int TOK = kRows / R;  // tokens per key tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  float* s_a = reinterpret_cast<float*>(gbase + kOffA);
  const uint32_t bar0 = sbase + kOffBar;
  auto kfull = [&](int s) { return bar0 + 8 * s; };
  auto kempty = [&](int s) { return bar0 + 8 * (kKSlots + s); };
  auto vfull = [&](int s) { return bar0 + 8 * (2 * kKSlots + s); };
  auto vempty = [&](int s) { return bar0 + 8 * (2 * kKSlots + kVSlots + s); };
  constexpr int kB1 = 2 * kKSlots + 2 * kVSlots;
  auto sfull = [&](int h, int b) { return bar0 + 8 * (kB1 + 2 * h + b); };
  auto wready = [&](int h, int b) { return bar0 + 8 * (kB1 + 4 + 2 * h + b); };
  auto odone = [&](int h) { return bar0 + 8 * (kB1 + 8 + h); };
  auto staged = [&](int b) { return bar0 + 8 * (kB1 + 10 + b); };
  const uint32_t qready = bar0 + 8 * (kB1 + 12);
  const uint32_t fin = bar0 + 8 * (kB1 + 13);
  volatile uint32_t* s_taddr = reinterpret_cast<volatile uint32_t*>(gbase + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // heavy query tiles first: blockIdx.y runs over query tiles from the last one down
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.y);
  const int hp = blockIdx.x % (kH / 2);  // heads 2 hp, 2 hp + 1
  const int b = blockIdx.x / (kH / 2);
  const int q0 = qt * kQ;
  const int len = p.seq_lens[b];
  const int P = len - p.n_tokens;
  if (len > p.capacity || P < 0) {
    if (tid == 0 && hp == 0 && qt == 0) atomicOr(p.err, TPA_DEVERR_PREFILL_LEN);
    return;
  }
  const int q_hi = min(q0 + kQ, p.n_tokens);  // queries [q0, q_hi) are real
  const int key_end = P + q_hi;                // keys [0, key_end) are needed
  const int nk = (key_end + TOK - 1) / TOK;
  const int a_x = kASlice * ((2 * hp) / kASlice);  // first head of the A slice
  const int a_off = 2 * hp - a_x;                   // heads 2 hp, 2 hp + 1 within the slice

  if (tid == 0) {
    for (int s = 0; s < kKSlots; ++s) {
      ptx::mbar_init(kfull(s), 1);
      ptx::mbar_init(kempty(s), 2);  // score-MMA commit + the stager (A_K read)
    }
    for (int s = 0; s < kVSlots; ++s) {
      ptx::mbar_init(vfull(s), 1);
      ptx::mbar_init(vempty(s), 2);  // value-MMA commit + the stager (A_V read, B_V rows zeroed)
    }
    for (int h = 0; h < 2; ++h) {
      for (int bf = 0; bf < 2; ++bf) {
        ptx::mbar_init(sfull(h, bf), 1);
        ptx::mbar_init(wready(h, bf), 4);
      }
      ptx::mbar_init(odone(h), 1);
      ptx::mbar_init(staged(h), 1);
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
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tbase = *s_taddr;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_bk);
      ptx::prefetch_tmap(&tm_bv);
      ptx::prefetch_tmap(&tm_ak);
      ptx::prefetch_tmap(&tm_av);
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < nk && ok; ++j) {
        if (*s_abort) {
          ok = false;
          break;
        }
        const int row0 = (b * p.capacity + j * TOK) * R;
        const int ks = j % kKSlots, vs = j % kVSlots;
        if (j >= kKSlots && !(ok = ptx::mbar_wait_bounded(kempty(ks), ((j / kKSlots) & 1) ^ 1))) break;
        const uint32_t kb = sbase + kOffK + ks * kSlotBytes;
        ptx::mbar_arrive_expect_tx(kfull(ks), kSlotBytes);
        ptx::tma_load_2d(kb, &tm_bk, 0, row0, kfull(ks));
        ptx::tma_load_2d(kb + kBBox, &tm_bk, 64, row0, kfull(ks));
        ptx::tma_load_2d(kb + kBBytes, &tm_ak, a_x, row0, kfull(ks));
        ++k_issued;
        if (j >= kVSlots && !(ok = ptx::mbar_wait_bounded(vempty(vs), ((j / kVSlots) & 1) ^ 1))) break;
        const uint32_t vb = sbase + kOffV + vs * kSlotBytes;
        ptx::mbar_arrive_expect_tx(vfull(vs), kSlotBytes);
        ptx::tma_load_2d(vb, &tm_bv, 0, row0, vfull(vs));
        ptx::tma_load_2d(vb + kBBox, &tm_bv, 64, row0, vfull(vs));
        ptx::tma_load_2d(vb + kBBytes, &tm_av, a_x, row0, vfull(vs));
        ++v_issued;
      }
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
        // every load already issued lands before the CTA can exit
        for (int k = max(0, k_issued - kKSlots); k < k_issued; ++k)
          ptx::mbar_wait_bounded(kfull(k % kKSlots), (k / kKSlots) & 1);
        for (int k = max(0, v_issued - kVSlots); k < v_issued; ++k)
          ptx::mbar_wait_bounded(vfull(k % kVSlots), (k / kVSlots) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Iteration j: the score MMAs of tile j for both heads, then the value MMAs of
    // tile j - 1 (whose W the softmax warps are finishing meanwhile).
    if (lane == 0) {
      auto score = [&](int h, int j) {
        const uint32_t kb = sbase + kOffK + (j % kKSlots) * kSlotBytes;
        const uint32_t qb = sbase + kOffQ + h * kQHead;
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // query hi, then query lo
#pragma unroll
          for (int k = 0; k < 8; ++k) {         // K = 128 features in steps of 16
            const uint64_t da =
                ptx::umma_desc_sw128(qb + half * 2 * kQBox + (k >> 2) * kQBox + (k & 3) * 32, 16, 1024);
            const uint64_t db = ptx::umma_desc_sw128(kb + (k >> 2) * kBBox + (k & 3) * 32, 16, 1024);
            ptx::umma_ss(tbase + 256u * h + 64u * (j & 1), da, db, kIdescScore, (half > 0 || k > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(sfull(h, j & 1));
      };
      auto value = [&](int h, int j) {
        const uint32_t vb = sbase + kOffV + (j % kVSlots) * kSlotBytes;
        const uint32_t ts = tbase + 256u * h + 64u * (j & 1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {    // W hi, then W lo
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {        // K = 64 cache rows in steps of 16
            const uint64_t db = ptx::umma_desc_sw128(vb + kk * 2048, kBBox, 1024);
            ptx::umma_ts(tbase + 256u * h + 128u, ts + 32u * half + 8u * kk, db, kIdescValue,
                         (j > 0 || half > 0 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(odone(h));
      };
      bool ok = ptx::mbar_wait_bounded(qready, 0);
      for (int j = 0; j <= nk && ok; ++j) {
        if (*s_abort) {
          ok = false;
          break;
        }
        if (j < nk) {
          if (!(ok = ptx::mbar_wait_bounded(kfull(j % kKSlots), (j / kKSlots) & 1))) break;
          for (int h = 0; h < 2 && ok; ++h) {
            // S buffer (j & 1) is free once the value MMA of tile j - 2 has read its W
            if (j >= 2) ok = ptx::mbar_wait_bounded(odone(h), (j - 2) & 1);
            if (!ok) break;
            ptx::tc_fence_after();
            score(h, j);
          }
          if (!ok) break;
          ptx::umma_commit(kempty(j % kKSlots));
        }
        if (j >= 1) {
          const int jv = j - 1;
          if (!(ok = ptx::mbar_wait_bounded(vfull(jv % kVSlots), (jv / kVSlots) & 1))) break;
          for (int h = 0; h < 2 && ok; ++h) {
            if (!(ok = ptx::mbar_wait_bounded(wready(h, jv & 1), (jv >> 1) & 1))) break;
            ptx::tc_fence_after();
            value(h, jv);
          }
          if (!ok) break;
          ptx::umma_commit(vempty(jv % kVSlots));
        }
      }
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      // every MMA issued by this thread completes before TMEM can be released
      ptx::umma_commit(fin);
      ptx::mbar_wait_bounded(fin, 0);
    }
  } else if (warp == kStagerWarp) {
    // ------------------------------------------------------------ A stager
    // Per tile: A_K (times scale log2(e)/R_K) and A_V (times 1/R_V) of both heads as fp32
    // rows of 64, zero past the sequence end, where B_V rows are zeroed as well.
    const int valid_rows_all = len * R;
    for (int j = 0; j < nk; ++j) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) break;  // the whole warp leaves together
      const int ks = j % kKSlots, vs = j % kVSlots, ab = j & 1;
      bool ok = ptx::mbar_wait_bounded(kfull(ks), (j / kKSlots) & 1) &&
                ptx::mbar_wait_bounded(vfull(vs), (j / kVSlots) & 1);
      // the softmax warps of both heads are done with buffer ab (tile j - 2)
      if (ok && j >= 2)
        ok = ptx::mbar_wait_bounded(wready(0, ab), ((j - 2) >> 1) & 1) &&
             ptx::mbar_wait_bounded(wready(1, ab), ((j - 2) >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
        break;
      }
      const uint8_t* ka = gbase + kOffK + ks * kSlotBytes + kBBytes;
      uint8_t* vslot = gbase + kOffV + vs * kSlotBytes;
      const uint8_t* va = vslot + kBBytes;
      float* sa = s_a + ab * 4 * kRows;
      bool zeroed = false;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int r = lane + 32 * half;
        const bool valid = j * kRows + r < valid_rows_all;
        const uint32_t k2 = *reinterpret_cast<const uint32_t*>(ka + r * 16 + a_off * 2);
        const uint32_t v2 = *reinterpret_cast<const uint32_t*>(va + r * 16 + a_off * 2);
        sa[0 * kRows + r] = valid ? ptx::bf16_lo(k2) * p.zs : 0.f;
        sa[1 * kRows + r] = valid ? ptx::bf16_hi(k2) * p.zs : 0.f;
        sa[2 * kRows + r] = valid ? ptx::bf16_lo(v2) * p.inv_rv : 0.f;
        sa[3 * kRows + r] = valid ? ptx::bf16_hi(v2) * p.inv_rv : 0.f;
        if (!valid) {
          // a B_V row past the sequence end may hold NaN; 0 * NaN would reach every O row
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(vslot + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(vslot + kBBox + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          zeroed = true;
        }
      }
      if (zeroed) ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(staged(ab));
        ptx::mbar_arrive(kempty(ks));
        ptx::mbar_arrive(vempty(vs));
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int h = (warp - 2) >> 2;             // head 2 hp + h
    const int head = 2 * hp + h;
    const int row = quad * 32 + lane;          // query row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tq = q0 + row;                   // query index in the chunk
    const int qslot = P + tq;                  // its cache slot: keys s <= qslot
    const uint32_t t_o = tbase + 256u * h + 128u;
    // stage this thread's query row as bf16 hi + lo (K-major, 128-byte swizzle; zeros past the chunk)
    {
      const float* qr = p.q + ((static_cast<size_t>(b) * p.n_tokens + tq) * kH + head) * kD;
      uint8_t* qh = gbase + kOffQ + h * kQHead;
#pragma unroll
      for (int c = 0; c < 16; ++c) {           // 16 chunks of 8 features
        float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
        if (tq < p.n_tokens) {
          v0 = *reinterpret_cast<const float4*>(qr + 8 * c);
          v1 = *reinterpret_cast<const float4*>(qr + 8 * c + 4);
        }
        const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = ptx::pack_bf16(f[2 * e], f[2 * e + 1]);
          lo[e] = ptx::pack_bf16(f[2 * e] - ptx::bf16_lo(hi[e]), f[2 * e + 1] - ptx::bf16_hi(hi[e]));
        }
        const int box = c >> 3, chunk = c & 7;
        const int off = box * kQBox + row * 128 + ((chunk ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(qh + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(qh + 2 * kQBox + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(qready);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int ab = j & 1;
      bool fail = *s_abort != 0;
      if (!fail)
        fail = !ptx::mbar_wait_bounded(sfull(h, ab), (j >> 1) & 1) ||
               !ptx::mbar_wait_bounded(staged(ab), (j >> 1) & 1);
      if (!__all_sync(0xffffffffu, !fail)) {  // warp-wide TMEM accesses follow: leave together
        if (lane == 0) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const float* ak = s_a + ab * 4 * kRows + h * kRows;        // scaled A_K of this head, per row
      const float* av = s_a + ab * 4 * kRows + (2 + h) * kRows;  // A_V / R_V of this head, per row
      const uint32_t ts = tbase + 256u * h + 64u * ab + lane_off;
      // ---- scores: z[s] for the TOK tokens of the tile (log2 units)
      float z[TOK];
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t sv[32];
        ptx::tmem_ld32(ts + 32 * c2, sv);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 a4 = reinterpret_cast<const float4*>(ak + 32 * c2)[e4];
          const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
          for (int u = 0; u < 4; u += R) {
            const int e = 4 * e4 + u;  // row within this 32-row chunk
            float acc = __uint_as_float(sv[e]) * a[u];
            if (R == 2) acc = fmaf(__uint_as_float(sv[e + 1]), a[u + 1], acc);
            z[(32 * c2 + e) / R] = acc;
          }
        }
      }
      const int tok0 = j * TOK;
      const bool need_mask = tok0 + TOK - 1 > P + q0;  // the tile reaches past some query's own slot
      float mx = -INFINITY;
#pragma unroll
      for (int s = 0; s < TOK; ++s) {
        if (need_mask && tok0 + s > qslot) z[s] = -INFINITY;
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
        const bool o_prev = ptx::mbar_wait_bounded(odone(h), (j - 1) & 1);
        if (!__all_sync(0xffffffffu, o_prev)) {
          if (lane == 0) {
            atomicOr(p.err, kErrTimeout);
            *s_abort = 1;
          }
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
      // ---- W = p A_V / R_V as bf16 hi + lo, two cache rows per TMEM column, over S
      uint32_t whi[32], wlo[32];
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 a4 = reinterpret_cast<const float4*>(av)[e4];
        const float a[4] = {a4.x, a4.y, a4.z, a4.w};
        float w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rr = 4 * e4 + u;
          const int s = rr / R;
          const float pz = exp2f(z[s] - m);  // 0 for masked keys (z = -inf, m finite)
          w[u] = pz * a[u];
          if (rr % R == 0) l += pz;
        }
        whi[2 * e4] = ptx::pack_bf16(w[0], w[1]);
        whi[2 * e4 + 1] = ptx::pack_bf16(w[2], w[3]);
        wlo[2 * e4] = ptx::pack_bf16(w[0] - ptx::bf16_lo(whi[2 * e4]), w[1] - ptx::bf16_hi(whi[2 * e4]));
        wlo[2 * e4 + 1] =
            ptx::pack_bf16(w[2] - ptx::bf16_lo(whi[2 * e4 + 1]), w[3] - ptx::bf16_hi(whi[2 * e4 + 1]));
      }
      ptx::tmem_st32(ts, whi);
      ptx::tmem_st32(ts + 32, wlo);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(wready(h, ab));
    }
    // ---- epilogue: O / l to out[b][t][head][:] once every MMA of this CTA has completed
    const bool o_ready = ok && ptx::mbar_wait_bounded(fin, 0);
    if (__all_sync(0xffffffffu, o_ready)) {  // the TMEM loads below are warp-wide
      ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* op = p.out + ((static_cast<size_t>(b) * p.n_tokens + tq) * kH + head) * kD;
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
    } else if (ok && lane == 0) {
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
  if ((e = encode_bf16_2d(&tbk, cv.b_k, kD, rows_k, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tbv, cv.b_v, kD, rows_v, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tak, cv.a_k, kH, rows_k, kASlice, kRows, 0)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tav, cv.a_v, kH, rows_v, kASlice, kRows, 0)) != cudaSuccess) return e;
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
  dim3 grid(cv.batch * (kH / 2), p.n_qtiles);
  auto kern = cv.r_k == 1 ? prefill_tc_kernel<1> : prefill_tc_kernel<2>;
  kern<<<grid, kThreads, kSmemBytes, stream>>>(p, tbk, tbv, tak, tav);
  return cudaGetLastError();
}

}  // namespace tpa
