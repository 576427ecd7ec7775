// Causal prefill on the 5th-generation tensor cores (tcgen05, TMEM
// accumulators, TMA), bf16 cache, h = 32, d_h = 128, R_K = R_V = R in {1, 2},
// R_Q <= 8.
//
// What it computes (Tensor Product Attention Is All You Need, sections
// 解决思路 for Q_t = (1/R_Q) A_Q^T B_Q, 关键设计 / 张量积分解 for the K/V
// factors, RoPE 兼容性 for RoPE on the B factors, FlashTPA for attention on
// the factors): for query t of a chunk (cache slot P + t) and head i,
//   q_{t,i}     = (1/R_Q) sum_j A_Q[t, j, i] RoPE(B_Q[t, j], pos_t)
//   S[t, (s,r)] = q_{t,i} . B~_K[s, r]                       (tensor cores)
//   z[t, s]     = scale/R_K sum_r A_K[s, r, i] S[t, (s, r)],  s <= P + t
//   W[t, (s,r)] = softmax_s(z)[t, s] A_V[s, r, i] / R_V
//   O[t, i, :]  = sum_(s,r) W[t, (s,r)] B_V[s, r, :]         (tensor cores)
// Keys and values stay factorized: the score MMA contracts the query with B_K
// rows, and the value MMA contracts the softmax weights with B_V rows.  Putting
// the head factors on the query side of the MMA (a dense query tile per head)
// costs 2 h d_h R_K tensor flops per (query, key) pair and little CUDA-core
// work; contracting B_Q with B_K first would save tensor flops but needs
// ~h R_Q R_K CUDA-core FMAs per pair to apply A_Q and A_K, on the CUDA cores
// that the softmax already keeps busy.
//
// Operands are fp16.  A pre-pass (prefill_prep_kernel, launched just before)
// writes to the workspace (i) fp16 copies of the B_K and B_V rows of every
// sequence's cached tokens, exact for bf16 values in fp16's normal range
// (bf16's 8 significant bits fit in fp16's 11; magnitudes above 65504 are not
// supported by this path and become infinite), and (ii) the chunk's B_Q rank
// rows rotated at their positions, rounded to fp16 and interleaved by 32
// queries (wq_chunk).  The dense per-head query is formed in this kernel from
// (ii) and A_Q, in fp32, and rounded once to fp16 in TMEM; it is never written
// to global memory.  With the softmax
// weights also rounded once to fp16 (11 significant bits: ~4e-4 relative each
// on the prefill workload, against ~3.5e-3 for a bf16 rounding) one MMA per
// contraction suffices where bf16 needed a high + low pair.
//
// CTA = (sequence, head, tile of 128 queries); heavy (late) query tiles are
// dispatched first.  Both MMAs take their A operand from TMEM, so shared
// memory only feeds their B operands (a 128-row B_K or B_V tile per 16 of K).
// Roles (352 threads): warp 0 issues TMA loads of 128-row tiles {B_K, B_V (the
// fp16 copies), the 8-head slices of A_K and A_V holding the head} into a
// 3-stage ring; warp 1 allocates all 512 TMEM columns and one of its threads
// issues the MMAs; warps 2-9 form the queries, then run the softmax, two
// threads per query row (TMEM lane): warps 2-5 take the first 64 cache rows
// of a tile, warps 6-9 the last 64; warp 10 stages A_K and A_V of the head as
// fp32 (scales folded in) and zeroes B_V rows past the sequence end, which
// may hold NaN.
// TMEM: S double-buffered in columns [128 b, +128) and overwritten in place by
// W (fp16, two cache rows per column, the first 64 columns), O in [256, 384),
// the query (fp16) in [384, 448).  Per key tile j:
//   S = Q B_K^T  (M = 128 queries, N = 128 rows, K = 128), into the buffer
//       that tile j - 1 does not use, so it overlaps the softmax of tile j - 1;
//   softmax: A_K weighting, causal mask, online softmax with a lazily
//       rescaled maximum (only when it grows by more than 2^4; the two threads
//       of a row share their maxima through shared memory), W = p A_V / R_V
//       with p = 2^(z - m - 2): the keys near the maximum get p in [1/4, 4],
//       so their weights stay in fp16's normal range for |A_V| / R_V from
//       2.4e-4 to 16376 (the row sum takes the same factor, which cancels in
//       O / l);
//   O += W B_V  (B_V MN-major).
// The softmax's per-tile work is trimmed: the second half of a thread's scores is loaded from
// TMEM while the first half is weighted, the row maximum is a tree of three-input maxima, and the
// weights use two-wide fp32 arithmetic.  At the end O / l goes through shared memory (the K/V
// stages, idle by then) and each warp writes whole 512-byte output rows.
// Every wait is bounded (2 s); a timeout sets the error word and an abort
// flag, and TMEM is released only after the MMA thread's last commit.
#include <cuda.h>
#include <cuda_fp16.h>
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
constexpr int kRows = 128;              // cache rows per key tile
constexpr int kHalfRows = kRows / 2;    // rows per softmax thread
constexpr int kStages = 3;
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = (3 + kSoftmaxWarps) * 32;
constexpr int kStagerWarp = 2 + kSoftmaxWarps;
constexpr int kBBox = kRows * 128;        // 64 features x 128 rows, bf16: 16 KB
constexpr int kBBytes = 2 * kBBox;        // one B tile
constexpr int kASlice = 8;                // heads in the A slice a tile carries (16 bytes per row)
constexpr int kABytes = kRows * kASlice * 2;
constexpr int kStageBytes = 2 * kBBytes + 2 * kABytes;  // B_K, B_V, A_K slice, A_V slice
constexpr int kOffStages = 0;
constexpr int kOffA = kOffStages + kStages * kStageBytes;  // fp32 [2 buffers][A_K, A_V][128]
constexpr int kOffMx = kOffA + 2 * 2 * kRows * 4;          // fp32 [2 buffers][2 halves][128 rows]
constexpr int kOffL = kOffMx + 2 * 2 * kQ * 4;             // fp32 [2 halves][128 rows]
constexpr int kOffBar = kOffL + 2 * kQ * 4;
// full[3], empty[3], sfull[2], wready[2], staged[2], qready, fin
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 1 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr size_t kSmemBytes = 1024 + kOffMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
static_assert(kStageBytes % 1024 == 0 && kBBox % 1024 == 0, "swizzle atoms stay aligned");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256, kColQ = 384;
constexpr unsigned kErrTimeout = 0x8u;
constexpr int kOPitch = kD + 4;          // floats per staged output row (528 bytes)
constexpr uint32_t kEpilogueBar = 5;     // named barrier of the softmax warps (1-4: the row pairs)
static_assert(kQ * kOPitch * 4 <= kStages * kStageBytes, "the staged output fits in the K/V stages");
constexpr float kLazy = 4.f;  // rescale only when a row maximum grows by more than 2^4
constexpr float kShift = 2.f;  // p = 2^(z - m - kShift): at most 2^(kLazy - kShift) = 4
constexpr int kMaxRq = 8;

// kind::f16 instruction descriptors, D fp32, A (TMEM) and B fp16, M = 128, N = 128;
// the value MMA's B (the B_V tile) is MN-major.
constexpr uint32_t kIdescScore = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescValue = kIdescScore | (1u << 16);

struct PrefillTcParams {
  const int32_t* seq_lens;
  int batch, capacity, n_tokens, n_qtiles;
  float zs;       // scale * log2(e) / R_K
  float inv_rv;   // 1 / R_V
  int r_q;
  float inv_rq;                // 1 / R_Q
  const __nv_bfloat16* a_q;    // [B][T][R_Q][32]
  const __half* bq_rot;        // [B][T][R_Q][128] rank rows rotated at their positions (the pre-pass)
  float* out;      // [B][T][32][128]
  unsigned int* err;
};

// Two-wide fp32 arithmetic: one instruction for both lanes of a pair.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(*reinterpret_cast<const uint64_t*>(&a)),
      "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(*reinterpret_cast<const uint64_t*>(&a)),
      "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&d);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(*reinterpret_cast<const uint64_t*>(&a)),
      "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<const float2*>(&d);
}

// max of three (one instruction)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// The maximum of n values as a tree of three-input maxima (depth log3 n instead of n).
template <int N>
__device__ __forceinline__ float max_tree(const float* v) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return fmaxf(v[0], v[1]);
  } else {
    constexpr int A = (N + 2) / 3, B = (N - A + 1) / 2;
    return max3(max_tree<A>(v), max_tree<B>(v + A), max_tree<N - A - B>(v + A + B));
  }
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float2 unpack_f16(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

struct PrepParams {
  const int32_t* seq_lens;
  int batch, capacity, r, n_tokens, r_q;
  const __nv_bfloat16* b_k;   // the cache planes
  const __nv_bfloat16* b_v;
  const __nv_bfloat16* b_q;   // [B][T][R_Q][128], unrotated
  const int32_t* q_pos;       // [B][T]
  __half* wk;                 // fp16 copies [B][cap][R][128]
  __half* wv;
  __half* wq;                 // rotated rank rows, interleaved by 32 queries (wq_chunk)
  RopeTable rope;
};

// The rotated B_Q rank rows in the workspace, in 16-byte chunks of 8 features: chunk c (features
// 64 hf + 8 c .. + 7) of rank j of query t = 32 blk + r sits at this index, so that the 32 queries
// a warp of the attention kernel forms (one per lane) read 512 contiguous bytes per load.
__host__ __device__ __forceinline__ size_t wq_chunk(int b, int n_blk, int blk, int r_q, int j, int hf, int c, int r) {
  return (((static_cast<size_t>(b) * n_blk + blk) * r_q + j) * 16 + hf * 8 + c) * 32 + r;
}

// The pre-pass.  blockIdx.z = 0, 1: fp16 copies of the B_K, B_V rows of every sequence's
// cached tokens (slots below seq_lens[b]), blockIdx.y striding over the sequences; z = 2: the
// chunk's B_Q rank rows rotated at their positions, rounded to fp16, into the interleaved layout
// of wq_chunk (one thread per (query, 8 features), queries fastest: the cos and sin of its 4
// pairs are formed once for all ranks).
__global__ void __launch_bounds__(256) prefill_prep_kernel(const __grid_constant__ PrepParams p) {
  ptx::pdl_launch_dependents();  // the attention grid may start its set-up
  if (blockIdx.z < 2) {
    for (int b = blockIdx.y; b < p.batch; b += gridDim.y) {
      const int len = min(max(p.seq_lens[b], 0), p.capacity);
      const size_t base = static_cast<size_t>(b) * p.capacity * p.r * kD;
      const uint4* src = reinterpret_cast<const uint4*>((blockIdx.z == 0 ? p.b_k : p.b_v) + base);
      uint4* dst = reinterpret_cast<uint4*>((blockIdx.z == 0 ? p.wk : p.wv) + base);
      const size_t nvec = static_cast<size_t>(len) * p.r * kD / 8;
      const size_t step = static_cast<size_t>(gridDim.x) * blockDim.x;
      // four 16-byte vectors per thread in flight, each load of the warp 512 contiguous bytes
      for (size_t v = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec; v += 4 * step) {
        uint4 x[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = v + k * step < nvec ? src[v + k * step] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (v + k * step < nvec) {
            uint4 y;
            y.x = pack_f16(ptx::bf16_lo(x[k].x), ptx::bf16_hi(x[k].x));
            y.y = pack_f16(ptx::bf16_lo(x[k].y), ptx::bf16_hi(x[k].y));
            y.z = pack_f16(ptx::bf16_lo(x[k].z), ptx::bf16_hi(x[k].z));
            y.w = pack_f16(ptx::bf16_lo(x[k].w), ptx::bf16_hi(x[k].w));
            dst[v + k * step] = y;
          }
        }
      }
    }
    return;
  }
  const int n_blk = (p.n_tokens + 31) / 32;
  const size_t n = static_cast<size_t>(p.batch) * n_blk * 16 * 32;
  const size_t stride = static_cast<size_t>(gridDim.x) * gridDim.y * blockDim.x;
  for (size_t e = (static_cast<size_t>(blockIdx.y) * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += stride) {
    const int r = static_cast<int>(e % 32);
    const int ch = static_cast<int>((e / 32) % 16);  // features 8 ch .. 8 ch + 7: pairs 4 ch .. 4 ch + 3
    const int blk = static_cast<int>((e / 512) % n_blk);
    const int b = static_cast<int>(e / (512 * static_cast<size_t>(n_blk)));
    const int t = 32 * blk + r;
    if (t >= p.n_tokens) continue;
    const size_t qrow = static_cast<size_t>(b) * p.n_tokens + t;
    const int pos = p.q_pos[qrow];
    float cs[4], sn[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) rope_cos_sin(pos, p.rope.theta[4 * ch + k], &cs[k], &sn[k]);
    uint4* dst = reinterpret_cast<uint4*>(p.wq);
    uint4 x[kMaxRq];  // every rank's 16 bytes in flight at once
#pragma unroll
    for (int j = 0; j < kMaxRq; ++j)
      x[j] = j < p.r_q ? reinterpret_cast<const uint4*>(p.b_q + (qrow * p.r_q + j) * kD)[ch] : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < kMaxRq; ++j) {
      if (j < p.r_q) {
        const uint32_t w[4] = {x[j].x, x[j].y, x[j].z, x[j].w};
        uint32_t y[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float a = ptx::bf16_lo(w[k]), bb = ptx::bf16_hi(w[k]);
          rope_pair(a, bb, cs[k], sn[k]);
          y[k] = pack_f16(a, bb);
        }
        dst[wq_chunk(b, n_blk, blk, p.r_q, j, ch >> 3, ch & 7, r)] = make_uint4(y[0], y[1], y[2], y[3]);
      }
    }
  }
}

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillTcParams p,
                      const __grid_constant__ CUtensorMap tm_bk, const __grid_constant__ CUtensorMap tm_bv,
                      const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_av) {
  constexpr int TOK = kRows / R;           // tokens per key tile
  constexpr int TOKH = kHalfRows / R;      // tokens per softmax thread
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  float* s_a = reinterpret_cast<float*>(gbase + kOffA);
  float* s_mx = reinterpret_cast<float*>(gbase + kOffMx);
  float* s_l = reinterpret_cast<float*>(gbase + kOffL);
  const uint32_t bar0 = sbase + kOffBar;
  auto full = [&](int s) { return bar0 + 8 * s; };
  auto empty = [&](int s) { return bar0 + 8 * (kStages + s); };
  auto sfull = [&](int b) { return bar0 + 8 * (2 * kStages + b); };
  auto wready = [&](int b) { return bar0 + 8 * (2 * kStages + 2 + b); };
  auto staged = [&](int b) { return bar0 + 8 * (2 * kStages + 4 + b); };
  const uint32_t qready = bar0 + 8 * (2 * kStages + 6);
  const uint32_t fin = bar0 + 8 * (2 * kStages + 7);
  volatile uint32_t* s_taddr = reinterpret_cast<volatile uint32_t*>(gbase + kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(gbase + kOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // heavy query tiles first: blockIdx.y runs over query tiles from the last one down
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.y);
  const int head = blockIdx.x % kH;
  const int b = blockIdx.x / kH;
  const int q0 = qt * kQ;
  const int len = p.seq_lens[b];
  const int P = len - p.n_tokens;
  if (len > p.capacity || P < 0) {
    if (tid == 0 && head == 0 && qt == 0) atomicOr(p.err, TPA_DEVERR_PREFILL_LEN);
    return;
  }
  const int q_hi = min(q0 + kQ, p.n_tokens);  // queries [q0, q_hi) are real
  const int key_end = P + q_hi;                // keys [0, key_end) are needed
  const int nk = (key_end + TOK - 1) / TOK;
  const int a_x = kASlice * (head / kASlice);  // first head of the A slice
  const int a_off = head - a_x;                 // the head within the slice

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 2);  // value-MMA commit + the stager (A slices read, B_V rows zeroed)
    }
    for (int bf = 0; bf < 2; ++bf) {
      ptx::mbar_init(sfull(bf), 1);
      ptx::mbar_init(wready(bf), kSoftmaxWarps);
      ptx::mbar_init(staged(bf), 1);
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
      ptx::pdl_wait();  // the fp16 copies of B_K and B_V
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        if (*s_abort) {
          ok = false;
          break;
        }
        const int st = j % kStages;
        if (j >= kStages && !(ok = ptx::mbar_wait_bounded(empty(st), ((j / kStages) & 1) ^ 1))) break;
        const int row0 = (b * p.capacity + j * TOK) * R;
        const uint32_t sb = sbase + kOffStages + st * kStageBytes;
        ptx::mbar_arrive_expect_tx(full(st), kStageBytes);
        ptx::tma_load_2d(sb, &tm_bk, 0, row0, full(st));
        ptx::tma_load_2d(sb + kBBox, &tm_bk, 64, row0, full(st));
        ptx::tma_load_2d(sb + kBBytes, &tm_bv, 0, row0, full(st));
        ptx::tma_load_2d(sb + kBBytes + kBBox, &tm_bv, 64, row0, full(st));
        ptx::tma_load_2d(sb + 2 * kBBytes, &tm_ak, a_x, row0, full(st));
        ptx::tma_load_2d(sb + 2 * kBBytes + kABytes, &tm_av, a_x, row0, full(st));
        ++issued;
      }
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
        // every load already issued lands before the CTA can exit
        for (int k = max(0, issued - kStages); k < issued; ++k)
          ptx::mbar_wait_bounded(full(k % kStages), (k / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Order: S(0); then for each tile j: S(j+1) into the other buffer (after the value MMA
    // of tile j-1 has consumed the W stored there), then O += W(j) B_V once the softmax of
    // tile j is done.  The score MMA of tile j+1 thus runs while the softmax works on tile j.
    if (lane == 0) {
      auto score = [&](int j) {
        const uint32_t sb = sbase + kOffStages + (j % kStages) * kStageBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // K = 128 features in steps of 16
          const uint64_t db = ptx::umma_desc_sw128(sb + (k >> 2) * kBBox + (k & 3) * 32, 16, 1024);
          ptx::umma_ts(tbase + 128u * (j & 1), tbase + kColQ + k * 8, db, kIdescScore, k > 0 ? 1u : 0u);
        }
        ptx::umma_commit(sfull(j & 1));
      };
      bool ok = ptx::mbar_wait_bounded(qready, 0) && ptx::mbar_wait_bounded(full(0), 0);
      if (ok) {
        ptx::tc_fence_after();
        score(0);
      }
      for (int j = 0; j < nk && ok; ++j) {
        if (*s_abort) {
          ok = false;
          break;
        }
        if (j + 1 < nk) {
          ok = ptx::mbar_wait_bounded(full((j + 1) % kStages), ((j + 1) / kStages) & 1);
          // the value MMA of tile j-1 has read W(j-1) there: its stage's release says so (the
          // stager's arrival for that stage came long before)
          if (ok && j > 0) ok = ptx::mbar_wait_bounded(empty((j - 1) % kStages), ((j - 1) / kStages) & 1);
          if (!ok) break;
          ptx::tc_fence_after();
          score(j + 1);
        }
        if (!(ok = ptx::mbar_wait_bounded(wready(j & 1), (j >> 1) & 1))) break;
        ptx::tc_fence_after();
        const uint32_t bv = sbase + kOffStages + (j % kStages) * kStageBytes + kBBytes;
        const uint32_t ts = tbase + 128u * (j & 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {  // K = 128 cache rows in steps of 16
          const uint64_t db = ptx::umma_desc_sw128(bv + kk * 2048, kBBox, 1024);
          ptx::umma_ts(tbase + kColO, ts + kk * 8, db, kIdescValue, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::umma_commit(empty(j % kStages));  // also tells the softmax that O holds tile j
      }
      if (!ok) {
        if (!*s_abort) atomicOr(p.err, kErrTimeout);
        *s_abort = 1;
      }
      // every MMA issued by this thread completes before TMEM can be released; TMEM is released
      // after the time limit all the same, with the error recorded
      ptx::umma_commit(fin);
      if (!ptx::mbar_wait_bounded(fin, 0)) atomicOr(p.err, kErrTimeout);
    }
  } else if (warp == kStagerWarp) {
    // ------------------------------------------------------------ A stager
    // Per tile: A_K (times scale log2(e)/R_K) and A_V (times 1/R_V) of the head as fp32
    // rows of 128, zero past the sequence end, where B_V rows are zeroed as well.
    const int valid_rows_all = len * R;
    for (int j = 0; j < nk; ++j) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) break;  // the whole warp leaves together
      const int st = j % kStages, ab = j & 1;
      bool ok = ptx::mbar_wait_bounded(full(st), (j / kStages) & 1);
      // both softmax halves are done with buffer ab (tile j - 2)
      if (ok && j >= 2) ok = ptx::mbar_wait_bounded(wready(ab), ((j - 2) >> 1) & 1);
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
        break;
      }
      uint8_t* sb = gbase + kOffStages + st * kStageBytes;
      const uint8_t* ka = sb + 2 * kBBytes;
      const uint8_t* va = ka + kABytes;
      float* sa = s_a + ab * 2 * kRows;
      bool zeroed = false;
#pragma unroll
      for (int u = 0; u < kRows / 32; ++u) {
        const int r = lane + 32 * u;
        const bool valid = j * kRows + r < valid_rows_all;
        const float ak = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(ka + r * 16 + a_off * 2));
        const float av = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(va + r * 16 + a_off * 2));
        sa[r] = valid ? ak * p.zs : 0.f;
        sa[kRows + r] = valid ? av * p.inv_rv : 0.f;
        if (!valid) {
          // a B_V row past the sequence end may hold NaN; 0 * NaN would reach every O row
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(sb + kBBytes + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(sb + kBBytes + kBBox + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
          }
          zeroed = true;
        }
      }
      if (zeroed) ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(staged(ab));
        ptx::mbar_arrive(empty(st));
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quad = warp & 3;                 // TMEM lanes 32*quad .. 32*quad+31
    const int hf = (warp - 2) >> 2;            // this thread's half of each key tile
    const int row = quad * 32 + lane;          // query row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tq = q0 + row;                   // query index in the chunk
    const int qslot = min(P + tq, len - 1);    // its cache slot: keys s <= qslot (a padding row: the cached ones)
    const uint32_t pair_bar = 1 + quad;        // named barrier of warps (quad, half 0) and (quad, half 1)
    // features [64 hf, +64) of this thread's query row, q = (1/R_Q) sum_j A_Q[t, j, head] B~_Q[t, j]
    // from the rotated rank rows of the pre-pass (read after the wait on it), formed in fp32 and
    // rounded once to fp16 in TMEM.  The rank rows are interleaved by 32 queries (wq_chunk), so
    // each load of the warp reads 512 contiguous bytes; two ranks' 16 loads are issued at once.
    {
      const size_t qrow = static_cast<size_t>(b) * p.n_tokens + tq;
      const bool real = tq < p.n_tokens;
      float aq[kMaxRq];
#pragma unroll
      for (int j = 0; j < kMaxRq; ++j)
        aq[j] = (real && j < p.r_q) ? __bfloat162float(p.a_q[(qrow * p.r_q + j) * kH + head]) * p.inv_rq : 0.f;
      ptx::pdl_wait();  // the rotated rank rows
      const int n_blk = (p.n_tokens + 31) / 32;
      const uint4* src = reinterpret_cast<const uint4*>(p.bq_rot) +
                         wq_chunk(b, n_blk, q0 / 32 + quad, p.r_q, 0, hf, 0, lane);  // rank j, chunk c: + 512 j + 32 c
      float acc[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) acc[e] = 0.f;
#pragma unroll
      for (int j0 = 0; j0 < kMaxRq; j0 += 2) {
        uint4 v[2][8];
#pragma unroll
        for (int jr = 0; jr < 2; ++jr) {
          const bool use = real && j0 + jr < p.r_q;
#pragma unroll
          for (int c = 0; c < 8; ++c) v[jr][c] = use ? src[512 * (j0 + jr) + 32 * c] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int jr = 0; jr < 2; ++jr) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t w[4] = {v[jr][c].x, v[jr][c].y, v[jr][c].z, v[jr][c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 f = unpack_f16(w[k]);
              acc[8 * c + 2 * k] = fmaf(aq[j0 + jr], f.x, acc[8 * c + 2 * k]);
              acc[8 * c + 2 * k + 1] = fmaf(aq[j0 + jr], f.y, acc[8 * c + 2 * k + 1]);
            }
          }
        }
      }
      uint32_t qh[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) qh[k] = pack_f16(acc[2 * k], acc[2 * k + 1]);
      ptx::tmem_st32(tbase + lane_off + kColQ + 32 * hf, qh);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(qready);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int ab = j & 1;
      bool fail = *s_abort != 0;
      if (!fail) fail = !ptx::mbar_wait_bounded(sfull(ab), (j >> 1) & 1) || !ptx::mbar_wait_bounded(staged(ab), (j >> 1) & 1);
      fail = !__all_sync(0xffffffffu, !fail);  // warp-uniform: warp-wide TMEM loads follow
      ptx::tc_fence_after();
      const float* ak = s_a + ab * 2 * kRows + kHalfRows * hf;          // scaled A_K of this thread's rows
      const float* av = s_a + ab * 2 * kRows + kRows + kHalfRows * hf;  // A_V / R_V of this thread's rows
      const uint32_t ts = tbase + 128u * ab + lane_off;
      // ---- scores: z[s] for this thread's TOKH tokens (log2 units)
      float z[TOKH];
      float mx = -INFINITY;
      if (!fail) {
        uint32_t sv[2][32];
        ptx::tmem_ld32(ts + kHalfRows * hf, sv[0]);
        ptx::tmem_wait_ld();
        ptx::tmem_ld32(ts + kHalfRows * hf + 32, sv[1]);  // in flight while the first half is used
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          if (c2 == 1) ptx::tmem_wait_ld();
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 a4 = reinterpret_cast<const float4*>(ak + 32 * c2)[e4];
            const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int u = 0; u < 4; u += R) {
              const int e = 4 * e4 + u;  // row within this 32-row chunk
              float acc = __uint_as_float(sv[c2][e]) * a[u];
              if (R == 2) acc = fmaf(__uint_as_float(sv[c2][e + 1]), a[u + 1], acc);
              z[(32 * c2 + e) / R] = acc;
            }
          }
        }
        const int tok0 = j * TOK + TOKH * hf;  // first token of this thread's rows
        const bool need_mask = j * TOK + TOK - 1 > P + q0;  // the tile reaches past some query's own slot
        if (need_mask) {
#pragma unroll
          for (int s = 0; s < TOKH; ++s)
            if (tok0 + s > qslot) z[s] = -INFINITY;
        }
        mx = max_tree<TOKH>(z);
      }
      // ---- the row maximum over both halves of the tile: exchange with the partner thread.
      // The pair barrier also orders both threads' S loads before either writes W over S, and
      // carries the abort decision, so that both warps of the pair leave at the same tile.
      float* mxbuf = s_mx + ab * 2 * kQ;
      mxbuf[hf * kQ + row] = mx;
      if (ptx::named_barrier_or(pair_bar, 64, fail)) {
        if (lane == 0) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
        ok = false;
        break;
      }
      mx = fmaxf(mx, mxbuf[(1 - hf) * kQ + row]);
      // ---- online softmax with a lazily rescaled maximum; both threads of a row take the same
      // decision, and the warp-wide TMEM rescale of O runs when any row of the warp needs it
      const bool grow = mx > m + kLazy || (m == -INFINITY && mx != -INFINITY);
      const float alpha = !grow ? 1.f : (m == -INFINITY ? 0.f : ptx::ex2(m - mx));
      if (grow) {
        l *= alpha;
        m = mx;
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // the value MMA of tile j-1 may still be accumulating into O; a timeout here is
        // acted on at the next pair barrier, which both warps of the pair reach
        const bool o_prev = ptx::mbar_wait_bounded(empty((j - 1) % kStages), ((j - 1) / kStages) & 1);
        if (__all_sync(0xffffffffu, o_prev)) {
          ptx::tc_fence_after();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {  // this thread's 64 columns of O
            uint32_t ov[32];
            const uint32_t col = tbase + lane_off + kColO + 64 * hf + 32 * c2;
            ptx::tmem_ld32(col, ov);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            ptx::tmem_st32(col, ov);
          }
        } else if (lane == 0) {
          atomicOr(p.err, kErrTimeout);
          *s_abort = 1;
        }
      }
      // ---- W = p A_V / R_V as fp16, two cache rows per TMEM column, over S; p = 2^(z - m - 2) <= 4
      // (every z <= m + 4 here): the weights near the maximum keep fp16's full precision
      const float mref = m + kShift;
      uint32_t wh[32];
      float2 l2 = make_float2(0.f, 0.f);  // two running partial sums, added at the end
#pragma unroll
      for (int e4 = 0; e4 < 16; ++e4) {
        const float4 a4 = reinterpret_cast<const float4*>(av)[e4];
        float w[4];
        if (R == 2) {
          // tokens s0, s1 = rows (4 e4, +1) and (4 e4 + 2, +3): two-wide fp32 ops
          const int s0 = 2 * e4;
          const float2 d = sub2(make_float2(z[s0], z[s0 + 1]), make_float2(mref, mref));
          const float2 pz = make_float2(ptx::ex2(d.x), ptx::ex2(d.y));  // 0 for masked keys
          l2 = add2(l2, pz);
          const float2 w01 = mul2(make_float2(pz.x, pz.x), make_float2(a4.x, a4.y));
          const float2 w23 = mul2(make_float2(pz.y, pz.y), make_float2(a4.z, a4.w));
          w[0] = w01.x; w[1] = w01.y; w[2] = w23.x; w[3] = w23.y;
        } else {
          const float2 d0 = sub2(make_float2(z[4 * e4], z[4 * e4 + 1]), make_float2(mref, mref));
          const float2 d1 = sub2(make_float2(z[4 * e4 + 2], z[4 * e4 + 3]), make_float2(mref, mref));
          const float2 p0 = make_float2(ptx::ex2(d0.x), ptx::ex2(d0.y));
          const float2 p1 = make_float2(ptx::ex2(d1.x), ptx::ex2(d1.y));
          l2 = add2(l2, add2(p0, p1));
          const float2 w01 = mul2(p0, make_float2(a4.x, a4.y));
          const float2 w23 = mul2(p1, make_float2(a4.z, a4.w));
          w[0] = w01.x; w[1] = w01.y; w[2] = w23.x; w[3] = w23.y;
        }
        wh[2 * e4] = pack_f16(w[0], w[1]);
        wh[2 * e4 + 1] = pack_f16(w[2], w[3]);
      }
      l += l2.x + l2.y;
      ptx::tmem_st32(ts + 32 * hf, wh);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(wready(ab));
    }
    // ---- epilogue: the row sum over both halves, then O / l to out[b][t][head][:]
    // (this thread's 64 features) once every MMA of this CTA has completed
    if (ok) {  // both warps of the pair finished the loop (they leave it only together)
      s_l[hf * kQ + row] = l;
      ptx::named_barrier(pair_bar, 64);
      l += s_l[(1 - hf) * kQ + row];
    }
    // O / l goes through shared memory, so that each warp then writes whole 512-byte output rows
    // (one row of out[b][t][head][:] per instruction) instead of 16 bytes into 32 rows 16 KB
    // apart.  Once every MMA has completed (fin), the K/V stages are no longer read or written:
    // rows of kOPitch floats there, padded so that the 32 rows a warp writes at once spread over
    // the banks.
    const bool o_ready = ok && ptx::mbar_wait_bounded(fin, 0);
    const bool warp_ready = __all_sync(0xffffffffu, o_ready);  // the TMEM loads below are warp-wide
    float* s_o = reinterpret_cast<float*>(gbase + kOffStages);
    if (warp_ready) {
      ptx::tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c2 = 0; c2 < 2; ++c2) {
        uint32_t ov[32];
        ptx::tmem_ld32(tbase + lane_off + kColO + 64 * hf + 32 * c2, ov);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          *reinterpret_cast<float4*>(s_o + row * kOPitch + 64 * hf + 32 * c2 + e) =
              make_float4(__uint_as_float(ov[e]) * inv, __uint_as_float(ov[e + 1]) * inv,
                          __uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
        }
      }
    } else if (ok && lane == 0) {
      atomicOr(p.err, kErrTimeout);
      *s_abort = 1;
    }
    ptx::tc_fence_before();
    // every softmax warp reaches this barrier; its OR says whether any of them could not stage O
    if (!ptx::named_barrier_or(kEpilogueBar, kSoftmaxWarps * 32, !warp_ready)) {
      const int sw = warp - 2;  // rows 16 sw .. 16 sw + 15
#pragma unroll 4
      for (int r = 16 * sw; r < 16 * sw + 16; ++r) {
        if (q0 + r < p.n_tokens) {
          const float4 v = reinterpret_cast<const float4*>(s_o + r * kOPitch)[lane];
          reinterpret_cast<float4*>(p.out + ((static_cast<size_t>(b) * p.n_tokens + q0 + r) * kH + head) * kD)[lane] = v;
        }
      }
    }
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
         r_q <= kMaxRq;
}

namespace {

// The workspace: fp16 copies of B_K and B_V [B][cap][R][128], then the rotated rank rows
// (fp16, B x T rounded up to 32 x R_Q x 128, interleaved as wq_chunk says), each section
// 256-byte aligned.
struct PrefillWorkspace {
  __half* wk;
  __half* wv;
  __half* wq;
  size_t bytes;
};

PrefillWorkspace carve_prefill(void* base, int batch, int capacity, int r, int n_tokens, int r_q) {
  const size_t plane = round256(static_cast<size_t>(batch) * capacity * r * kD * 2);
  const size_t qb = round256(static_cast<size_t>(batch) * ((n_tokens + 31) / 32 * 32) * r_q * kD * 2);
  char* c = static_cast<char*>(base);
  PrefillWorkspace w;
  w.wk = reinterpret_cast<__half*>(c);
  w.wv = reinterpret_cast<__half*>(c ? c + plane : nullptr);
  w.wq = reinterpret_cast<__half*>(c ? c + 2 * plane : nullptr);
  w.bytes = 2 * plane + qb;
  return w;
}

}  // namespace

size_t tensor_prefill_workspace_bytes(int batch, int capacity, int r, int n_tokens, int r_q) {
  return carve_prefill(nullptr, batch, capacity, r, n_tokens, r_q).bytes;
}

cudaError_t launch_tensor_prefill(const TensorPrefillArgs& a, cudaStream_t stream) {
  const CacheView& cv = a.cache;
  const int T = a.n_tokens;
  const int R = cv.r_k;
  const PrefillWorkspace ws = carve_prefill(a.workspace, cv.batch, cv.capacity, R, T, a.r_q);
  PrepParams pp;
  pp.seq_lens = cv.seq_lens;
  pp.batch = cv.batch;
  pp.capacity = cv.capacity;
  pp.r = R;
  pp.n_tokens = T;
  pp.r_q = a.r_q;
  pp.b_k = static_cast<const __nv_bfloat16*>(cv.b_k);
  pp.b_v = static_cast<const __nv_bfloat16*>(cv.b_v);
  pp.b_q = static_cast<const __nv_bfloat16*>(a.b_q);
  pp.q_pos = a.q_pos;
  pp.wk = ws.wk;
  pp.wv = ws.wv;
  pp.wq = ws.wq;
  pp.rope = a.rope;
  // about eight CTAs of 256 threads per SM over the three parts
  const int sms = a.sms > 0 ? a.sms : 148;
  const int gy = min(cv.batch, 65535);
  const size_t vec_per_seq = static_cast<size_t>(cv.capacity) * R * kD / 8;
  size_t gx = (vec_per_seq + 4 * 256 - 1) / (4 * 256);
  const size_t cap_x = static_cast<size_t>(max(1, 8 * sms / max(1, 3 * gy)));
  if (gx > cap_x) gx = cap_x;
  if (gx < 1) gx = 1;
  prefill_prep_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 3), 256, 0, stream>>>(pp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const uint64_t rows = static_cast<uint64_t>(cv.batch) * cv.capacity * R;
  CUtensorMap tbk, tbv, tak, tav;
  // the fp16 copies move as plain 2-byte elements
  if ((e = encode_bf16_2d(&tbk, ws.wk, kD, rows, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tbv, ws.wv, kD, rows, 64, kRows, 128)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tak, cv.a_k, kH, rows, kASlice, kRows, 0)) != cudaSuccess) return e;
  if ((e = encode_bf16_2d(&tav, cv.a_v, kH, rows, kASlice, kRows, 0)) != cudaSuccess) return e;
  if ((e = set_smem_once(R)) != cudaSuccess) return e;
  PrefillTcParams p;
  p.seq_lens = cv.seq_lens;
  p.batch = cv.batch;
  p.capacity = cv.capacity;
  p.n_tokens = T;
  p.n_qtiles = (T + kQ - 1) / kQ;
  p.zs = a.scale * kLog2e / static_cast<float>(R);
  p.inv_rv = 1.f / static_cast<float>(cv.r_v);
  p.r_q = a.r_q;
  p.inv_rq = 1.f / static_cast<float>(a.r_q);
  p.a_q = static_cast<const __nv_bfloat16*>(a.a_q);
  p.bq_rot = ws.wq;
  p.out = a.out;
  p.err = a.err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cv.batch * kH, p.n_qtiles);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = R == 1 ? prefill_tc_kernel<1> : prefill_tc_kernel<2>;
  return cudaLaunchKernelEx(&cfg, kern, p, tbk, tbv, tak, tav);
}

}  // namespace tpa
