// step_fused.cu -- one LoSA denoising step in one kernel launch.
//
// LoSA paper, methodology: locality pruning (MSE of Q_t vs Q_{t-1}, top-|A|
// per head), reuse of the cached prefix state for stable tokens, QUEST page
// selection for active queries only, union of the selected pages, sparse
// prefix attention, dense intra-block suffix, online-softmax merge, cache
// update.
//
// One thread-block cluster of C CTAs per (sequence, KV head) group: up to 16
// (the non-portable cluster size) when every CTA attends the pages of its
// own rows, up to 8 when the whole union is attended and the CTAs' partials
// are combined across the cluster.  The CTAs exchange what they found
// through distributed shared memory at cluster barriers.  Per CTA:
//
//  1. The group's current and previous queries (cp.async), then a ring of
//     32 KB TMA bulk stages over the metadata records of the CTA's
//     contiguous range of prefix pages (with the pages' rounded-up norms),
//     the block's own K/V by cp.async.
//  2. Locality: one thread per token row sums (Qc - Qp)^2 over the channels
//     in channel order, one fp32 rounding per operation -- the oracle's
//     arithmetic exactly, so the active set (top-|A| per head, ties to the
//     lower token) is exact.  Every CTA of the cluster computes it.
//  3. Dense suffix of the CTA's share of the block's token rows on tensor
//     cores (stable rows are merged with their untouched cache and written).
//  4. QUEST bound of every page of the range for the R = G*|A| active rows on
//     tensor cores, U' = [q- | q+] . [kmin ; kmax] (bf16 products exact, the
//     sum the tensor core's).  The channel-order fp32 sum U of the oracle
//     lies within e = |q-| |kmin| + |q+| |kmax| (times 2^-14, every factor
//     rounded up) of U'.  Per row and score chunk: a lower bound of the k-th
//     largest U from group maxima, the pages whose U' + e reaches it, those
//     rescored in the oracle's channel-order arithmetic, and the exact top k
//     by key (value, then lower page first).  fp32 inputs are scored
//     exactly on CUDA cores.
//  5. Cluster barrier.  CTA c merges the rows r = c (mod C) from every CTA's
//     exact list (distributed shared memory): the row's top k over all pages
//     is among the keys at or above the largest k-th key of the lists.  The
//     selection is the oracle's, exactly, by construction.
//  6. Own pages (the default): CTA c gathers the pages of its rows, once
//     each, by 2-D tiled TMA (no multicast, 128-byte swizzle) and folds them
//     into one online-softmax partial per row on tensor cores (P split into
//     bf16 high and remainder parts); with the row's suffix that gives the
//     new o_p / L_p and the output, with no further exchange.  Whole union
//     (an option): the group's union in ascending page order, slot u on CTA
//     u % C, then a cluster barrier and CTA c combines rows r = c (mod C)
//     from every CTA's partial.
//  7. A last cluster barrier keeps every CTA's shared memory alive until the
//     others have read it.
//
// Every wait on a TMA copy is bounded (clock64); a wait that gives up sets
// LOSA_ERR_DEVICE_TIMEOUT in the status word, and the CTA skips the work
// that needs the copy but still takes every cluster barrier.
#include <algorithm>
#include <climits>
#include <cstring>
#include <mutex>

#include "losa_common.cuh"
#include "ptx.cuh"

namespace losa {

// Phase timestamps of the step kernel, compiled in only for the tracing
// build of the library (-DLOSA_PHASE_TRACE; phase_trace.py reads them):
// thread 0 of each of the first kPhaseCtas CTAs stamps the %globaltimer at
// each phase boundary.  The product build has none of this.
constexpr int kPhases = 48;
constexpr int kPhaseCtas = 512;
#ifdef LOSA_PHASE_TRACE
__device__ unsigned long long g_phase[kPhaseCtas * kPhases];
#define LOSA_PHASE(i)                                                                   \
  do {                                                                                  \
    if (threadIdx.x == 0) {                                                             \
      const unsigned cta_ = blockIdx.y * gridDim.x + blockIdx.x;                        \
      if (cta_ < static_cast<unsigned>(kPhaseCtas)) {                                   \
        unsigned long long t_;                                                          \
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                          \
        g_phase[cta_ * kPhases + (i)] = t_;                                             \
      }                                                                                 \
    }                                                                                   \
  } while (0)
// (the same from another thread: `th` instead of thread 0)
#define LOSA_PHASE_BY(i, th)                                                            \
  do {                                                                                  \
    if (threadIdx.x == (th)) {                                                          \
      const unsigned cta_ = blockIdx.y * gridDim.x + blockIdx.x;                        \
      if (cta_ < static_cast<unsigned>(kPhaseCtas)) {                                   \
        unsigned long long t_;                                                          \
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                          \
        g_phase[cta_ * kPhases + (i)] = t_;                                             \
      }                                                                                 \
    }                                                                                   \
  } while (0)
#else
#define LOSA_PHASE(i) \
  do {                \
  } while (0)
#define LOSA_PHASE_BY(i, th) \
  do {                       \
  } while (0)
#endif

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
// CTAs per cluster at most: 8 (the portable size) when the CTAs' partials
// are combined across the cluster, 16 (the non-portable size) when every CTA
// attends the pages of its own rows and nothing is combined across CTAs
constexpr int kMaxCombineCtas = 8;
constexpr int kMaxClusterCtas = 16;
constexpr int kStageBytes = 32 * 1024;
constexpr int kMinStages = 2;
constexpr int kMaxStages = 6;
constexpr int kListSlack = 4;       // buffer entries beyond k kept after a compaction before an exact refinement
constexpr int kMaxGatherPages = 16; // union pages in flight per CTA
constexpr float kEpsScale = 6.103515625e-05f;  // 2^-14: interval half-width per unit of sum |terms|

typedef unsigned long long u64;

// Four elements (channels 4*lane..4*lane+3) of row j of a [16][128] page held
// in shared memory in the element type.
template <int DT>
__device__ __forceinline__ float4 row4(const char* base, int j, int lane) {
  if (DT == LOSA_BF16) {
    const uint2 raw = *reinterpret_cast<const uint2*>(base + (j * kD + 4 * lane) * 2);
    return make_float4(__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                       __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u));
  }
  return *reinterpret_cast<const float4*>(base + (j * kD + 4 * lane) * 4);
}

// Online-softmax update of one row (lane owns 4 channels) with `ntok` <= 16
// keys/values of a page held in shared memory in element type DT.
template <int DT>
__device__ __forceinline__ void attend_page(float4 q, const char* Ks, const char* Vs, int ntok,
                                            float scale_log2, float& m, float& l, float4& acc,
                                            float* Ps) {
  const int lane = threadIdx.x & 31;
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float4 k = row4<DT>(Ks, j, lane);
    v[j] = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    const float send = hi ? v[i] : v[i + 8];
    v[i] = (hi ? v[i + 8] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    const float send = hi ? v[i] : v[i + 4];
    v[i] = (hi ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    const float send = hi ? v[i] : v[i + 2];
    v[i] = (hi ? v[i + 2] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool hi = lane & 2;
    const float send = hi ? v[0] : v[1];
    v[0] = (hi ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  const int key = lane >> 1;  // lanes 2j, 2j+1 hold key j
  const float sc = key < ntok ? v[0] * scale_log2 : -INFINITY;
  const float m_new = fmaxf(m, warp_max(sc));
  const float alpha = exp2f(m - m_new);
  const float p = exp2f(sc - m_new);
  __syncwarp();
  if ((lane & 1) == 0) Ps[key] = p;
  __syncwarp();
  float psum = 0.f;
  float4 o = make_float4(acc.x * alpha, acc.y * alpha, acc.z * alpha, acc.w * alpha);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (j < ntok) {  // rows past the page's last token are never read
      const float pj = Ps[j];
      psum += pj;
      const float4 vv = row4<DT>(Vs, j, lane);
      o.x += pj * vv.x;
      o.y += pj * vv.y;
      o.z += pj * vv.z;
      o.w += pj * vv.w;
    }
  }
  acc = o;
  l = l * alpha + psum;
  m = m_new;
}

// Byte offset of 16-byte chunk c of row j inside a [rows][kD] tile: bf16 tiles
// XOR-swizzle the chunks by row (conflict-free ldmatrix), fp32 tiles are plain.
template <int DT>
__device__ __forceinline__ int tile_off(int j, int c) {
  return DT == LOSA_BF16 ? j * 256 + ((c ^ (j & 7)) << 4) : j * 512 + c * 16;
}

// ---------------------------------------------------------------------------
// Tensor-core attention of one m16 tile of query rows (bf16).  One warp holds
// the tile's state: lane (g4 = lane / 4, t4 = lane % 4) keeps rows g4 and
// g4 + 8 -- the running max m (base-2 units of the scaled score), its share
// of the running sum l (the four lanes of a row are summed at the end), and
// o[n][0..1] (row g4), o[n][2..3] (row g4 + 8) = channels 8n + 2*t4, +1 of
// the unnormalised output.
// ---------------------------------------------------------------------------
struct TileAcc {
  float m[2], l[2];
  float o[16][4];
};

__device__ __forceinline__ void tile_init(TileAcc& t) {
  t.m[0] = t.m[1] = -INFINITY;
  t.l[0] = t.l[1] = 0.f;
#pragma unroll
  for (int n = 0; n < 16; ++n) t.o[n][0] = t.o[n][1] = t.o[n][2] = t.o[n][3] = 0.f;
}

// Byte offset of 16-byte chunk ch (0..15) of key row `key` in a page of K or
// V held in shared memory.  TMA = false: [16][256 B] rows with the chunks
// XOR-swizzled by key (cp.async staging); TMA = true: the two 64-channel
// halves of a 2-D tiled TMA load with the 128-byte swizzle, [2][16][128 B],
// chunks XOR-swizzled by key inside each 128-byte row.
template <bool TMA>
__device__ __forceinline__ int kv_off(int key, int ch) {
  return TMA ? (ch >> 3) * 2048 + key * 128 + (((ch & 7) ^ (key & 7)) << 4)
             : key * 256 + ((ch ^ (key & 7)) << 4);
}

// Fold one page (K, V in the kv_off<TMA> layout, bf16) into the state of the
// 16 query rows at q16 ([16][256 B], chunks swizzled by row).  Row i of the
// tile takes part iff bit i of `rows` is set; keys >= ntok are masked (their
// V rows must be finite: the loaders zero them).
template <bool TMA>
__device__ __forceinline__ void tile_attend(TileAcc& t, const char* q16, const char* Kp,
                                         const char* Vp, uint32_t rows, int ntok, float sl2) {
  const int lane = threadIdx.x & 31, g4 = lane >> 2, t4 = lane & 3;
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ks += 2) {
    uint32_t a0[4], a1[4];
    {
      const int mi = lane >> 3, row = (mi & 1) * 8 + (lane & 7);
      const int ch0 = ks * 2 + (mi >> 1), ch1 = ch0 + 2;
      ldsm_x4(su32(q16 + row * 256 + ((ch0 ^ (row & 7)) << 4)), a0[0], a0[1], a0[2], a0[3]);
      ldsm_x4(su32(q16 + row * 256 + ((ch1 ^ (row & 7)) << 4)), a1[0], a1[1], a1[2], a1[3]);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t b0, b1, b2, b3;
      const int key = nt * 8 + (lane & 7), ch = ks * 2 + (lane >> 3);
      ldsm_x4(su32(Kp + kv_off<TMA>(key, ch)), b0, b1, b2, b3);
      mma_bf16(s[nt], a0, b0, b1);
      mma_bf16(s[nt], a1, b2, b3);
    }
  }
  const bool okA = (rows >> g4) & 1u, okB = (rows >> (g4 + 8)) & 1u;
  float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const bool kv = nt * 8 + 2 * t4 + c < ntok;
      s[nt][c] = (okA && kv) ? s[nt][c] * sl2 : -INFINITY;
      s[nt][2 + c] = (okB && kv) ? s[nt][2 + c] * sl2 : -INFINITY;
      mxA = fmaxf(mxA, s[nt][c]);
      mxB = fmaxf(mxB, s[nt][2 + c]);
    }
  }
  mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
  mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
  mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
  mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
  const float mnA = fmaxf(t.m[0], mxA), mnB = fmaxf(t.m[1], mxB);
  // a row that has seen no key yet keeps m = -inf and exponentiates against 0
  const float uA = mnA == -INFINITY ? 0.f : mnA, uB = mnB == -INFINITY ? 0.f : mnB;
  const float alA = exp2f(t.m[0] - uA), alB = exp2f(t.m[1] - uB);
  t.m[0] = mnA;
  t.m[1] = mnB;
  float psA = 0.f, psB = 0.f;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      s[nt][c] = exp2f(s[nt][c] - uA);
      s[nt][2 + c] = exp2f(s[nt][2 + c] - uB);
      psA += s[nt][c];
      psB += s[nt][2 + c];
    }
  }
  t.l[0] = t.l[0] * alA + psA;
  t.l[1] = t.l[1] * alB + psB;
#pragma unroll
  for (int n = 0; n < 16; ++n) {
    t.o[n][0] *= alA;
    t.o[n][1] *= alA;
    t.o[n][2] *= alB;
    t.o[n][3] *= alB;
  }
  // P (16 rows x 16 keys) as the A operand: bf16 high part and remainder
  uint32_t ah[4], al[4];
  {
    const float pv[8] = {s[0][0], s[0][1], s[0][2], s[0][3], s[1][0], s[1][1], s[1][2], s[1][3]};
    float rem[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) rem[i] = pv[i] - __bfloat162float(__float2bfloat16_rn(pv[i]));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ah[i] = pack_bf16x2(pv[2 * i], pv[2 * i + 1]);
      al[i] = pack_bf16x2(rem[2 * i], rem[2 * i + 1]);
    }
  }
#pragma unroll
  for (int np = 0; np < 8; ++np) {
    uint32_t b0, b1, b2, b3;
    const int key = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int ch = 2 * np + (lane >> 4);
    ldsm_x4_trans(su32(Vp + kv_off<TMA>(key, ch)), b0, b1, b2, b3);
    mma_bf16(t.o[2 * np], ah, b0, b1);
    mma_bf16(t.o[2 * np + 1], ah, b2, b3);
    mma_bf16(t.o[2 * np], al, b0, b1);
    mma_bf16(t.o[2 * np + 1], al, b2, b3);
  }
}

// Sum the four lanes' shares of l.
__device__ __forceinline__ void tile_finish(TileAcc& t) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    t.l[h] += __shfl_xor_sync(0xffffffffu, t.l[h], 1);
    t.l[h] += __shfl_xor_sync(0xffffffffu, t.l[h], 2);
  }
}

// Merge of two normalised attentions (o1, L1), (o2, L2) (natural-log units).
__device__ __forceinline__ void lse_weights(float L1, float L2, float& a, float& b, float& L) {
  const float m = fmaxf(L1, L2);
  const float x = __expf(L1 - m), y = __expf(L2 - m);
  const float inv = __frcp_rn(x + y);
  a = x * inv;
  b = y * inv;
  L = m + __logf(x + y);
}


// ---------------------------------------------------------------------------
// Selection keys with error intervals.  A page scored u on the tensor cores
// has its oracle score (the channel-order fp32 sum) in [u - e, u + e], with
// e = 2^-14 T rounded up and T >= the sum of the terms' magnitudes.  The
// terms are q-_i kmin_i and q+_i kmax_i, so by Cauchy-Schwarz on each half
// T = ||q-|| ||kmin|| + ||q+|| ||kmax|| (every norm and operation rounded
// up) bounds it.  The lower key lk and the upper key uk of [u - e, u + e]
// bracket the page's true key; e = 0 (an exact score) gives lk == uk == the
// exact key.
// ---------------------------------------------------------------------------
// The oracle's bound of page p for one active row, bit for bit: channels in
// order 0..d-1, fp32, one rounding per operation,
//   acc = acc + max(q_i * kmax_i, q_i * kmin_i).
// kmin_i <= kmax_i and rounding is monotone, so for finite values the max is
// q_i * kmax_i when q_i >= 0 and q_i * kmin_i otherwise (a zero product of
// either sign leaves acc unchanged: acc starts at +0 and a sum in
// round-to-nearest is never -0 unless both addends are).  Per 32-bit word of
// two channels, a byte permute that replicates each channel's q sign bit
// gives a 16-bit mask per channel, and one logic op picks kmin under it and
// kmax elsewhere.
// qrow: the row's q (bf16, 16-byte chunks swizzled by r & 7, as staged for
// the tensor cores); rec: page p's metadata record (global or shared memory;
// chunks swizzled by p & 7 as losa_build_page_meta stores them).
__device__ __noinline__ float exact_bound_bf16(const char* qrow, int r, const char* rec, int p) {
  const int rs = r & 7, ps = p & 7;
  // the whole record first (its 32 loads in flight together), then the sum
  uint4 mn[16], mx[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    mn[c] = *reinterpret_cast<const uint4*>(rec + ((c ^ ps) << 4));
    mx[c] = *reinterpret_cast<const uint4*>(rec + ((16 + (c ^ ps)) << 4));
  }
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < 16; ++c) {  // 16-byte chunks of 8 channels, in channel order
    const uint4 q4 = *reinterpret_cast<const uint4*>(qrow + ((c ^ rs) << 4));
    const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
    const uint32_t nw[4] = {mn[c].x, mn[c].y, mn[c].z, mn[c].w};
    const uint32_t xw[4] = {mx[c].x, mx[c].y, mx[c].z, mx[c].w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      // bytes 0-1: the sign of byte 1 (channel 2u's q), bytes 2-3: of byte 3
      const uint32_t neg = prmt(qw[u], 0u, 0xbb99u);
      const uint32_t kw = (nw[u] & neg) | (xw[u] & ~neg);
      // low half = the lower channel
      acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(qw[u] << 16), __uint_as_float(kw << 16)));
      acc = __fadd_rn(acc, __fmul_rn(__uint_as_float(qw[u] & 0xffff0000u),
                                     __uint_as_float(kw & 0xffff0000u)));
    }
  }
  return acc;
}

// Bound scores of one 8-page n-tile for the 16 rows of the A fragments
// ([q- | q+], bf16): u = [q- | q+] . [kmin ; kmax].  u[0..1]: row g4, pages
// 2*t4, 2*t4+1; u[2..3]: row g4 + 8.  `rec0` points to the tile's first
// record; records are [kmin | kmax] with 16-byte chunks swizzled by the page
// index (congruent to the record index mod 8 inside a ring stage).
__device__ __forceinline__ void bound_ntile(const uint32_t (&a)[16][4], const char* rec0,
                                            float (&u)[4]) {
  const int lane = threadIdx.x & 31;
  const int pg = lane & 7;
  // two accumulator chains (even / odd k-steps), added at the end: half the
  // dependent MMA latency
  float u1[4] = {0.f, 0.f, 0.f, 0.f};
  u[0] = u[1] = u[2] = u[3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 16; ks += 2) {
    uint32_t b0, b1, b2, b3;
    const int ch = ks * 2 + (lane >> 3);
    ldsm_x4(su32(rec0 + pg * 512 + ((ch ^ pg) << 4)), b0, b1, b2, b3);
    mma_bf16(u, a[ks], b0, b1);
    mma_bf16(u1, a[ks + 1], b2, b3);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) u[i] += u1[i];
}

// ---------------------------------------------------------------------------
// Per-row candidate lists.  After the CTA's pages are scored, row r's list
// holds its exact top min(k, pages) among the CTA's pages (exact keys), and
// thr[r] the k-th of them; the cluster merge takes the row's top k from the
// C lists.  One warp selects a row.
// ---------------------------------------------------------------------------

// A lower bound of the k-th largest of the 64 values v0, v1 of the warp's
// lanes (0 = none): k rounds each take the largest head over the lanes
// (redux) and pop it from every lane holding it.  Repeats can pop several
// values in a round, which only lowers the result; 0 when fewer than k
// rounds find a value.
__device__ __forceinline__ uint32_t warp_kth64_lb(uint32_t v0, uint32_t v1, int k) {
  uint32_t h0 = max(v0, v1), h1 = min(v0, v1);
  uint32_t m = 0u;
#pragma unroll 1
  for (int i = 0; i < k; ++i) {
    m = __reduce_max_sync(0xffffffffu, h0);
    const bool pop = h0 == m;
    h0 = pop ? h1 : h0;
    h1 = pop ? 0u : h1;
  }
  return m;
}

// The float whose ordered value bits are x (x != 0).
__device__ __forceinline__ float ordered_value(uint32_t x) {
  return __uint_as_float((x & 0x80000000u) ? (x & 0x7fffffffu) : ~x);
}

// Candidates of one active row after another chunk of np of the CTA's
// pages (one warp), in three steps so that a warp can rescore the
// candidates of two rows together.  su[p] is the page's tensor-core score
// (exact for fp32), its interval half-width e = q2.x ||kmin_p|| +
// q2.y ||kmax_p|| (bf16; every operation rounded up).  Before: the row's
// list lk[0..cnt) holds its exact top min(k, pages) over the chunks before,
// thr the k-th key.  After: the same over this chunk's pages too.
//   row_survivors: into the warp's buffer wl/wu go the list and the chunk's
//     pages whose upper key's value word reaches tau0 -- the larger of
//     thr's value word and (a lower bound of) the k-th largest of group
//     maxima of lower-key value words (gm[0..ng), kept by the scoring
//     threads over all pages so far (bf16), else (gm null) 64 sub-maxima of
//     this chunk's pages: lane l, pages l + 32 i, one for even and one for
//     odd i).  A page is tested with u + emax first (emax >= every page's
//     half-width).  More than lb of them (many near-equal scores): the
//     exact path for the chunk.  Returns the buffer's entry count;
//   the caller rescores the inexact entries exactly (the oracle's
//     arithmetic);
//   row_topk: the list keeps the exact top min(k, n) by key, thr the k-th.
// ---------------------------------------------------------------------------
struct ListCount {
  int n;     // entries
  u64 thr;   // their threshold key
};

template <int DT>
__device__ __noinline__ ListCount row_candidates_exact(float* su, int np, int pbase, int k,
                                                       u64* lk, u64* uk, const char* qrow, int r,
                                                       const char* meta_g);

template <int DT>
__device__ __forceinline__ int row_survivors(float* su, const float2* pn, float2 q2, int np,
                                             int pbase, int k, int lb, u64* wl, u64* wu,
                                             const u64* lk, int n0, u64 thr0, const char* qrow,
                                             int r, const char* meta_g, const uint32_t* gm, int ng,
                                             float emax) {
  const int lane = threadIdx.x & 31;
  auto half_width = [&](int p) {
    if (DT != LOSA_BF16) return 0.f;
    const float2 nk = pn[p];
    return __fadd_ru(__fmul_ru(q2.x, nk.x), __fmul_ru(q2.y, nk.y));
  };
  for (int i = lane; i < n0; i += 32) wl[i] = wu[i] = lk[i];
  uint32_t gmax[2] = {0u, 0u};
  if (gm) {
    gmax[0] = lane < ng ? gm[lane] : 0u;
    gmax[1] = lane + 32 < ng ? gm[lane + 32] : 0u;
  } else {
    int i = 0;
#pragma unroll 1
    for (int p = lane; p < np; p += 32, ++i) {
      const uint32_t lo = ordered_bits(__fsub_rd(su[p], half_width(p)));
      if (i & 1)
        gmax[1] = max(gmax[1], lo);
      else
        gmax[0] = max(gmax[0], lo);
    }
  }
  const uint32_t t0 = max(warp_kth64_lb(gmax[0], gmax[1], k), static_cast<uint32_t>(thr0 >> 32));
  const float t0f = t0 ? ordered_value(t0) : -INFINITY;
  // 16 pages per lane at a time (pages p00 + 32 i + lane): a mask of the
  // pages whose u + emax reaches tau0, the exact test of those (few), then
  // the survivors' places by a prefix sum over the lanes
  int ns = n0;
#pragma unroll 1
  for (int p00 = 0; p00 < np; p00 += 32 * 16) {
    uint32_t mask = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int p = p00 + 32 * i + lane;
      if (p < np && __fadd_ru(su[p], emax) >= t0f) mask |= 1u << i;
    }
    uint32_t keep = 0u;
    for (uint32_t m = mask; m; m &= m - 1) {
      const int i = __ffs(m) - 1, p = p00 + 32 * i + lane;
      if (ordered_bits(__fadd_ru(su[p], half_width(p))) >= t0) keep |= 1u << i;
    }
    const int c = __popc(keep);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = ns + incl - c;
    for (uint32_t m = keep; m; m &= m - 1, ++pos) {
      const int i = __ffs(m) - 1, p = p00 + 32 * i + lane;
      const float u = su[p], e = half_width(p);
      if (pos < lb) {
        wl[pos] = sel_key(__fsub_rd(u, e), pbase + p);
        wu[pos] = sel_key(__fadd_ru(u, e), pbase + p);
      }
    }
    ns += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  if (ns > lb || ns > 256) {
    // this chunk's exact top k beside the list (n0 + k <= lb by the plan)
    return n0 + row_candidates_exact<DT>(su, np, pbase, k, wl + n0, wu + n0, qrow, r, meta_g).n;
  }
  return ns;
}

// The exact top min(k, n) of the (exact, distinct) keys wl[0..n): an
// entry's rank is the number of entries above it; the list takes ranks < k
// in rank order, thr the larger of thr0 and the k-th key (if there are k).
__device__ __forceinline__ void row_topk(const u64* wl, int n, int k, u64* lk, int* cnt, u64* thr,
                                         u64 thr0) {
  const int lane = threadIdx.x & 31;
  u64 kth = 0;
#pragma unroll 1
  for (int i = lane; i < n; i += 32) {
    const u64 x = wl[i];
    int rk = 0;
#pragma unroll 4
    for (int j = 0; j < n; ++j) rk += wl[j] > x;
    if (rk < k) lk[rk] = x;
    if (rk == k - 1) kth = x;
  }
  kth = warp_max_u64(kth);
  if (lane == 0) {
    *cnt = min(n, k);
    *thr = kth > thr0 ? kth : thr0;
  }
  __syncwarp();
}

// The exact path (many near-equal scores): every page of the row is
// rescored exactly (the oracle's arithmetic; fp32 scores are exact already)
// and the row's list gets exactly its top min(k, np) pages by exact key
// (value descending, lower page first), thr the k-th of them.
template <int DT>
__device__ __noinline__ ListCount row_candidates_exact(float* su, int np, int pbase, int k,
                                                       u64* lk, u64* uk, const char* qrow, int r,
                                                       const char* meta_g) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  if (DT == LOSA_BF16) {
#pragma unroll 1
    for (int p = lane; p < np; p += 32)
      su[p] = exact_bound_bf16(qrow, r, meta_g + static_cast<size_t>(pbase + p) * 512, pbase + p);
    __syncwarp();
  }
  const int kk = min(k, np);
  // X: the largest value word with at least kk pages at or above it
  uint32_t X = 0u;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = X | (1u << bit);
    int c = 0;
    for (int p = lane; p < np; p += 32) c += ordered_bits(su[p]) >= cand;
    if (__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)) >= static_cast<unsigned>(kk)) X = cand;
  }
  int above = 0;
  for (int p = lane; p < np; p += 32) above += ordered_bits(su[p]) > X;
  const int need_eq = kk - static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(above)));
  // every page above X, then the first need_eq pages (in page order) at X
  int n = 0, eq = 0;
#pragma unroll 1
  for (int p0 = 0; p0 < np; p0 += 32) {
    const int p = p0 + lane;
    const uint32_t x = p < np ? ordered_bits(su[p]) : 0u;
    const bool at = p < np && x == X;
    const unsigned bal_eq = __ballot_sync(0xffffffffu, at);
    const bool in = (p < np && x > X) || (at && eq + __popc(bal_eq & lt) < need_eq);
    eq += __popc(bal_eq);
    const unsigned bal = __ballot_sync(0xffffffffu, in);
    if (in) {
      const int pos = n + __popc(bal & lt);
      lk[pos] = uk[pos] = sel_key(su[p], pbase + p);
    }
    n += __popc(bal);
  }
  __syncwarp();
  return ListCount{n, static_cast<u64>(X) << 32};  // (warp-uniform)
}

// ---------------------------------------------------------------------------
// bf16: the same for a warp's two rows at once (A and B; B absent when
// !hasB), each step of the two rows interleaved so that their latencies
// overlap.  Per row: tau0 = the larger of thr's value word and a lower bound
// of the k-th largest lower-key value word (k rounds over the 64 group
// maxima of the scan); the survivors are the chunk's pages with
// u + emax >= tau0 (rounded up: emax bounds every page's half-width, so no
// page of the row's true top k is dropped); they are rescored exactly (the
// oracle's arithmetic), and with the list they give the exact top k by key.
// More than lb survivors: that row takes the exact path for the chunk.
// ---------------------------------------------------------------------------
struct PairRow {
  const float* su;       // the chunk's tensor-core scores of the row
  u64* w;                // the warp's buffer for the row [lb]
  u64* lk;               // the row's list [lcap]
  int* n;                // its entry count
  u64* thr;              // its threshold key
  const uint32_t* gm;    // group maxima of lower-key value words [ng]
  float emax;            // the largest half-width of the row's pages so far
  const char* qrow;      // the row's staged q
  int r;                 // the active row
};

// Records still in the metadata ring (the last chunk: its last stages are
// not refilled) are read from shared memory by the rescoring.
struct RingView {
  const char* ring;  // the ring's first slot
  int first;         // CTA-local index of the first page still in the ring (or INT_MAX)
  int pr0;           // the CTA's first page
  int tile, stages;  // pages per stage, slots
  __device__ __forceinline__ const char* rec(const char* meta_g, int p) const {
    const int pl = p - pr0;
    if (pl >= first)
      return ring + (pl / tile % stages) * kStageBytes + (pl % tile) * 512;
    return meta_g + static_cast<size_t>(p) * 512;
  }
};

__device__ __forceinline__ void select_pair_bf16(const PairRow& A, const PairRow& B, bool hasB,
                                                 int np, int pbase, int k, int lb, int ng,
                                                 const char* meta_g, const RingView& rv) {
  const int lane = threadIdx.x & 31;
  const int n0A = *A.n, n0B = hasB ? *B.n : 0;
  const u64 thr0A = *A.thr, thr0B = hasB ? *B.thr : 0ull;
  for (int i = lane; i < n0A; i += 32) A.w[i] = A.lk[i];
  for (int i = lane; i < n0B; i += 32) B.w[i] = B.lk[i];
  // tau0 of both rows: k rounds, each popping every lane's head equal to
  // the round's maximum (repeats pop together, which only lowers the bound)
  uint32_t tA, tB;
  {
    const uint32_t a0 = lane < ng ? A.gm[lane] : 0u, a1 = lane + 32 < ng ? A.gm[lane + 32] : 0u;
    const uint32_t b0 = hasB && lane < ng ? B.gm[lane] : 0u;
    const uint32_t b1 = hasB && lane + 32 < ng ? B.gm[lane + 32] : 0u;
    uint32_t ha0 = max(a0, a1), ha1 = min(a0, a1), hb0 = max(b0, b1), hb1 = min(b0, b1);
    uint32_t ma = 0u, mb = 0u;
#pragma unroll 2
    for (int i = 0; i < k; ++i) {
      ma = __reduce_max_sync(0xffffffffu, ha0);
      mb = __reduce_max_sync(0xffffffffu, hb0);
      const bool pa = ha0 == ma, pb = hb0 == mb;
      ha0 = pa ? ha1 : ha0;
      ha1 = pa ? 0u : ha1;
      hb0 = pb ? hb1 : hb0;
      hb1 = pb ? 0u : hb1;
    }
    tA = max(ma, static_cast<uint32_t>(thr0A >> 32));
    tB = max(mb, static_cast<uint32_t>(thr0B >> 32));
  }
  const float tAf = tA ? ordered_value(tA) : -INFINITY;
  const float tBf = tB ? ordered_value(tB) : -INFINITY;
  // survivors: 16 pages per lane and row at a time (pages p00 + 32 i +
  // lane), all loads first, then the places by a prefix sum over the lanes
  int nA = n0A, nB = n0B;
#pragma unroll 1
  for (int p00 = 0; p00 < np; p00 += 32 * 16) {
    float va[16], vb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int p = min(p00 + 32 * i + lane, np - 1);
      va[i] = A.su[p];
      vb[i] = B.su[p];  // (B's pointers are A's when B is absent)
    }
    uint32_t ma = 0u, mb = 0u;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const bool in = p00 + 32 * i + lane < np;
      if (in && __fadd_ru(va[i], A.emax) >= tAf) ma |= 1u << i;
      if (in && hasB && __fadd_ru(vb[i], B.emax) >= tBf) mb |= 1u << i;
    }
    const int ca = __popc(ma), cb = __popc(mb);
    int ia = ca, ib = cb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, ia, o);
      const int yb = __shfl_up_sync(0xffffffffu, ib, o);
      if (lane >= o) {
        ia += ya;
        ib += yb;
      }
    }
    int pa = nA + ia - ca, pb = nB + ib - cb;
    for (uint32_t m = ma; m; m &= m - 1, ++pa)
      if (pa < lb) A.w[pa] = sel_key(0.f, pbase + p00 + 32 * (__ffs(m) - 1) + lane);
    for (uint32_t m = mb; m; m &= m - 1, ++pb)
      if (pb < lb) B.w[pb] = sel_key(0.f, pbase + p00 + 32 * (__ffs(m) - 1) + lane);
    nA += __shfl_sync(0xffffffffu, ia, 31);
    nB += __shfl_sync(0xffffffffu, ib, 31);
  }
  __syncwarp();
  LOSA_PHASE(19);
  // too many survivors (many near-equal scores): the row's exact path
  // (its list and this chunk's exact top k, n0 + k <= lb by the plan)
  int fA = n0A, fB = n0B;  // first entry to rescore
  if (nA > lb) {
    nA = n0A + row_candidates_exact<LOSA_BF16>(const_cast<float*>(A.su), np, pbase, k, A.w + n0A,
                                               A.w + n0A, A.qrow, A.r, meta_g).n;
    fA = nA;
  }
  if (nB > lb) {
    nB = n0B + row_candidates_exact<LOSA_BF16>(const_cast<float*>(B.su), np, pbase, k, B.w + n0B,
                                               B.w + n0B, B.qrow, B.r, meta_g).n;
    fB = nB;
  }
  // the survivors rescored exactly, both rows' entries over the lanes
  const int xa = nA - fA, xt = xa + nB - fB;
#pragma unroll 1
  for (int i = lane; i < xt; i += 32) {
    const bool b = i >= xa;
    u64* slot = b ? B.w + fB + (i - xa) : A.w + fA + i;
    const int p = key_index(*slot);
    const float v = exact_bound_bf16(b ? B.qrow : A.qrow, b ? B.r : A.r, rv.rec(meta_g, p), p);
    *slot = sel_key(v, p);
  }
  __syncwarp();
  LOSA_PHASE(20);
  // each row's exact top min(k, n) by rank (keys are distinct); the entry
  // of rank k - 1 sets the threshold
#pragma unroll 1
  for (int i = lane; i < nA + nB; i += 32) {
    const bool b = i >= nA;
    const int n = b ? nB : nA;
    const u64* w = b ? B.w : A.w;
    const u64 x = w[b ? i - nA : i];
    int rk = 0;
#pragma unroll 4
    for (int j = 0; j < n; ++j) rk += w[j] > x;
    if (rk < k) (b ? B.lk : A.lk)[rk] = x;
    const u64 t0 = b ? thr0B : thr0A;
    if (rk == k - 1) *(b ? B.thr : A.thr) = x > t0 ? x : t0;
  }
  if (lane == 0) {
    *A.n = min(nA, k);
    if (hasB) *B.n = min(nB, k);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Merge of one active row's lists from the C CTAs of the cluster (one warp).
// Every CTA's list holds its exact top min(k, its pages) by exact key, and
// thr its k-th key; the row's top k over all pages is among them, at or
// above the largest thr.  The row's k pages (value descending, lower page
// first) go to sel[0..k) in ascending page order (then -1 when the sequence
// has fewer pages).  `buf` holds the gathered keys (C * lcap of them).
// ---------------------------------------------------------------------------
struct MergeCtx {
  const u64* lk;   // this CTA's list keys [R][lcap] (the same offsets in every CTA)
  const int* n;
  const u64* thr;
  int lcap;        // entries per row list
  int C;
};

__device__ __forceinline__ void merge_row(const MergeCtx& M, int r, int k, u64* blk,
                                          int32_t* sel) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  // one round of remote loads: every CTA's count and threshold (lane = CTA)
  // and every slot of every CTA's list (lane l: slots l, l + 32, ...; slot
  // s is entry s % lcap of CTA s / lcap, the lists at the same offsets in
  // every CTA); slots at or past their CTA's count are dropped below
  int nc = 0;
  u64 th = 0;
  if (lane < M.C) {
    nc = ld_dsmem_s32(dsmem(M.n + r, lane));
    th = ld_dsmem_u64(dsmem(M.thr + r, lane));
  }
  const int slots = M.C * M.lcap;
  const u64* row = M.lk + static_cast<size_t>(r) * M.lcap;
  int cnt = 0;
  u64 tau0 = 0;
#pragma unroll 1
  for (int s0 = 0; s0 < slots; s0 += 4 * 32) {
    u64 x[4];
    int cta[4], idx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int sl = s0 + 32 * i + lane;
      cta[i] = sl < slots ? sl / M.lcap : 0;
      idx[i] = sl - cta[i] * M.lcap;
      x[i] = sl < slots ? ld_dsmem_u64(dsmem(row + idx[i], cta[i])) : 0ull;
    }
    // the row's top k over all pages is among the keys at or above the
    // largest k-th key of the lists
    if (s0 == 0) tau0 = warp_max_u64(th);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int sl = s0 + 32 * i + lane;
      const int ncta = __shfl_sync(0xffffffffu, nc, cta[i]);
      const bool in = sl < slots && idx[i] < ncta && x[i] >= tau0;
      const unsigned bal = __ballot_sync(0xffffffffu, in);
      if (in) blk[cnt + __popc(bal & lt)] = x[i];
      cnt += __popc(bal);
    }
  }
  __syncwarp();
  // the top min(k, cnt) by rank (distinct keys)
#pragma unroll 1
  for (int i = lane; i < cnt; i += 32) {
    const u64 x = blk[i];
    int rk = 0;
#pragma unroll 4
    for (int j = 0; j < cnt; ++j) rk += blk[j] > x;
    if (rk < k) sel[rk] = key_index(x);
  }
  __syncwarp();
  const int nsel = min(cnt, k);
  // ascending page order, then -1 past the selection
  int pv[4];
  int pr[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int e = lane + 32 * t;
    pv[t] = e < nsel ? sel[e] : -1;
    pr[t] = -1;
    if (e < nsel) {
      int rk = 0;
      for (int e2 = 0; e2 < nsel; ++e2) rk += sel[e2] < pv[t];
      pr[t] = rk;
    }
  }
  __syncwarp();
#pragma unroll
  for (int t = 0; t < 4; ++t)
    if (pr[t] >= 0) sel[pr[t]] = pv[t];
  for (int e = nsel + lane; e < k; e += 32) sel[e] = -1;
  __syncwarp();
}

// ---------------------------------------------------------------------------
// The step kernel
// ---------------------------------------------------------------------------
struct StepLayout {
  int ring;     // metadata ring; afterwards merge scratch, gathered pages, warp partials
  int qc, qp;   // the group's queries (current, previous) [GB][rowb]
  int lists;    // candidate lists [R][lcap] (exact keys); per warp survivor keys [2][2][lb]
  int sc;       // fp32: the warps' probability rows (16 floats each)
  int part_o;   // the CTA's partial outputs [R16][kD] floats (bf16: in the ring)
  int part_ml;  // the CTA's partial (m, l) [R16][2] (bf16: in the ring)
  int qa;       // active rows' q_cur [R16][rowb] (bf16 chunks swizzled by row)
  int kbv;      // the block's K then V: [bpad][rowb] each
  int sq;       // this CTA's suffix rows' queries [ns16][rowb]
  int ocache, lcache;  // cached o_p / L_p of its stable suffix rows
  int sfx_o, sfx_l;    // o_s / L_s of its active suffix rows
  int l_n, l_thr;      // list lengths [R], thresholds [R]
  int sel;             // the rows' selected pages [R][k]
  int bitmap, wbase;   // union bitmap and its words' prefix counts
  int lpages, masks;   // this CTA's union pages and their row masks
  int misc;            // per-token / per-row ints and scalars
  int scores;          // the active rows' bound scores of the CTA's pages [R][cp] floats
  int pnorm;           // the CTA's page norms [cp] float2 (bf16)
  int gmx, emx;        // bf16: the rows' group maxima [R16][8 * warps per m16 tile] and
                       // largest half-widths [R16]
  int qn;              // active rows' 2^-14 ||q-||, 2^-14 ||q+|| [R16] float2
  int mbar;            // kMaxStages ring barriers, the queries', the gather's
  int total;
};

struct StepParams {
  const void* qc;
  const void* qp;
  const char* meta;
  const float2* norms;  // the page-norm section of the metadata (row stride pn)
  const void* K;
  const void* V;
  const void* kb;
  const void* vb;
  float* o_p;
  float* l_p;
  float* out;
  float* out_lse;
  int32_t* active_idx;
  int32_t* page_idx;
  int32_t* union_count;
  void* qref;      // drift-safe locality: active rows' q_cur written here (may be null)
  int* status;
  Dims d;
  int C;           // CTAs per cluster (one cluster per (sequence, KV head))
  int cp;          // pages scored per CTA (a multiple of 8)
  int tile;        // pages per ring stage
  int stages;      // ring stages
  int rec;         // bytes per metadata record
  int spc;         // pages per score chunk (a multiple of the stage's pages)
  int lb, lcap;    // survivor buffer entries per warp; list entries per row (k + slack)
  int qstride;     // bytes per staged query row (padded: no bank conflicts between rows)
  int nmw;         // merge warps
  int mstride;     // bytes of a merge warp's scratch (in the ring area)
  int max_lp;      // union pages per CTA, at most
  int ngp;         // union pages in flight per CTA
  int early;       // release the dependent launch at the start (the grid fits one wave)
  int page3d;      // bf16 gather: kmap/vmap are 3-D page maps (one copy per page of K or V)
  int pn;          // page-norm entries per (sequence, KV head)
  StepLayout lo;
};

// misc int area (offsets in ints)
constexpr int kMiscMse = 0;                          // [128] float mse per token row
constexpr int kMiscActTok = kMaxRowsPerGroup;        // [R] active row -> token
constexpr int kMiscActRow = 2 * kMaxRowsPerGroup;    // [R] active row -> token row (h*B + t)
constexpr int kMiscActSlot = 3 * kMaxRowsPerGroup;   // [GB] token row -> active row or -1
constexpr int kMiscSfxTok = 4 * kMaxRowsPerGroup;    // [ns] suffix row -> token row
constexpr int kMiscScal = 5 * kMaxRowsPerGroup;      // scalars below
constexpr int kMiscInts = kMiscScal + 32;
// scalars
constexpr int kSFail = 0, kSNlp = 1, kSWt = 4 /*[4]*/, kSWsum = 8 /*[8]*/;

template <int DT>
__global__ void __launch_bounds__(kThreads, 1)
    losa_step_kernel(const __grid_constant__ StepParams prm,
                     const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap) {
  extern __shared__ __align__(1024) char smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled TMA tiles (the same offset
  // in every CTA, so distributed shared-memory addresses agree)
  char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                       ~static_cast<uintptr_t>(1023));
  const Dims& d = prm.d;
  const StepLayout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int C = prm.C;
  const int c = static_cast<int>(cluster_rank());
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int GB = G * B;
  const int R16 = (R + 15) / 16 * 16;
  constexpr int rowb = DT == LOSA_BF16 ? kD * 2 : kD * 4;
  constexpr int cpr = rowb / 16;
  constexpr int pbytes = kPS * rowb;  // one page of K (or V)
  const int bpad = (B + kPS - 1) / kPS * kPS;
  const size_t grow0 = (static_cast<size_t>(s) * d.Hq + g * G) * B;  // the group's first row
  const bool sel = R > 0 && !d.all_pages;
  const unsigned lt = (1u << lane) - 1u;

  char* ring = smem + lo.ring;
  const char* qcs = smem + lo.qc;
  const char* qps = smem + lo.qp;
  char* qa = smem + lo.qa;
  char* kbv = smem + lo.kbv;
  char* sq = smem + lo.sq;
  float* ocache = reinterpret_cast<float*>(smem + lo.ocache);
  float* lcache = reinterpret_cast<float*>(smem + lo.lcache);
  float* sfx_o = reinterpret_cast<float*>(smem + lo.sfx_o);
  float* sfx_l = reinterpret_cast<float*>(smem + lo.sfx_l);
  // the CTA's partial per active row: bf16 in the ring once the gathered
  // pages are consumed, fp32 in its own area (its running state lives there)
  float* part_o = reinterpret_cast<float*>(smem + lo.part_o);
  float* part_ml = reinterpret_cast<float*>(smem + lo.part_ml);
  // the rows' candidate lists [R][lcap] (exact keys), then per warp its
  // survivor buffers for two rows: lower keys [2][lb], upper keys [2][lb]
  u64* l_lk = reinterpret_cast<u64*>(smem + lo.lists);
  u64* w_lk = l_lk + static_cast<size_t>(R) * prm.lcap + static_cast<size_t>(warp) * 4 * prm.lb;
  u64* w_uk = w_lk + 2 * prm.lb;
  const int qst = prm.qstride;
  float* fscr = reinterpret_cast<float*>(smem + lo.sc);
  int* l_n = reinterpret_cast<int*>(smem + lo.l_n);
  u64* l_thr = reinterpret_cast<u64*>(smem + lo.l_thr);
  int32_t* sel_all = reinterpret_cast<int32_t*>(smem + lo.sel);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + lo.bitmap);
  int32_t* wbase = reinterpret_cast<int32_t*>(smem + lo.wbase);
  int32_t* lpages = reinterpret_cast<int32_t*>(smem + lo.lpages);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + lo.masks);
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  float* s_mse = reinterpret_cast<float*>(misc + kMiscMse);
  int32_t* act_tok = misc + kMiscActTok;
  int32_t* act_row = misc + kMiscActRow;
  int32_t* act_slot = misc + kMiscActSlot;
  int32_t* sfx_tok = misc + kMiscSfxTok;
  int32_t* scal = misc + kMiscScal;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  float* scores = reinterpret_cast<float*>(smem + lo.scores);
  float2* pnorm = reinterpret_cast<float2*>(smem + lo.pnorm);
  uint32_t* gmx = reinterpret_cast<uint32_t*>(smem + lo.gmx);
  uint32_t* emx = reinterpret_cast<uint32_t*>(smem + lo.emx);
  float2* qn = reinterpret_cast<float2*>(smem + lo.qn);
  uint64_t* gbar = mbar + kMaxStages;  // [2]: the gather's two page buffers
  uint64_t* ebar = gbar + 2;            // [kMaxStages]: ring slot released by every warp

  // the next kernel of the stream may be scheduled now when this grid fits
  // one wave (it waits for this grid's completion before it reads anything);
  // otherwise at exit, so that its CTAs never take SMs this grid's later
  // clusters need
  if (prm.early) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (DT == LOSA_BF16 && tid == 0 && d.R > 0) {  // (the page gather's maps; no data read)
    prefetch_tmap(&kmap);
    prefetch_tmap(&vmap);
  }
  // nothing is read before the work queued ahead of the step has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  LOSA_PHASE(0);

  const int Ls = seq_len(d, s);                 // this sequence's prefix length
  const int Ps = (Ls + kPS - 1) / kPS;
  // this CTA's range of pages to score: the sequence's own pages split over
  // the cluster (a sequence shorter than the longest gives each CTA fewer;
  // the plan's buffers are sized for the longest)
  const int cps = min(prm.cp, (((Ps + C - 1) / C) + 7) / 8 * 8);
  const int pr0 = c * cps;
  const int npg = sel ? max(0, min(Ps, pr0 + cps) - pr0) : 0;
  const int nstg = (npg + prm.tile - 1) / prm.tile;
  const char* meta_g = prm.meta + static_cast<size_t>(sg) * d.Pc * prm.rec;
  const float2* norm_g = prm.norms + static_cast<size_t>(sg) * prm.pn;
  // ring stage t (slot t % stages): its records; stage 0 also brings (bf16)
  // the norms of all the CTA's pages, rounded up to a 16-byte copy (the norm
  // rows are padded to 8 entries)
  auto issue_stage = [&](int t) {
    const int st = t % prm.stages;
    const int np = min(prm.tile, npg - t * prm.tile);
    const uint32_t bytes = static_cast<uint32_t>(np * prm.rec);
    const uint32_t nbytes =
        DT == LOSA_BF16 && t == 0 ? static_cast<uint32_t>((npg + 1) / 2 * 16) : 0u;
    mbar_expect_tx(&mbar[st], bytes + nbytes);
    bulk_g2s(ring + st * kStageBytes, meta_g + static_cast<size_t>(pr0 + t * prm.tile) * prm.rec,
             bytes, &mbar[st]);
    if (nbytes) bulk_g2s(pnorm, norm_g + pr0, nbytes, &mbar[st]);
  };

  // the group's current and previous queries (cp.async group 0), rows
  // padded to qst bytes
  {
    const char* qcg = static_cast<const char*>(prm.qc) + grow0 * rowb;
    const char* qpg = static_cast<const char*>(prm.qp) + grow0 * rowb;
    const int per = GB * cpr;
#pragma unroll 1
    for (int e = tid; e < 2 * per; e += kThreads) {
      const int h = e >= per ? 1 : 0, rem = e - h * per, row = rem / cpr, cc = rem - row * cpr;
      cp_async16(su32(smem + (h ? lo.qp : lo.qc) + row * qst + cc * 16),
                 (h ? qpg : qcg) + static_cast<size_t>(row) * rowb + cc * 16, 16u);
    }
    cp_async_commit();
  }
  // the metadata ring (after the queries: they are needed first)
  if (tid == 0) {
    for (int i = 0; i < kMaxStages + 2; ++i) mbar_init(&mbar[i], 1);
    for (int i = 0; i < kMaxStages; ++i) mbar_init(&ebar[i], kWarps);
    fence_mbar_init();
    scal[kSFail] = 0;
    if (c == 0 && g == 0 && seq_len_bad(d, s)) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
#pragma unroll 1
    for (int t = 0; t < min(nstg, prm.stages); ++t) issue_stage(t);
  }
  // the block's K and V (rows >= B zero), chunks swizzled for ldmatrix
  // (cp.async group 1)
  {
    const char* kbg = static_cast<const char*>(prm.kb) + static_cast<size_t>(sg) * B * rowb;
    const char* vbg = static_cast<const char*>(prm.vb) + static_cast<size_t>(sg) * B * rowb;
    const int per = bpad * cpr;
#pragma unroll 1
    for (int e = tid; e < 2 * per; e += kThreads) {
      const int h = e >= per ? 1 : 0, rem = e - h * per, j = rem / cpr, cc = rem - j * cpr;
      const bool ok = j < B;
      const char* src = (h ? vbg : kbg) + static_cast<size_t>(ok ? j : 0) * rowb + cc * 16;
      cp_async16(su32(kbv + h * bpad * rowb + tile_off<DT>(j, cc)), src, ok ? 16u : 0u);
    }
    cp_async_commit();
  }
  cp_async_wait<1>();  // the queries
  __syncthreads();
  const bool qok = true;
  LOSA_PHASE(1);

  // ---- locality: one thread per token row, the oracle's arithmetic exactly
  // (channels in order, fp32, one rounding per operation)
  if (tid < GB) {
    float acc = 0.f;
    if (qok) {
      const char* x = qcs + tid * qst;
      const char* y = qps + tid * qst;
#pragma unroll 2
      for (int cc = 0; cc < cpr; ++cc) {
        const uint4 a = *reinterpret_cast<const uint4*>(x + cc * 16);
        const uint4 b = *reinterpret_cast<const uint4*>(y + cc * 16);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (DT == LOSA_BF16) {
            const float d0 = __fsub_rn(__uint_as_float(aw[u] << 16), __uint_as_float(bw[u] << 16));
            acc = __fadd_rn(acc, __fmul_rn(d0, d0));
            const float d1 = __fsub_rn(__uint_as_float(aw[u] & 0xffff0000u),
                                       __uint_as_float(bw[u] & 0xffff0000u));
            acc = __fadd_rn(acc, __fmul_rn(d1, d1));
          } else {
            const float d0 = __fsub_rn(__uint_as_float(aw[u]), __uint_as_float(bw[u]));
            acc = __fadd_rn(acc, __fmul_rn(d0, d0));
          }
        }
      }
    }
    s_mse[tid] = acc * (1.0f / kD);  // exact: kD is a power of two
  }
  __syncthreads();

  LOSA_PHASE(2);
  // ---- active set: one warp per head, lane = token; rank by (mse desc,
  // token asc); an active row is r = h * A + (its rank among the head's
  // active tokens in token order)
#pragma unroll 1
  for (int h = warp; h < G; h += kWarps) {
    const float x = lane < B ? s_mse[h * B + lane] : 0.f;
    int rk = 0;
#pragma unroll 4
    for (int u = 0; u < B; ++u) {
      const float y = s_mse[h * B + u];
      rk += (y > x) || (y == x && u < lane);
    }
    const bool act = lane < B && rk < A;
    const unsigned bal = __ballot_sync(0xffffffffu, act);
    const int slot = __popc(bal & lt);
    const bool ok = act && slot < A;  // (always, unless an input is NaN)
    if (lane < B) act_slot[h * B + lane] = ok ? h * A + slot : -1;
    if (ok) {
      act_tok[h * A + slot] = lane;
      act_row[h * A + slot] = h * B + lane;
      if (c == 0 && prm.active_idx)
        prm.active_idx[(static_cast<size_t>(s) * d.Hq + g * G + h) * A + slot] = lane;
    }
  }
  __syncthreads();

  // ---- the active rows' interval factors 2^-14 ||q-||, 2^-14 ||q+|| (bf16;
  // one warp per row, every operation rounded up)
  if (DT == LOSA_BF16) {
#pragma unroll 1
    for (int r = warp; r < R; r += kWarps) {
      const uint2 w = *reinterpret_cast<const uint2*>(qcs + act_row[r] * qst + 8 * lane);
      const float x[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                          __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u)};
      float sn = 0.f, sp = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (__float_as_uint(x[i]) & 0x80000000u)
          sn = __fmaf_ru(x[i], x[i], sn);
        else
          sp = __fmaf_ru(x[i], x[i], sp);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sn = __fadd_ru(sn, __shfl_xor_sync(0xffffffffu, sn, o));
        sp = __fadd_ru(sp, __shfl_xor_sync(0xffffffffu, sp, o));
      }
      if (lane == 0)
        qn[r] = make_float2(__fmul_ru(__fsqrt_ru(sn), kEpsScale), __fmul_ru(__fsqrt_ru(sp), kEpsScale));
    }
  }

  // ---- active rows' q_cur for the page tiles and the exact rescoring
  if (DT == LOSA_BF16) {
#pragma unroll 1
    for (int e = tid; e < R16 * 16; e += kThreads) {
      const int r = e / 16, cc = e % 16;
      const uint4 v = r < R ? *reinterpret_cast<const uint4*>(qcs + act_row[r] * qst + cc * 16)
                            : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(qa + tile_off<DT>(r, cc)) = v;
    }
  } else {
#pragma unroll 1
    for (int e = tid; e < R * cpr; e += kThreads) {
      const int r = e / cpr, cc = e % cpr;
      *reinterpret_cast<uint4*>(qa + r * rowb + cc * 16) =
          *reinterpret_cast<const uint4*>(qcs + act_row[r] * qst + cc * 16);
    }
  }

  // ---- this CTA's suffix rows: its active rows r = c + C*j, then every C-th
  // stable token row (in token order)
  const int n_oa = R > c ? (R - c + C - 1) / C : 0;
  const int n_os = GB - R > c ? (GB - R - c + C - 1) / C : 0;
  const int ns = n_oa + n_os;
  {
    bool st = false;
    int pre = 0;
    if (warp < 4) {  // G*B <= 128 token rows
      st = tid < GB && act_slot[tid] < 0;
      const unsigned bal = __ballot_sync(0xffffffffu, st);
      pre = __popc(bal & lt);
      if (lane == 0) scal[kSWt + warp] = __popc(bal);
    }
#pragma unroll 1
    for (int j = tid; j < n_oa; j += kThreads) sfx_tok[j] = act_row[c + C * j];
    __syncthreads();
    if (st) {
      for (int w = 0; w < warp; ++w) pre += scal[kSWt + w];
      if (pre % C == c && n_oa + pre / C < ns) sfx_tok[n_oa + pre / C] = tid;
    }
  }
  __syncthreads();
  {
    const int nsr = DT == LOSA_BF16 ? (ns + 15) / 16 * 16 : ns;
#pragma unroll 1
    for (int e = tid; e < nsr * cpr; e += kThreads) {
      const int n = e / cpr, cc = e - n * cpr;
      const uint4 v = n < ns ? *reinterpret_cast<const uint4*>(qcs + sfx_tok[n] * qst + cc * 16)
                             : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(sq + tile_off<DT>(n, cc)) = v;
    }
#pragma unroll 1
    for (int e = tid; e < n_os * (kD / 4); e += kThreads) {
      const int n = e / (kD / 4), cc = e - n * (kD / 4);
      const size_t grow = grow0 + sfx_tok[n_oa + n];
      cp_async16(su32(ocache + n * kD + 4 * cc), prm.o_p + grow * kD + 4 * cc, 16u);
    }
#pragma unroll 1
    for (int n = tid; n < n_os; n += kThreads)
      cp_async4(su32(lcache + n), prm.l_p + grow0 + sfx_tok[n_oa + n]);
    cp_async_commit();
  }
  __syncthreads();

  LOSA_PHASE(3);
  // ---- the bound's A operand stays in registers for the whole scan (one
  // m16 tile of active rows per warp)
  const int ntm = R16 / 16;
  const int wpm = ntm > 0 ? kWarps / ntm : 1;  // warps per m16 tile (ntm <= 8)
  const int mt = warp / wpm, sub = warp % wpm;
  const bool sw = sel && mt < ntm;
  uint32_t a[16][4];
  if (DT == LOSA_BF16 && sw) {
    // m16n8k16 A fragments of [q- | q+] (K = 256): ldmatrix of the active
    // rows' q_cur (8 channel steps of 16), then a[kc] = the negative part
    // and a[kc + 8] = the non-negative part (sign bit tests, exact; -0 goes
    // to q-).  a[.][0] and a[.][2] hold row g4, a[.][1] and a[.][3] row g4 + 8.
    const int mi = lane >> 3, trow = mt * 16 + (mi & 1) * 8 + (lane & 7);
    const char* qsrc = qcs + act_row[trow < R ? trow : 0] * qst + (mi >> 1) * 16;
    const bool okA = mt * 16 + g4 < R, okB = mt * 16 + g4 + 8 < R;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t w[4];
      ldsm_x4(su32(qsrc + kc * 32), w[0], w[1], w[2], w[3]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool okr = (j & 1) ? okB : okA;
        const uint32_t x = okr ? w[j] : 0u;
        const uint32_t neg = ((x >> 15) & 0x00010001u) * 0xffffu;
        a[kc][j] = x & neg;
        a[kc + 8][j] = x & ~neg;
      }
    }
  }

  for (int r = tid; r < R; r += kThreads) {
    l_n[r] = 0;
    l_thr[r] = 0ull;
    if (DT == LOSA_BF16 && sel) emx[r] = 0u;
  }
  __syncthreads();  // the query area becomes the buffer area
  LOSA_PHASE(4);

  // ---- bound scores of this CTA's pages, stage by stage, stored per row
  // for a chunk of spc pages (scores[r][p - chunk start]).  Each warp goes
  // through the stages at its own pace: it waits for a stage's bytes, scores
  // its tiles and releases the slot; thread 0 refills a slot once all warps
  // have released it.  After a chunk's last stage (a barrier) each active
  // row's candidates take in the chunk's pages (one warp per row).
  const int rA = mt * 16 + g4, rB = rA + 8;
  const int spc = prm.spc;
  // bf16: each scoring thread keeps, for its two rows, the maxima of the
  // lower-key value words of its pages in two groups (n-tile parity) and the
  // largest half-width; they go to gmx [R16][ng] and emx [R16] before each
  // chunk's selection
  const int ng = 8 * wpm;
  uint32_t gA0 = 0u, gA1 = 0u, gB0 = 0u, gB1 = 0u;
  float eA = 0.f, eB = 0.f;
  const float2 qnA = DT == LOSA_BF16 && sw && rA < R ? qn[rA] : make_float2(0.f, 0.f);
  const float2 qnB = DT == LOSA_BF16 && sw && rB < R ? qn[rB] : make_float2(0.f, 0.f);
#pragma unroll 1
  for (int t = 0; t < nstg; ++t) {
    const int st = t % prm.stages;
    const uint32_t parity = (t / prm.stages) & 1;
    const char* stage = ring + st * kStageBytes;
    const int nps = min(prm.tile, npg - t * prm.tile);
    const int pl0 = t * prm.tile;  // the stage's first page (CTA-local)
    // the producer (thread 0) refills the slot of the stage before this one
    // once every warp has released it
    if (tid == 0 && t >= 1 && t - 1 + prm.stages < nstg && scal[kSFail] == 0) {
      if (mbar_wait(&ebar[(t - 1) % prm.stages], ((t - 1) / prm.stages) & 1)) {
        issue_stage(t - 1 + prm.stages);
        if (t - 1 + prm.stages < 8) LOSA_PHASE(32 + t - 1 + prm.stages);
      }
      else
        scal[kSFail] = 1;
    }
    // each thread waits for the stage itself (the wait makes the bytes the
    // copy wrote visible to it)
    if (scal[kSFail] == 0 && mbar_wait(&mbar[st], parity)) {
      if (t < 8) LOSA_PHASE(24 + t);
      if (t == 0) LOSA_PHASE(5);
      if (t == nstg - 1) LOSA_PHASE(6);
      if (DT == LOSA_BF16) {
        const int nnt = (nps + 7) / 8;
#pragma unroll 1
        for (int nt = sub; sw && nt < nnt; nt += wpm) {
          float u[4];
          bound_ntile(a, stage + nt * 8 * 512, u);
          const int pl = pl0 + nt * 8 + 2 * t4;  // this lane's pages pl, pl + 1 (pl even)
          if (pl < npg) {  // (pl + 1 stays inside the chunk's row: spc is even)
            const int ps = pl % spc;
            if (rA < R) *reinterpret_cast<float2*>(scores + rA * spc + ps) = make_float2(u[0], u[1]);
            if (rB < R) *reinterpret_cast<float2*>(scores + rB * spc + ps) = make_float2(u[2], u[3]);
            const float4 nk = *reinterpret_cast<const float4*>(pnorm + pl);
            const bool v1 = pl + 1 < npg;
            const float e0 = __fadd_ru(__fmul_ru(qnA.x, nk.x), __fmul_ru(qnA.y, nk.y));
            const float e1 = v1 ? __fadd_ru(__fmul_ru(qnA.x, nk.z), __fmul_ru(qnA.y, nk.w)) : 0.f;
            const float e2 = __fadd_ru(__fmul_ru(qnB.x, nk.x), __fmul_ru(qnB.y, nk.y));
            const float e3 = v1 ? __fadd_ru(__fmul_ru(qnB.x, nk.z), __fmul_ru(qnB.y, nk.w)) : 0.f;
            const uint32_t lA = max(ordered_bits(__fsub_rd(u[0], e0)),
                                    v1 ? ordered_bits(__fsub_rd(u[1], e1)) : 0u);
            const uint32_t lB = max(ordered_bits(__fsub_rd(u[2], e2)),
                                    v1 ? ordered_bits(__fsub_rd(u[3], e3)) : 0u);
            if (nt & 1) {
              gA1 = max(gA1, lA);
              gB1 = max(gB1, lB);
            } else {
              gA0 = max(gA0, lA);
              gB0 = max(gB0, lB);
            }
            eA = fmaxf(eA, fmaxf(e0, e1));
            eB = fmaxf(eB, fmaxf(e2, e3));
          }
        }
      } else {
        // fp32: exact scores on CUDA cores (the oracle's arithmetic)
#pragma unroll 1
        for (int e = tid; e < nps * R; e += kThreads) {
          const int pl = e % nps, r = e / nps;
          const int pg = pr0 + pl0 + pl;
          const char* recp = stage + pl * prm.rec;
          const float* q = reinterpret_cast<const float*>(qa + r * rowb);
          float acc = 0.f;
#pragma unroll 1
          for (int cc = 0; cc < kD / 4; ++cc) {
            const float4 mn = *reinterpret_cast<const float4*>(recp + meta_swz(16u * cc, pg));
            const float4 mx =
                *reinterpret_cast<const float4*>(recp + meta_swz(16u * (cc + kD / 4), pg));
            const float mns[4] = {mn.x, mn.y, mn.z, mn.w}, mxs[4] = {mx.x, mx.y, mx.z, mx.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float qi = q[4 * cc + u];
              acc = __fadd_rn(acc, fmaxf(__fmul_rn(qi, mxs[u]), __fmul_rn(qi, mns[u])));
            }
          }
          scores[r * spc + (pl0 + pl) % spc] = acc;
        }
      }
    } else {
      scal[kSFail] = 1;
    }
    // the warp has read the stage: release its slot
    __syncwarp();
    if (lane == 0) mbar_arrive(&ebar[st]);
    if (t < 8) LOSA_PHASE_BY(40 + t, 4 * 32);  // (warp 4: warp 0's scheduler partner)
    const bool chunk_end = ((t + 1) * prm.tile) % spc == 0 || t == nstg - 1;
    if (DT == LOSA_BF16 && chunk_end && sw) {
      const int slot = ((sub * 4) + t4) * 2;
      if (rA < R) {
        gmx[rA * ng + slot] = gA0;
        gmx[rA * ng + slot + 1] = gA1;
        atomicMax(emx + rA, __float_as_uint(eA));
      }
      if (rB < R) {
        gmx[rB * ng + slot] = gB0;
        gmx[rB * ng + slot + 1] = gB1;
        atomicMax(emx + rB, __float_as_uint(eB));
      }
    }
    if (chunk_end) {
      __syncthreads();  // every warp's scores and maxima of the chunk are in
      const int cb = t * prm.tile / spc * spc;  // the chunk's first page
      const int cn = min(npg, cb + spc) - cb;
      if (t == nstg - 1) LOSA_PHASE(7);
      if (sel && scal[kSFail] == 0) {
        // rows r0 and r0 + 8 per warp: their survivors, rescored together,
        // then each row's exact top k
#pragma unroll 1
        for (int r0 = warp; r0 < R; r0 += 2 * kWarps) {
          const int r1 = r0 + kWarps;
          if (DT == LOSA_BF16) {
            auto row = [&](int r, int h) {
              return PairRow{scores + r * spc,
                             w_lk + h * prm.lb,
                             l_lk + static_cast<size_t>(r) * prm.lcap,
                             l_n + r,
                             l_thr + r,
                             gmx + r * ng,
                             __uint_as_float(emx[r]),
                             qa + r * rowb,
                             r};
            };
            const bool hasB = r1 < R;
            // (the last chunk: the pages of the ring's last stages are still there)
            const RingView rv{ring, t == nstg - 1 ? max(0, nstg - prm.stages) * prm.tile : INT_MAX,
                              pr0, prm.tile, prm.stages};
            select_pair_bf16(row(r0, 0), row(hasB ? r1 : r0, 1), hasB, cn, pr0 + cb, k, prm.lb,
                             ng, meta_g, rv);
          } else {
            auto survivors = [&](int r, int h) {
              return row_survivors<DT>(scores + r * spc, pnorm + cb, make_float2(0.f, 0.f), cn,
                                       pr0 + cb, k, prm.lb, w_lk + h * prm.lb, w_uk + h * prm.lb,
                                       l_lk + static_cast<size_t>(r) * prm.lcap, l_n[r], l_thr[r],
                                       qa + r * rowb, r, meta_g, nullptr, ng, 0.f);
            };
            const int nA = survivors(r0, 0);
            const int nB = r1 < R ? survivors(r1, 1) : 0;
            row_topk(w_lk, nA, k, l_lk + static_cast<size_t>(r0) * prm.lcap, l_n + r0,
                     l_thr + r0, l_thr[r0]);
            if (r1 < R)
              row_topk(w_lk + prm.lb, nB, k, l_lk + static_cast<size_t>(r1) * prm.lcap, l_n + r1,
                       l_thr + r1, l_thr[r1]);
          }
        }
      }
      __syncthreads();
    }
  }

  LOSA_PHASE(8);
  // ================= cluster barrier 1: every CTA's lists are final ========
  cluster_sync();
  const bool ok1 = scal[kSFail] == 0;
  LOSA_PHASE(9);

  // ---- each row's k pages from the lists of all CTAs of the cluster: CTA c
  // merges rows r = c (mod C), one warp per row
  const int nwords = (d.P + 31) / 32;
  if (sel) {
    if (ok1) {
      const MergeCtx MC = {l_lk, l_n, l_thr, prm.lcap, C};
      u64* buf = reinterpret_cast<u64*>(ring + warp * prm.mstride);
#pragma unroll 1
      for (int i = warp; warp < prm.nmw && c + C * i < R; i += prm.nmw)
        merge_row(MC, c + C * i, k, buf, sel_all + (c + C * i) * k);
    }
    __syncthreads();
    if (prm.page_idx) {
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int r = e / k, j = e - r * k;
        if (r % C != c) continue;
        const int hl = r / A, aa = r % A;
        prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + aa) * k + j] = sel_all[e];
      }
    }
  }

  LOSA_PHASE(10);
  // Which pages this CTA attends.  By default (own): the pages of the rows
  // it merged -- every active row is finished by one CTA, with no union
  // round and no cross-CTA combine; a page two of its rows share is read
  // once, a page rows of two CTAs share is read by both.  With the
  // whole-union variant, or when every page is selected: the CTA's share of
  // the group's union (slots u = c mod C), and the CTAs' partials are
  // combined through distributed shared memory.
  const bool own = sel && !d.attend_union;
  // (own pages, no union count asked for: this CTA reads no other CTA's
  // shared memory from here on, so it arrives at the last cluster barrier
  // now and only waits there at the end.  The arrival is relaxed: the only
  // thing it has to follow is the merge's loads from the other CTAs, and
  // their values are already in this CTA's selections -- a release would
  // also wait for the page_idx stores to become visible, for nothing)
  const bool early_exit_arrival = own && !prm.union_count;
  if (!own) {
    // ================= cluster barrier 1b: every row's selection is final ====
    cluster_sync();
  } else if (early_exit_arrival) {
    cluster_arrive_relaxed();
  }

  // ---- the page bitmap: this CTA's rows' selections (own), or every row's,
  // read from their CTAs
  if (sel) {
    if (!own) {
#pragma unroll 1
      for (int w = tid; w < nwords; w += kThreads) bitmap[w] = 0u;
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int r = e / k;
        if (r % C != c) sel_all[e] = ld_dsmem_s32(dsmem(sel_all + e, r % C));
      }
      __syncthreads();
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int p = sel_all[e];
        if (p >= 0 && p < d.P) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
        else if (p >= 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
      }
    }
  } else if (R > 0 && prm.page_idx) {
    // every page of the sequence, then -1
#pragma unroll 1
    for (int e = tid; e < R * k; e += kThreads) {
      const int r = e / k, j = e - r * k;
      if (r % C != c) continue;
      const int hl = r / A, aa = r % A;
      prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + aa) * k + j] =
          j < Ps ? j : -1;
    }
  }
  const int MW = (R + 31) / 32;
#pragma unroll 1
  for (int e = tid; e < prm.max_lp * MW; e += kThreads) masks[e] = 0u;
  __syncthreads();

  // ---- the slots: own, every page of the bitmap (u = slot); else the
  // group's union and this CTA's share (union slots u = c mod C)
  const int Cs = own ? 1 : C, cs = own ? 0 : c;
  if (R == 0 && c == 0 && tid == 0 && prm.union_count) prm.union_count[sg] = 0;
  if (R > 0) {
    if (!sel) {
      const int U = Ps;
      const int nlp = U > c ? (U - c + C - 1) / C : 0;
      if (tid == 0) {
        scal[kSNlp] = min(nlp, prm.max_lp);
        if (c == 0 && prm.union_count) prm.union_count[sg] = U;
      }
#pragma unroll 1
      for (int j = tid; j < min(nlp, prm.max_lp); j += kThreads) lpages[j] = c + j * C;
#pragma unroll 1
      for (int e = tid; e < min(nlp, prm.max_lp) * MW; e += kThreads) {
        const int nb = min(32, R - 32 * (e % MW));
        masks[e] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
      }
    } else if (own) {
      // the CTA's rows' pages, once each (warp 0): entry e is position
      // e % k of its j = e / k -th row (r = c + C j); an entry takes the slot
      // of its page if an earlier chunk made one, else the lowest lane with
      // the same page makes a new slot; every entry sets its row's bit in
      // its slot's mask
      if (warp == 0) {
        const int ne = n_oa * k;
        int nu = 0;
#pragma unroll 1
        for (int e0 = 0; e0 < ne; e0 += 32) {
          const int e = e0 + lane;
          const int r = c + C * (e / k);
          int p = e < ne ? sel_all[r * k + e % k] : -1;
          if (p >= d.P) {
            atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
            p = -1;
          }
          int slot = -1;
          if (p >= 0)
            for (int u = 0; u < nu && slot < 0; ++u) slot = lpages[u] == p ? u : -1;
          const bool fresh = p >= 0 && slot < 0;
          const unsigned same = __match_any_sync(0xffffffffu, fresh ? p : -1);
          const int leader = __ffs(same) - 1;
          const bool lead = fresh && leader == lane;
          const unsigned bal = __ballot_sync(0xffffffffu, lead);
          const int mine = nu + __popc(bal & lt);
          const int from_leader = __shfl_sync(0xffffffffu, mine, leader);
          if (fresh) slot = from_leader;
          if (lead && slot < prm.max_lp) lpages[slot] = p;
          if (p >= 0 && slot < prm.max_lp) atomicOr(&masks[slot * MW + (r >> 5)], 1u << (r & 31));
          nu += __popc(bal);
          __syncwarp();
        }
        if (lane == 0) {
          scal[kSNlp] = min(nu, prm.max_lp);
          if (nu > prm.max_lp) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
        }
      }
    } else {
      // exclusive prefix of the words' popcounts: a run of words per thread,
      // a warp scan, then the warps' totals
      const int per = (nwords + kThreads - 1) / kThreads;
      const int w0 = tid * per, w1 = min(nwords, w0 + per);
      int sum = 0;
#pragma unroll 1
      for (int w = w0; w < w1; ++w) sum += __popc(bitmap[w]);
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane == 31) scal[kSWsum + warp] = incl;
      __syncthreads();
      int off = 0, U = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int cnt = scal[kSWsum + w];
        off += w < warp ? cnt : 0;
        U += cnt;
      }
      int run = off + incl - sum;
#pragma unroll 1
      for (int w = w0; w < w1; ++w) {
        wbase[w] = run;
        run += __popc(bitmap[w]);
      }
      const int nlp = U > cs ? (U - cs + Cs - 1) / Cs : 0;
      if (tid == 0) {
        scal[kSNlp] = min(nlp, prm.max_lp);
        if (nlp > prm.max_lp) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
        if (!own && c == 0 && prm.union_count) prm.union_count[sg] = U;
      }
      __syncthreads();
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int r = e / k;
        if (own && r % C != c) continue;
        const int p = sel_all[e];
        if (p < 0 || p >= d.P) continue;
        const int w = p >> 5;
        const int u = wbase[w] + __popc(bitmap[w] & ((1u << (p & 31)) - 1u));
        if (u % Cs != cs || u / Cs >= prm.max_lp) continue;
        lpages[u / Cs] = p;
        atomicOr(&masks[(u / Cs) * MW + (r >> 5)], 1u << (r & 31));
      }
      __syncthreads();
      if (d.attend_union) {
        // every active row attends to the group's whole union
#pragma unroll 1
        for (int e = tid; e < scal[kSNlp] * MW; e += kThreads) {
          const int nb = min(32, R - 32 * (e % MW));
          masks[e] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
        }
      }
    }
    // drift-safe locality: this CTA's active rows' reference := q_cur (every
    // CTA of the cluster has read the reference before barrier 1)
    if (prm.qref) {
      const char* qg = static_cast<const char*>(prm.qc) + grow0 * rowb;
      char* qr = static_cast<char*>(prm.qref) + grow0 * rowb;
#pragma unroll 1
      for (int e = tid; e < n_oa * cpr; e += kThreads) {
        const int j = e / cpr, cc = e - j * cpr;
        const size_t o = static_cast<size_t>(sfx_tok[j]) * rowb + cc * 16;
        *reinterpret_cast<uint4*>(qr + o) = *reinterpret_cast<const uint4*>(qg + o);
      }
    }
  }
  __syncthreads();

  LOSA_PHASE(11);
  // ---- gather: the union pages of this CTA (TMA, no multicast), each
  // folded into the active rows whose mask has it
  const int nlp = R > 0 ? scal[kSNlp] : 0;
  const bool ok2 = scal[kSFail] == 0;
  const float sl2 = d.scale_log2;
  // two page buffers of ngp pages: batch b lands in buffer b & 1 while the
  // previous batch is folded in
  const int nbat = (nlp + prm.ngp - 1) / prm.ngp;
  // (warp 0 issues a batch: lane i the pages i, i + 32, ...)
  auto issue = [&](int bt) {
    const int b0 = bt * prm.ngp, nb = min(prm.ngp, nlp - b0);
    char* bufp = ring + (bt & 1) * prm.ngp * 2 * pbytes;
    if (DT == LOSA_BF16) {
      if (lane == 0) mbar_expect_tx(&gbar[bt & 1], static_cast<uint32_t>(nb * 2 * pbytes));
      __syncwarp();
#pragma unroll 1
      for (int i = lane; i < nb; i += 32) {
        const int p = lpages[b0 + i];
        const int row = sg * d.Lc + p * kPS;
        char* dk = bufp + 2 * i * pbytes;
        if (prm.page3d) {
          tma_load_3d(dk, &kmap, 0, row, 0, &gbar[bt & 1]);
          tma_load_3d(dk + pbytes, &vmap, 0, row, 0, &gbar[bt & 1]);
        } else {
          tma_load_2d(dk, &kmap, 0, row, &gbar[bt & 1]);
          tma_load_2d(dk + 2048, &kmap, 64, row, &gbar[bt & 1]);
          tma_load_2d(dk + pbytes, &vmap, 0, row, &gbar[bt & 1]);
          tma_load_2d(dk + pbytes + 2048, &vmap, 64, row, &gbar[bt & 1]);
        }
      }
    } else if (lane == 0) {
      uint32_t bytes = 0;
      for (int i = 0; i < nb; ++i) bytes += 2u * min(kPS, Ls - lpages[b0 + i] * kPS) * rowb;
      mbar_expect_tx(&gbar[bt & 1], bytes);
#pragma unroll 1
      for (int i = 0; i < nb; ++i) {
        const int p = lpages[b0 + i];
        const uint32_t nbytes = static_cast<uint32_t>(min(kPS, Ls - p * kPS) * rowb);
        const size_t off = (static_cast<size_t>(sg) * d.Lc + static_cast<size_t>(p) * kPS) * rowb;
        bulk_g2s(bufp + 2 * i * pbytes, static_cast<const char*>(prm.K) + off, nbytes,
                 &gbar[bt & 1]);
        bulk_g2s(bufp + (2 * i + 1) * pbytes, static_cast<const char*>(prm.V) + off, nbytes,
                 &gbar[bt & 1]);
      }
    }
  };
  if (warp == 0 && ok2) {
    if (nbat > 0) issue(0);
    if (nbat > 1) issue(1);
  }
  LOSA_PHASE(12);

  // ---- while the pages land: the block's K/V and the cached state are in
  // (cp.async groups 1 and 2)
  cp_async_wait<0>();
  __syncthreads();
  // ---- dense suffix of this CTA's rows over the block's own keys: stable
  // rows merge with their untouched cache and are finished; active rows keep
  // (o_s, L_s) for the combine
  if (qok) {
    if (DT == LOSA_BF16) {
      const int nmt = (ns + 15) / 16;
#pragma unroll 1
      for (int m2 = warp; m2 < nmt; m2 += kWarps) {
        TileAcc t;
        tile_init(t);
#pragma unroll 1
        for (int j0 = 0; j0 < B; j0 += kPS)
          tile_attend<false>(t, sq + m2 * 16 * 256, kbv + j0 * 256, kbv + (bpad + j0) * 256,
                             0xffffu, min(kPS, B - j0), d.scale_log2);
        tile_finish(t);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = m2 * 16 + g4 + 8 * h;
          if (n >= ns) continue;
          const float inv = __frcp_rn(t.l[h]);
          const float Lsx = (t.m[h] + __log2f(t.l[h])) * kLn2;
          if (n < n_oa) {
            if (t4 == 0) sfx_l[n] = Lsx;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc)
              *reinterpret_cast<float2*>(sfx_o + n * kD + cc * 8 + 2 * t4) =
                  make_float2(t.o[cc][2 * h] * inv, t.o[cc][2 * h + 1] * inv);
          } else {
            const int m = n - n_oa;
            const size_t grow = grow0 + sfx_tok[n];
            float wa, wb, L;
            lse_weights(lcache[m], Lsx, wa, wb, L);
            const float* op = ocache + m * kD;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) {
              const int ch = cc * 8 + 2 * t4;
              const float2 o = *reinterpret_cast<const float2*>(op + ch);
              *reinterpret_cast<float2*>(prm.out + grow * kD + ch) =
                  make_float2(wa * o.x + wb * (t.o[cc][2 * h] * inv),
                              wa * o.y + wb * (t.o[cc][2 * h + 1] * inv));
            }
            if (prm.out_lse && t4 == 0) prm.out_lse[grow] = L;
          }
        }
      }
    } else {
      float* Ps = fscr + warp * 16;
#pragma unroll 1
      for (int n = warp; n < ns; n += kWarps) {
        const float4 q = row4<DT>(sq, n, lane);
        float m = -INFINITY, l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int j0 = 0; j0 < B; j0 += kPS)
          attend_page<DT>(q, kbv + j0 * rowb, kbv + (bpad + j0) * rowb, min(kPS, B - j0),
                          d.scale_log2, m, l, acc, Ps);
        const float inv = __frcp_rn(l);
        const float4 os = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        const float Lsx = (m + __log2f(l)) * kLn2;
        if (n < n_oa) {
          if (lane == 0) sfx_l[n] = Lsx;
          *reinterpret_cast<float4*>(sfx_o + n * kD + 4 * lane) = os;
        } else {
          const int mm = n - n_oa;
          const size_t grow = grow0 + sfx_tok[n];
          float wa, wb, L;
          lse_weights(lcache[mm], Lsx, wa, wb, L);
          const float4 op = *reinterpret_cast<const float4*>(ocache + mm * kD + 4 * lane);
          *reinterpret_cast<float4*>(prm.out + grow * kD + 4 * lane) =
              make_float4(wa * op.x + wb * os.x, wa * op.y + wb * os.y, wa * op.z + wb * os.z,
                          wa * op.w + wb * os.w);
          if (prm.out_lse && lane == 0) prm.out_lse[grow] = L;
        }
      }
    }
  }
  __syncthreads();

  LOSA_PHASE(13);
  if (DT == LOSA_BF16) {
    const int wpg = ntm > 0 ? kWarps / ntm : 1;
    const int mtg = warp / wpg, subg = warp % wpg;
    const bool aw = ntm > 0 && mtg < ntm;
    TileAcc t;
    tile_init(t);
#pragma unroll 1
    for (int bt = 0; bt < nbat; ++bt) {
      const int b0 = bt * prm.ngp, nb = min(prm.ngp, nlp - b0);
      char* bufp = ring + (bt & 1) * prm.ngp * 2 * pbytes;
      if (ok2 && scal[kSFail] == 0 && !mbar_wait(&gbar[bt & 1], (bt >> 1) & 1)) scal[kSFail] = 1;
      if (bt == 0) LOSA_PHASE(14);
      // V rows past the sequence's end of its partial last page may hold
      // anything (P is 0 there, but 0 times NaN is NaN): zero them
      if (Ls % kPS) {
#pragma unroll 1
        for (int i = 0; i < nb; ++i) {
          const int p = lpages[b0 + i];
          if (p != Ps - 1) continue;
          const int ntok = Ls - p * kPS;
          char* dv = bufp + (2 * i + 1) * pbytes;
          for (int e = tid; e < 2 * (kPS - ntok) * 8; e += kThreads) {
            const int h = e / ((kPS - ntok) * 8), rem = e % ((kPS - ntok) * 8);
            *reinterpret_cast<uint4*>(dv + h * 2048 + ntok * 128 + rem * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      __syncthreads();
      if (scal[kSFail] == 0) {
#pragma unroll 1
        for (int i = subg; aw && i < nb; i += wpg) {
          const uint32_t bits = (masks[(b0 + i) * MW + (mtg >> 1)] >> ((mtg & 1) * 16)) & 0xffffu;
          if (!bits) continue;
          const int p = lpages[b0 + i];
          tile_attend<true>(t, qa + mtg * 16 * 256, bufp + 2 * i * pbytes,
                            bufp + (2 * i + 1) * pbytes, bits, min(kPS, Ls - p * kPS), sl2);
        }
      }
      __syncthreads();  // the buffer is free: the batch after next may land in it
      if (warp == 0 && ok2 && scal[kSFail] == 0 && bt + 2 < nbat) issue(bt + 2);
    }
    tile_finish(t);
    if (R > 0 && wpg == 1) {
      // one warp per m16 tile: its state is the CTA's partial of those rows
      if (aw) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = mtg * 16 + g4 + 8 * h;
          if (t4 == 0) {
            part_ml[2 * row] = t.m[h];
            part_ml[2 * row + 1] = t.l[h];
          }
#pragma unroll
          for (int cc = 0; cc < 16; ++cc)
            *reinterpret_cast<float2*>(part_o + row * kD + cc * 8 + 2 * t4) =
                make_float2(t.o[cc][2 * h], t.o[cc][2 * h + 1]);
        }
      }
    } else if (R > 0) {
      // several warps per m16 tile: their partials (ring, ahead of part_o)
      // merge into one partial per row
      // [warp][16][4 + kD]: m, l, 2 pad, o (16-byte aligned rows and o)
      float* wp = reinterpret_cast<float*>(ring);
      constexpr int ws = 4 + kD;
      if (aw) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float* pr = wp + (warp * 16 + g4 + 8 * h) * ws;
          if (t4 == 0) {
            pr[0] = t.m[h];
            pr[1] = t.l[h];
          }
#pragma unroll
          for (int cc = 0; cc < 16; ++cc)
            *reinterpret_cast<float2*>(pr + 4 + cc * 8 + 2 * t4) =
                make_float2(t.o[cc][2 * h], t.o[cc][2 * h + 1]);
        }
      }
      __syncthreads();
      // (own pages: only the rows this CTA finishes, r = c + C j)
      const int nmr = own ? n_oa : R;
#pragma unroll 1
      for (int jr = warp; jr < nmr; jr += kWarps) {
        const int r = own ? c + C * jr : jr;
        const int m16 = r >> 4, i = r & 15;
        float M = -INFINITY;
        for (int w = 0; w < wpg; ++w) M = fmaxf(M, wp[((m16 * wpg + w) * 16 + i) * ws]);
        float l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (M != -INFINITY) {
          for (int w = 0; w < wpg; ++w) {
            const float* pr = wp + ((m16 * wpg + w) * 16 + i) * ws;
            if (pr[0] == -INFINITY) continue;
            const float wgt = exp2f(pr[0] - M);
            l += wgt * pr[1];
            const float4 o4 = *reinterpret_cast<const float4*>(pr + 4 + 4 * lane);
            acc.x += wgt * o4.x;
            acc.y += wgt * o4.y;
            acc.z += wgt * o4.z;
            acc.w += wgt * o4.w;
          }
        }
        *reinterpret_cast<float4*>(part_o + r * kD + 4 * lane) = acc;
        if (lane == 0) {
          part_ml[2 * r] = M;
          part_ml[2 * r + 1] = l;
        }
      }
    }
  } else {
    // fp32: one warp per active row on CUDA cores; the running state lives in
    // part_o / part_ml
#pragma unroll 1
    for (int e = tid; e < R * kD; e += kThreads) part_o[e] = 0.f;
#pragma unroll 1
    for (int r = tid; r < R; r += kThreads) {
      part_ml[2 * r] = -INFINITY;
      part_ml[2 * r + 1] = 0.f;
    }
    float* Ps = fscr + warp * 16;
    __syncthreads();
#pragma unroll 1
    for (int bt = 0; bt < nbat; ++bt) {
      const int b0 = bt * prm.ngp, nb = min(prm.ngp, nlp - b0);
      char* bufp = ring + (bt & 1) * prm.ngp * 2 * pbytes;
      if (ok2 && scal[kSFail] == 0 && !mbar_wait(&gbar[bt & 1], (bt >> 1) & 1)) scal[kSFail] = 1;
      __syncthreads();
      if (scal[kSFail] == 0) {
#pragma unroll 1
        for (int r = warp; r < R; r += kWarps) {
          bool have = false;
#pragma unroll 1
          for (int i = 0; i < nb; ++i) have |= (masks[(b0 + i) * MW + (r >> 5)] >> (r & 31)) & 1u;
          if (!have) continue;
          const float4 q = row4<DT>(qa, r, lane);
          float m = part_ml[2 * r], l = part_ml[2 * r + 1];
          float4 acc = *reinterpret_cast<const float4*>(part_o + r * kD + 4 * lane);
#pragma unroll 1
          for (int i = 0; i < nb; ++i) {
            if (!((masks[(b0 + i) * MW + (r >> 5)] >> (r & 31)) & 1u)) continue;
            const int p = lpages[b0 + i];
            attend_page<DT>(q, bufp + 2 * i * pbytes, bufp + (2 * i + 1) * pbytes,
                            min(kPS, Ls - p * kPS), sl2, m, l, acc, Ps);
          }
          __syncwarp();
          if (lane == 0) {
            part_ml[2 * r] = m;
            part_ml[2 * r + 1] = l;
          }
          *reinterpret_cast<float4*>(part_o + r * kD + 4 * lane) = acc;
        }
      }
      __syncthreads();
      if (warp == 0 && ok2 && scal[kSFail] == 0 && bt + 2 < nbat) issue(bt + 2);
    }
  }

  LOSA_PHASE(15);
  // ================= cluster barrier 2: every CTA's partials are final =====
  // (own pages: each CTA's partial of its rows is the whole prefix result)
  if (!own) cluster_sync();
  __syncthreads();

  LOSA_PHASE(16);
  // ---- combine: CTA c finishes its active rows r = c + C*j
  if (scal[kSFail] == 0) {
#pragma unroll 1
    for (int j = warp; j < n_oa; j += kWarps) {
      const int r = c + C * j;
      float2 mlj = make_float2(-INFINITY, 0.f);
      if (own) {
        if (lane == 0) mlj = *reinterpret_cast<const float2*>(part_ml + 2 * r);
      } else if (lane < C) {
        mlj = ld_dsmem_f2(dsmem(part_ml + 2 * r, lane));
      }
      const uint32_t nz = __ballot_sync(0xffffffffu, mlj.x != -INFINITY);
      float4 ac[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if ((nz >> q) & 1u)
          ac[q] = own ? *reinterpret_cast<const float4*>(part_o + r * kD + 4 * lane)
                      : ld_dsmem_f4(dsmem(part_o + r * kD + 4 * lane, q));
      float M = mlj.x;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float wj = mlj.x == -INFINITY ? 0.f : exp2f(mlj.x - M);
      float lsum = wj * mlj.y;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float w = __shfl_sync(0xffffffffu, wj, q);
        if ((nz >> q) & 1u) {
          acc.x += w * ac[q].x;
          acc.y += w * ac[q].y;
          acc.z += w * ac[q].z;
          acc.w += w * ac[q].w;
        }
      }
      const float inv = __frcp_rn(lsum);
      const float4 op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      const float Lp = (M + __log2f(lsum)) * kLn2;
      const size_t grow = grow0 + act_row[r];
      *reinterpret_cast<float4*>(prm.o_p + grow * kD + 4 * lane) = op;
      if (lane == 0) prm.l_p[grow] = Lp;
      float wa, wb, L;
      lse_weights(Lp, sfx_l[j], wa, wb, L);
      const float4 os = *reinterpret_cast<const float4*>(sfx_o + j * kD + 4 * lane);
      *reinterpret_cast<float4*>(prm.out + grow * kD + 4 * lane) =
          make_float4(wa * op.x + wb * os.x, wa * op.y + wb * os.y, wa * op.z + wb * os.z,
                      wa * op.w + wb * os.w);
      if (prm.out_lse && lane == 0) prm.out_lse[grow] = L;
    }
  }

  // own pages: the group's union size, if asked for, from every row's
  // selection once all merges are done
  if (own && prm.union_count) {
    cluster_sync();
    if (c == 0) {
#pragma unroll 1
      for (int w = tid; w < nwords; w += kThreads) bitmap[w] = 0u;
      __syncthreads();
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int r = e / k;
        const int p = r % C == c ? sel_all[e] : ld_dsmem_s32(dsmem(sel_all + e, r % C));
        if (p >= 0 && p < d.P) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
      }
      __syncthreads();
      int cnt = 0;
#pragma unroll 1
      for (int w = tid; w < nwords; w += kThreads) cnt += __popc(bitmap[w]);
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (lane == 0) scal[kSWsum + warp] = cnt;
      __syncthreads();
      if (tid == 0) {
        int U = 0;
        for (int w = 0; w < kWarps; ++w) U += scal[kSWsum + w];
        prm.union_count[sg] = U;
      }
    }
  }

  LOSA_PHASE(17);
  // ================= cluster barrier 3: no CTA leaves while another may
  // still read its shared memory
  if (early_exit_arrival) cluster_wait();
  else cluster_sync();
  if (tid == 0 && scal[kSFail]) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
  LOSA_PHASE(18);
}

// ---------------------------------------------------------------------------
// host side: cluster geometry, shared-memory plan, attributes, launch
// ---------------------------------------------------------------------------
int align_up(int x, int a) { return (x + a - 1) / a * a; }

struct Taker {
  long long off = 0;
  int operator()(long long bytes, int align) {
    off = (off + align - 1) / align * align;
    const long long o = off;
    off += bytes;
    return static_cast<int>(std::min<long long>(o, 1LL << 30));
  }
};

// clusters of 8 and of 16 CTAs that can be resident at once (1 CTA per SM)
struct ClusterRoom {
  int c8 = 0, c16 = 0;
};

bool plan_step(const Dims& d, StepParams* prm, int max_dyn, const ClusterRoom& room) {
  *prm = StepParams();
  prm->d = d;
  const bool bf = d.esz == 2;
  const int rowb = kD * d.esz;
  const int pbytes = kPS * rowb;
  const int GB = d.G * d.B;
  const int R = d.R, R16 = (R + 15) / 16 * 16;
  const bool sel = R > 0 && !d.all_pages;
  prm->rec = 2 * kD * d.esz;
  prm->tile = kStageBytes / prm->rec;  // 64 (bf16) or 32 (fp32) pages per ring stage
  // CTAs per cluster: a ring stage of pages each at least, more when many
  // active rows share the combine
  // (up to 16 when the CTAs attend their own rows' pages and the 16-CTA
  // clusters of the whole grid fit one wave)
  const long long NG = static_cast<long long>(d.S) * d.Hkv;
  const bool own = bf && sel && !d.attend_union;
  const int cmax = own && NG <= room.c16 ? kMaxClusterCtas : kMaxCombineCtas;
  int C = std::max((d.P + prm->tile - 1) / prm->tile, (R + 15) / 16);
  C = std::max(1, std::min(cmax, C));
  if (R == 0) C = 1;
  prm->C = C;
  prm->cp = align_up((d.P + C - 1) / C, 8);
  // candidate lists: entries per row left for the merge, and room for the
  // survivors of the first bound
  prm->lcap = d.k + kListSlack;
  // (the survivor buffer takes a row's list beside a chunk's exact top k)
  prm->lb = std::max(prm->lcap + 64, prm->lcap + d.k);
  if (sel && prm->lb > 256) return false;
  const int cp_t = align_up(prm->cp, prm->tile);
  const long long cap_all = static_cast<long long>(C) * prm->lcap;
  // merge warp scratch: the gathered keys
  prm->mstride = align_up(static_cast<int>(std::min<long long>(cap_all * 8, 1 << 30)), 16);
  prm->qstride = rowb + 16;  // rows 16 bytes apart in bank order
  // union pages per CTA
  const int Umax = d.all_pages ? d.P : std::min(d.P, R * d.k);
  prm->max_lp = R > 0 ? (Umax + C - 1) / C : 0;
  // (own pages: the pages of the CTA's ceil(R / C) rows)
  if (R > 0 && !d.all_pages)
    prm->max_lp = std::max(prm->max_lp, std::min(d.P, (R + C - 1) / C * d.k));
  const int n_oa = (R + C - 1) / C;
  const int n_os = (GB - R + C - 1) / C;
  const int ns = n_oa + n_os;
  const int nwords = (d.P + 31) / 32;
  const int MW = (R + 31) / 32;
  // one wave: every cluster resident at once (the next launch may then be
  // scheduled from the start)
  prm->early = NG <= (C > kMaxCombineCtas ? room.c16 : room.c8);

  // the largest plan that fits, with at least 4 ring stages when any plan
  // allows it: most pages per score chunk, then most union pages in flight,
  // then most ring stages
  for (int pass = 0; pass < 2; ++pass) {
  const int smin = pass == 0 ? std::min(4, kMaxStages) : kMinStages;
  for (int spc = cp_t; spc >= prm->tile; spc = (spc / 2 >= prm->tile ? align_up(spc / 2, prm->tile) : 0)) {
  prm->spc = spc;
  for (int ngp = std::min(kMaxGatherPages, std::max(1, prm->max_lp)); ngp >= 1; ngp /= 2) {
    for (int stages = kMaxStages; stages >= smin; --stages) {
      long long ring = 0;
      if (sel) ring = std::max(ring, static_cast<long long>(stages) * kStageBytes);
      if (sel) ring = std::max(ring, static_cast<long long>(prm->mstride));  // one merge warp
      if (R > 0) ring = std::max(ring, 4LL * ngp * pbytes);  // two buffers of ngp pages
      // bf16: the warps' partials (when several warps share an m16 tile),
      // then the CTA's partial per row
      const int ntm = R16 / 16;
      const long long wpart = (bf && ntm > 0 && kWarps / ntm > 1) ? 1LL * kWarps * 16 * (4 + kD) * 4 : 0;
      if (R > 0 && bf) ring = std::max(ring, wpart + R16 * (kD + 2) * 4LL);
      StepLayout& lo = prm->lo;
      Taker take;
      lo.ring = take(ring, 1024);
      // the queries; once they are staged, the lists, the scores and the
      // fp32 probability rows in the same bytes
      const long long qarea = 2LL * GB * prm->qstride;
      const long long larea = sel ? (1LL * prm->lcap * R + kWarps * 4LL * prm->lb) * 8 : 0;
      const long long carea = sel ? 4LL * R * prm->spc : 0;
      const long long sarea = bf ? 0LL : kWarps * 16LL * 4;
      const int qbase = take(std::max(qarea, larea + carea + sarea), 1024);
      lo.qc = qbase;
      lo.qp = qbase + GB * prm->qstride;
      lo.lists = qbase;
      lo.scores = qbase + static_cast<int>(larea);
      lo.sc = qbase + static_cast<int>(larea + carea);
      if (bf) {  // after the gather: the warps' partials, then the CTA's
        lo.part_o = lo.ring + static_cast<int>(wpart);
        lo.part_ml = lo.part_o + R16 * kD * 4;
      } else {
        lo.part_o = take(R > 0 ? 1LL * R * kD * 4 : 0, 128);
        lo.part_ml = take(R16 * 8LL, 16);
      }
      lo.qa = take(1LL * (bf ? R16 : R) * rowb, 128);
      lo.kbv = take(2LL * ((d.B + kPS - 1) / kPS * kPS) * rowb, 128);
      lo.sq = take(1LL * (bf ? (ns + 15) / 16 * 16 : ns) * rowb, 128);
      lo.ocache = take(4LL * n_os * kD, 16);
      lo.lcache = take(4LL * n_os, 16);
      lo.sfx_o = take(4LL * n_oa * kD, 16);
      lo.sfx_l = take(4LL * n_oa, 16);
      lo.l_n = take(4LL * R, 16);
      lo.l_thr = take(8LL * R, 16);
      lo.sel = take(sel ? 4LL * R * d.k : 0, 16);
      lo.bitmap = take(4LL * nwords, 16);
      lo.wbase = take(4LL * nwords, 16);
      lo.lpages = take(4LL * prm->max_lp, 16);
      lo.masks = take(4LL * prm->max_lp * MW, 16);
      lo.misc = take(4LL * kMiscInts, 16);
      lo.pnorm = take(bf && sel ? 8LL * prm->cp : 0, 128);
      const int ntm_ = std::max(1, R16 / 16);
      lo.gmx = take(bf && sel ? 4LL * R16 * 8 * std::max(1, kWarps / ntm_) : 0, 16);
      lo.emx = take(bf && sel ? 4LL * R16 : 0, 16);
      lo.qn = take(8LL * R16, 16);
      lo.mbar = take(8LL * (2 * kMaxStages + 2), 16);
      // + 1 KB: the kernel aligns its shared-memory base to 1024 bytes
      lo.total = static_cast<int>(std::min<long long>(take.off + 1024, 1LL << 30));
      if (take.off + 1024 > max_dyn) continue;
      prm->stages = sel ? stages : 0;
      prm->ngp = ngp;
      prm->nmw = sel ? static_cast<int>(std::min<long long>(kWarps, ring / prm->mstride)) : 0;
      if (sel && prm->nmw < 1) continue;
      return true;
    }
  }
  }
  }
  return false;
}

std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices] = {};
int g_attr_dyn[kMaxDevices] = {};
ClusterRoom g_attr_room[kMaxDevices];

template <int DT>
cudaError_t set_attrs(int optin, int* dyn) {
  const void* fn = reinterpret_cast<const void*>(losa_step_kernel<DT>);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  const int mine = optin - static_cast<int>(fa.sharedSizeBytes);
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, mine);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  *dyn = std::min(*dyn, mine);
  return cudaSuccess;
}

// clusters of `csize` step CTAs (the largest shared-memory plan) resident at
// once; 0 when the device cannot place one
int room_for(int csize, int dyn) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(csize, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(dyn);
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = csize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, losa_step_kernel<LOSA_BF16>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();  // (not sticky) a size the device cannot place
    return 0;
  }
  return n;
}

int ensure_attributes(int* max_dyn, ClusterRoom* room) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return LOSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (!g_attr_done[dev]) {
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    int dyn = optin;
    if ((e = set_attrs<LOSA_BF16>(optin, &dyn)) != cudaSuccess) return record_cuda_error(e);
    if ((e = set_attrs<LOSA_F32>(optin, &dyn)) != cudaSuccess) return record_cuda_error(e);
    g_attr_dyn[dev] = dyn;
    g_attr_room[dev].c8 = room_for(kMaxCombineCtas, dyn);
    g_attr_room[dev].c16 = room_for(kMaxClusterCtas, dyn);
    g_attr_done[dev] = true;
  }
  *max_dyn = g_attr_dyn[dev];
  if (room) *room = g_attr_room[dev];
  return LOSA_OK;
}

}  // namespace

bool fused_step_fits(const Dims& d, int max_dyn) {
  // (the 8-CTA plan; a 16-CTA plan of the same shape needs less per CTA)
  StepParams p;
  return plan_step(d, &p, max_dyn, ClusterRoom());
}

int launch_fused_step(const Dims& d, const void* q_cur, const void* q_prev, const void* k_prefix,
                      const void* v_prefix, const void* page_meta, const void* k_blk,
                      const void* v_blk, float* o_p, float* l_p, float* out, float* out_lse,
                      int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                      void* workspace, cudaStream_t st, void* q_ref_out) {
  int max_dyn = 0;
  ClusterRoom room;
  int rc = ensure_attributes(&max_dyn, &room);
  if (rc != LOSA_OK) return rc;
  StepParams prm;
  if (!plan_step(d, &prm, max_dyn, room) && !plan_step(d, &prm, max_dyn, ClusterRoom()))
    return LOSA_ERR_UNSUPPORTED;
  const long long NG = static_cast<long long>(d.S) * d.Hkv;
  if (NG > 65535) return LOSA_ERR_UNSUPPORTED;
  prm.qc = q_cur;
  prm.qp = q_prev;
  prm.meta = static_cast<const char*>(page_meta);
  prm.norms = reinterpret_cast<const float2*>(static_cast<const char*>(page_meta) +
                                              meta_norm_offset(d));
  prm.pn = meta_norm_stride(d);
  prm.K = k_prefix;
  prm.V = v_prefix;
  prm.kb = k_blk;
  prm.vb = v_blk;
  prm.o_p = o_p;
  prm.l_p = l_p;
  prm.out = out;
  prm.out_lse = out_lse;
  prm.active_idx = active_idx;
  prm.page_idx = page_idx;
  prm.union_count = union_count;
  prm.qref = q_ref_out;
  prm.status = reinterpret_cast<int*>(static_cast<char*>(workspace) + d.off_status);
  CUtensorMap kmap, vmap;
  std::memset(&kmap, 0, sizeof(kmap));
  std::memset(&vmap, 0, sizeof(vmap));
  if (d.dtype == LOSA_BF16 && d.R > 0) {
    // one 3-D copy per page when the driver takes the page map, else two
    // 2-D copies (one per 64-channel half)
    const unsigned long long rows = static_cast<unsigned long long>(NG) * d.Lc;
    prm.page3d = make_page_tmap(&kmap, k_prefix, rows) == LOSA_OK &&
                 make_page_tmap(&vmap, v_prefix, rows) == LOSA_OK;
    if (!prm.page3d && (make_tmap(&kmap, k_prefix, rows, kPS) != LOSA_OK ||
                        make_tmap(&vmap, v_prefix, rows, kPS) != LOSA_OK))
      return record_cuda_error(cudaErrorInvalidValue);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(prm.C, static_cast<unsigned>(NG), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(prm.lo.total);
  cfg.stream = st;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = prm.C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;  // overlaps the previous kernel's tail
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = d.dtype == LOSA_BF16
                            ? cudaLaunchKernelEx(&cfg, losa_step_kernel<LOSA_BF16>, prm, kmap, vmap)
                            : cudaLaunchKernelEx(&cfg, losa_step_kernel<LOSA_F32>, prm, kmap, vmap);
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}

}  // namespace losa

#ifdef LOSA_PHASE_TRACE
// (tracing build only) copy out / clear the phase timestamps
extern "C" int losa_phase_read(unsigned long long* host, int n) {
  if (!host || n < 0 || n > losa::kPhaseCtas * losa::kPhases) return LOSA_ERR_INVALID_ARG;
  return cudaMemcpyFromSymbol(host, losa::g_phase, sizeof(unsigned long long) * n) == cudaSuccess
             ? LOSA_OK
             : LOSA_ERR_CUDA;
}
extern "C" int losa_phase_clear(void) {
  static unsigned long long zero[losa::kPhaseCtas * losa::kPhases] = {};
  return cudaMemcpyToSymbol(losa::g_phase, zero, sizeof(zero)) == cudaSuccess ? LOSA_OK
                                                                            : LOSA_ERR_CUDA;
}
#endif
