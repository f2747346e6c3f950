// dense.cu -- cold-start dense prefix pass (first denoising step of a block).
//
// LoSA needs the full prefix attention of every block token once per block
// to seed the reuse cache (LoSA paper, limitations: the first denoising
// iteration of each block stays dense).  Flash-decode layout: the prefix of
// each (sequence, KV head) is split into page ranges; one CTA streams one
// range for all G*B query rows of the group and writes an unnormalised
// online-softmax partial per row; the finish kernel merges the partials, adds
// the dense suffix over the block's own keys and writes cache and output.
// bf16 runs on the 5th-generation tensor cores (tcgen05, TMEM), fp32 on
// CUDA cores.
#include <mutex>

#include "losa_common.cuh"
#include "ptx.cuh"
#include "umma.cuh"

namespace losa {
namespace {

constexpr int kDenseWarps = 8;
constexpr int kRowsPerWarp = 8;

// Copies `ntok` rows of one page (d floats each) into shared memory as fp32,
// zero-filling rows ntok..15.
__device__ __forceinline__ void load_page_f32(const void* src, size_t elem0, int ntok, int dtype,
                                              float* dst, int tid, int nthreads) {
  for (int e = tid; e < kPS * kD / 4; e += nthreads) {
    const int j = e / (kD / 4), c = (e % (kD / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (j < ntok) v = ld4(src, elem0 + static_cast<size_t>(j) * kD + c, dtype);
    *reinterpret_cast<float4*>(dst + j * kD + c) = v;
  }
}

__global__ void __launch_bounds__(kDenseWarps * 32)
    dense_partial_kernel(const void* __restrict__ Q, const void* __restrict__ K,
                         const void* __restrict__ V, float* __restrict__ part,
                         int* __restrict__ status, Dims d) {
  __shared__ __align__(16) float Ks[kPS * kD];
  __shared__ __align__(16) float Vs[kPS * kD];
  __shared__ float Ps[kDenseWarps][kPS];
  const int sg = blockIdx.y, split = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = d.G * d.B;
  const int L = seq_len(d, s);  // this sequence's prefix length
  const int p0 = split * d.split_pages;
  const int p1 = min((L + kPS - 1) / kPS, p0 + d.split_pages);  // none past its end
  const size_t kv0 = static_cast<size_t>(sg) * d.Lc * kD;
  if (split == 0 && threadIdx.x == 0 && seq_len_bad(d, s)) atomicCAS(status, 0, LOSA_ERR_DEVICE_BOUNDS);

  for (int rbase = 0; rbase < rows; rbase += kDenseWarps * kRowsPerWarp) {
    float4 q[kRowsPerWarp], acc[kRowsPerWarp];
    float m[kRowsPerWarp], l[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int r = rbase + warp * kRowsPerWarp + i;
      const int rr = r < rows ? r : 0;
      const int h = g * d.G + rr / d.B, t = rr % d.B;
      q[i] = ld4(Q, ((static_cast<size_t>(s) * d.Hq + h) * d.B + t) * kD + 4 * lane, d.dtype);
      acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      m[i] = -INFINITY;
      l[i] = 0.f;
    }
    for (int p = p0; p < p1; ++p) {
      const int ntok = min(kPS, L - p * kPS);
      __syncthreads();
      load_page_f32(K, kv0 + static_cast<size_t>(p) * kPS * kD, ntok, d.dtype, Ks, threadIdx.x,
                    blockDim.x);
      load_page_f32(V, kv0 + static_cast<size_t>(p) * kPS * kD, ntok, d.dtype, Vs, threadIdx.x,
                    blockDim.x);
      __syncthreads();
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i) {
        if (rbase + warp * kRowsPerWarp + i < rows)
          attend_page_row(q[i], Ks, Vs, ntok, d.scale_log2, m[i], l[i], acc[i], Ps[warp]);
      }
    }
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int r = rbase + warp * kRowsPerWarp + i;
      if (r >= rows) continue;
      float* dst = part + ((static_cast<size_t>(sg) * d.nsplit + split) * rows + r) * kPartStride;
      if (lane == 0) {
        dst[0] = m[i];
        dst[1] = l[i];
      }
      *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = acc[i];
    }
  }
}

// Dense attention of one query row over the block's own B keys (Kb/Vb in
// shared memory, B <= 32 rows, zero-filled to a multiple of 16); returns the
// normalised output channels of this lane and the natural log-normaliser.
__device__ __forceinline__ void suffix_row(float4 q, const float* Kb, const float* Vb, int B,
                                           float scale_log2, float* Ps, float4& o, float& L) {
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j0 = 0; j0 < B; j0 += kPS)
    attend_page_row(q, Kb + j0 * kD, Vb + j0 * kD, min(kPS, B - j0), scale_log2, m, l, acc, Ps);
  const float inv = 1.f / l;
  o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  L = (m + __log2f(l)) * kLn2;
}

constexpr int kFinishWarps = 4;   // rows (one per warp) per CTA of the dense finish
constexpr int kFinishBatch = 18;  // splits' partials in flight per row (one round at 18 splits)

__global__ void __launch_bounds__(kFinishWarps * 32)
    dense_finish_kernel(const void* __restrict__ Q, const void* __restrict__ Kb,
                        const void* __restrict__ Vb, const float* __restrict__ part,
                        float* __restrict__ o_p, float* __restrict__ l_p, float* __restrict__ out,
                        float* __restrict__ out_lse, Dims d) {
  extern __shared__ __align__(16) float fsm[];  // the block's K then V, [Bpad][d] each
  __shared__ float Ps[kFinishWarps][kPS];
  const int sh = blockIdx.x;  // s * Hq + h
  const int s = sh / d.Hq, h = sh % d.Hq, g = h / d.G;
  const int sg = s * d.Hkv + g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = d.G * d.B;
  const int Bpad = (d.B + kPS - 1) / kPS * kPS;
  float* Ksb = fsm;
  float* Vsb = fsm + Bpad * kD;
  for (int e = threadIdx.x; e < Bpad * kD / 4; e += blockDim.x) {
    const int j = e / (kD / 4), c = (e % (kD / 4)) * 4;
    float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
    if (j < d.B) {
      const size_t idx = (static_cast<size_t>(sg) * d.B + j) * kD + c;
      kv = ld4(Kb, idx, d.dtype);
      vv = ld4(Vb, idx, d.dtype);
    }
    *reinterpret_cast<float4*>(Ksb + j * kD + c) = kv;
    *reinterpret_cast<float4*>(Vsb + j * kD + c) = vv;
  }
  __syncthreads();
  // launched behind the split kernel (programmatic dependent launch): its
  // partials are read only after it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // one warp per row: rows blockIdx.y * kFinishWarps + warp of head h
  for (int t = blockIdx.y * kFinishWarps + warp;
       t < min(d.B, (blockIdx.y + 1) * kFinishWarps); t += kFinishWarps) {
    const size_t row = static_cast<size_t>(sh) * d.B + t;
    const int r = (h - g * d.G) * d.B + t;
    // merge the prefix partials (base-2 units) of every split in one pass,
    // kFinishBatch splits' loads in flight at a time, the running sums rescaled when
    // a batch raises the maximum
    const float* p0 = part + (static_cast<size_t>(sg) * d.nsplit * rows + r) * kPartStride;
    const size_t pstride = static_cast<size_t>(rows) * kPartStride;
    float M = -INFINITY, lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
    for (int s0 = 0; s0 < d.nsplit; s0 += kFinishBatch) {
      float mc[kFinishBatch], lc[kFinishBatch];
      float4 ac[kFinishBatch];
#pragma unroll
      for (int i = 0; i < kFinishBatch; ++i) {
        mc[i] = -INFINITY;
        if (s0 + i < d.nsplit) {
          const float* src = p0 + (s0 + i) * pstride;
          mc[i] = __ldcg(src);
          lc[i] = __ldcg(src + 1);
          ac[i] = __ldcg(reinterpret_cast<const float4*>(src + 4) + lane);
        }
      }
      float Mh = M;
#pragma unroll
      for (int i = 0; i < kFinishBatch; ++i) Mh = fmaxf(Mh, mc[i]);
      const float rs = exp2f(M - Mh);  // 0 while nothing is accumulated
      lsum *= rs;
      acc.x *= rs;
      acc.y *= rs;
      acc.z *= rs;
      acc.w *= rs;
#pragma unroll
      for (int i = 0; i < kFinishBatch; ++i) {
        if (s0 + i < d.nsplit) {
          const float w = exp2f(mc[i] - Mh);
          lsum += w * lc[i];
          acc.x += w * ac[i].x;
          acc.y += w * ac[i].y;
          acc.z += w * ac[i].z;
          acc.w += w * ac[i].w;
        }
      }
      M = Mh;
    }
    const float inv = 1.f / lsum;
    const float4 op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    const float Lp = (M + __log2f(lsum)) * kLn2;
    *reinterpret_cast<float4*>(o_p + row * kD + 4 * lane) = op;
    if (lane == 0) l_p[row] = Lp;
    const float4 q = ld4(Q, row * kD + 4 * lane, d.dtype);
    float4 os;
    float Ls;
    suffix_row(q, Ksb, Vsb, d.B, d.scale_log2, Ps[warp], os, Ls);
    float4 o;
    float L;
    lse_merge(op, Lp, os, Ls, o, L);
    *reinterpret_cast<float4*>(out + row * kD + 4 * lane) = o;
    if (out_lse && lane == 0) out_lse[row] = L;
  }
}

// ---------------------------------------------------------------------------
// bf16: 5th-generation tensor cores (tcgen05, accumulators in TMEM).
// CTA = (split, group), 288 threads, one CTA per SM: eight softmax warps
// (0-7) and a producer warp (8) whose lane 0 drives the TMA and the tensor
// core.  The group's G*B query rows, zero-padded to MR = 64 or 128 MMA rows,
// arrive once by 2-D tiled TMA in the 128-byte-swizzled layout the matrix
// descriptors describe; 128-key K and V tiles stream through a 2-stage K
// ring and a 2- (MR = 128) or 3-stage (MR = 64) V ring (the tensor maps'
// 64-channel x 128-row boxes).  Per tile: S = Q K^T (M = MR, N = 128,
// K = 128) into one of two TMEM score buffers, issued a tile ahead so the
// tensor core runs while the softmax warps work; the softmax warps read S
// from TMEM (MR = 64: the 16x256b fragment, two real rows per thread), run
// the online softmax in base 2 (the two halves of a row exchange maxima
// through shared memory) against a reference max that moves only when the
// row max grows by more than 2^8 (O and l are then rescaled in TMEM), and
// write P in bf16 to one of two shared-memory buffers; the row sum l adds the
// same rounded weights, so the output is an exactly normalised average of
// the values under weights perturbed by at most 2^-9 relative.  Then
// O += P V (N = 128, K = 128: P in two K-major 64-key atoms, V the MN-major
// operand) into a TMEM accumulator; every MMA group commits to an mbarrier.
// At the end each thread writes its rows' O, m and l to the split partials.
// Every wait is bounded; a wait that gives up records
// LOSA_ERR_DEVICE_TIMEOUT.
// ---------------------------------------------------------------------------
constexpr int kUKeys = 128;                         // keys per tile (the S MMA's N)
constexpr int kUHalf = kUKeys / 2;                  // keys of a tile per softmax warp
constexpr int kUTile = kUKeys * kD * 2;             // 32 KB: one K (or V) tile
constexpr uint32_t kUCols = 512;                    // TMEM: S [0, 256) (two tiles), O [256, 384)

// Shared-memory plan per MMA row count MR (64 or 128): the query tile and the
// P buffers scale with MR; what a 64-row group saves goes to a deeper V ring,
// so V tiles are requested a tile before their P V MMAs.
template <int MR>
struct UPlan {
  static constexpr int kst = 2;                    // K ring stages
  static constexpr int vst = MR == 64 ? 3 : 2;     // V ring stages
  static constexpr int qbytes = MR * kD * 2;       // the query tile
  static constexpr int pbytes = MR * kUKeys * 2;   // one P buffer
  static constexpr int nbars = 1 + 2 + 2 + kst + vst + 2;  // Q, S[2], O[2], K[kst], V[vst], P[2]
  static constexpr int smem = 1024 + qbytes + (kst + vst) * kUTile + 2 * pbytes + 1024 +
                              nbars * 8 + 16;
};
static_assert(UPlan<64>::smem <= 232448 && UPlan<128>::smem <= 232448, "dense plan > 227 KB");

template <int MR>
__global__ void __launch_bounds__(288, 1)
    dense_umma_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, float* __restrict__ part,
                      int* __restrict__ status, Dims d) {
  using C = UPlan<MR>;
  constexpr int kUKst = C::kst, kUVst = C::vst, kUQ = C::qbytes, kUP = C::pbytes;
  constexpr int kUBars = C::nbars;
  extern __shared__ char dsm_raw[];
  // the finish kernel may be scheduled now; it waits for this grid's
  // completion before it reads a partial
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // 1024-byte alignment for the swizzled tiles
  char* dsm = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  // MR = MMA rows (64 or 128): the group's query rows, zero-padded
  char* qs = dsm;                                     // [MR rows], 2 atoms of MR x 128 B
  char* kring = qs + kUQ;                             // kUKst K tiles (2 atoms of 16 KB)
  char* vring = kring + kUKst * kUTile;               // kUVst V tiles
  char* pbuf = vring + kUVst * kUTile;                // [2] P buffers
  float* xmax = reinterpret_cast<float*>(pbuf + 2 * kUP);     // [2][128]: the halves' row maxima
  uint64_t* bars = reinterpret_cast<uint64_t*>(xmax + 256);
  uint64_t* bQ = bars;
  uint64_t* bS = bars + 1;     // [2] S buffer ready
  uint64_t* bO = bars + 3;     // [2] O += P V of an even / odd tile done
  uint64_t* bK = bars + 5;     // [kUKst] K tile landed
  uint64_t* bV = bars + 5 + kUKst;  // [kUVst] V tile landed
  uint64_t* bP = bars + 5 + kUKst + kUVst;  // [2] P buffer written (256 arrivals)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + kUBars);
  int* s_fail = reinterpret_cast<int*>(tslot + 1);
  const int sg = blockIdx.y, split = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int rows = d.G * d.B;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int key0 = split * d.split_pages * kPS;
  const int key1 = min(seq_len(d, s), key0 + d.split_pages * kPS);
  const int n = key1 > key0 ? (key1 - key0 + kUKeys - 1) / kUKeys : 0;
  if (split == 0 && tid == 0 && seq_len_bad(d, s)) atomicCAS(status, 0, LOSA_ERR_DEVICE_BOUNDS);
  if (n == 0) {  // a split past a shorter sequence's end: an empty partial per row
    float* dst0 = part + (static_cast<size_t>(sg) * d.nsplit + split) * rows * kPartStride;
    for (int e = tid; e < rows * kPartStride; e += blockDim.x)
      dst0[e] = (e % kPartStride) == 0 ? -INFINITY : 0.f;
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < kUBars; ++i) mbar_init(&bars[i], i >= 5 + kUKst + kUVst ? 256 : 1);
    fence_mbar_init();
    *s_fail = 0;
  }
  if (warp == 0) tmem_alloc(tslot, kUCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const uint32_t tO = tbase + 2 * kUKeys;  // S tiles: columns [0, 128) and [128, 256)
  bool ok = true;
  // V rows of a partial last tile past the split's end are outside the
  // prefix (a capacity region or a shorter sequence's unused tokens) and may
  // hold anything; P is 0 there, but 0 times a NaN or Inf of V would still
  // reach O, so the softmax warps zero those rows once the tile has landed
  // and before they publish P (rows r of both 64-channel atoms are the bytes
  // [128 r, 128 r + 128): the swizzle permutes chunks inside a row)
  auto zero_v_tail = [&](int t) {
    const int nv = key1 - (key0 + t * kUKeys);  // real keys of the tile, 1 .. 127
    ok = ok && mbar_wait(&bV[t % kUVst], (t / kUVst) & 1);
    char* vt = vring + (t % kUVst) * kUTile;
    const int per = (kUKeys - nv) * 8;  // 16-byte chunks past the real rows, per atom
    for (int e = tid; e < 2 * per; e += 256) {
      const int a = e >= per ? 1 : 0;
      *reinterpret_cast<uint4*>(vt + a * (kUTile / 2) + nv * 128 + (e - a * per) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
  };

  if (warp == 8) {
    // ---- producer: TMA loads and tensor-core MMAs, one thread
    if (lane == 0) {
      const int kv_row0 = sg * d.Lc + key0;           // first key of the split, as a tensor row
      const int q_row0 = (s * d.Hq + g * d.G) * d.B;  // the group's first query row
      auto load_k = [&](int t) {
        uint64_t* bar = &bK[t % kUKst];
        char* dst = kring + (t % kUKst) * kUTile;
        mbar_expect_tx(bar, kUTile);
        tma_load_2d(dst, &kmap, 0, kv_row0 + t * kUKeys, bar);
        tma_load_2d(dst + kUTile / 2, &kmap, 64, kv_row0 + t * kUKeys, bar);
      };
      auto load_v = [&](int t) {
        uint64_t* bar = &bV[t % kUVst];
        char* dst = vring + (t % kUVst) * kUTile;
        mbar_expect_tx(bar, kUTile);
        tma_load_2d(dst, &vmap, 0, kv_row0 + t * kUKeys, bar);
        tma_load_2d(dst + kUTile / 2, &vmap, 64, kv_row0 + t * kUKeys, bar);
      };
      constexpr uint32_t idesc_s = umma_idesc_bf16(MR, kUKeys, 0);
      constexpr uint32_t idesc_o = umma_idesc_bf16(MR, kD, 1);
      // descriptors at offset 0; a k-step adds its byte offset >> 4 to the
      // start-address field (no carry: shared addresses stay below 256 KB)
      const uint64_t dq = umma_desc(su32(qs), 16, 1024);
      auto issue_s = [&](int t) {  // S = Q K^T of tile t into S buffer t & 1
        const uint64_t dk = umma_desc(su32(kring + (t % kUKst) * kUTile), 16, 1024);
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t ko = (ks >> 2) * (MR * 128) + (ks & 3) * 32;
          const uint32_t kk = (ks >> 2) * (kUKeys * 128) + (ks & 3) * 32;
          umma_bf16(tbase + (t & 1) * kUKeys, dq + (ko >> 4), dk + (kk >> 4), idesc_s, ks > 0);
        }
        umma_commit(&bS[t & 1]);
      };
      mbar_expect_tx(bQ, MR * 256);
      tma_load_2d(qs, &qmap, 0, q_row0, bQ);
      tma_load_2d(qs + MR * 128, &qmap, 64, q_row0, bQ);
      for (int t = 0; t < min(n, kUKst); ++t) load_k(t);
      int vnext = 0;  // the next V tile to request
      while (vnext < min(n, kUVst)) load_v(vnext++);
      ok = ok && mbar_wait(bQ, 0) && mbar_wait(&bK[0], 0);
      issue_s(0);
#pragma unroll 1
      for (int t = 0; t < n && ok; ++t) {  // (a failed wait ends the stream; the softmax warps give up too)
        if (t + 1 < n) {  // the next tile's scores run during this tile's softmax
          ok = ok && mbar_wait(&bK[(t + 1) % kUKst], ((t + 1) / kUKst) & 1);
          issue_s(t + 1);
        }
        ok = ok && mbar_wait(&bS[t & 1], (t >> 1) & 1);
        if (t + kUKst < n) load_k(t + kUKst);  // tile t's K stage is free again
        // P V of two tiles back has finished (before this barrier completes
        // again): the V stages of tiles <= t - 2 are free
        if (t >= 2) {
          ok = ok && mbar_wait(&bO[t & 1], ((t - 2) >> 1) & 1);
          while (vnext < n && vnext <= t - 2 + kUVst) load_v(vnext++);
        }
        ok = ok && mbar_wait(&bP[t & 1], (t >> 1) & 1) && mbar_wait(&bV[t % kUVst], (t / kUVst) & 1);
        tc_fence_after();
        const uint64_t dv = umma_desc(su32(vring + (t % kUVst) * kUTile), kUKeys * 128, 1024);
        const uint64_t dp = umma_desc(su32(pbuf + (t & 1) * kUP), 16, 1024);
#pragma unroll
        for (int ks = 0; ks < kUKeys / 16; ++ks)  // P: two K-major atoms of 64 keys
          umma_bf16(tO, dp + (((ks >> 2) * (MR * 128) + (ks & 3) * 32) >> 4),
                    dv + ((ks * 16 * 128) >> 4), idesc_o, (t > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&bO[t & 1]);
      }
      if (!ok) *s_fail = 1;
    }
  } else if constexpr (MR == 64) {
    // ---- softmax warps, 64 accumulator rows: rows 16q .. 16q + 15 of
    // sub-partition q = w % 4 live in TMEM lanes 32q .. 32q + 15; the 16x256b
    // fragment gives thread t rows 16q + t/4 and 16q + t/4 + 8, so every
    // lane holds real scores.  Warp w takes key half w / 4 of each S tile
    // (64 keys: 16 per row and thread, two 32-column blocks) and the same
    // half of O's columns.
    const int q4 = warp & 3, half = warp >> 2, tq = lane & 3;
    const int rr[2] = {16 * q4 + (lane >> 2), 16 * q4 + (lane >> 2) + 8};
    const bool valid[2] = {rr[0] < rows, rr[1] < rows};
    const bool busy = 16 * q4 < rows;  // (warp-uniform) some row of this warp is real
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const float sl2 = d.scale_log2;
    float mref[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
#pragma unroll 1
    for (int t = 0; t < n; ++t) {
      ok = ok && mbar_wait(&bS[t & 1], (t >> 1) & 1);
      // the P buffers of this parity are free once P V of two tiles back is done
      ok = ok && (t < 2 || mbar_wait(&bO[t & 1], ((t - 2) >> 1) & 1));
      tc_fence_after();
      // block b, register r: row rr[(r >> 1) & 1], key kb + 32 b + 8 (r >> 2)
      // + 2 tq + (r & 1)
      const int kb = key0 + t * kUKeys + half * kUHalf;
      float sv[2][16];
      float mx[2] = {-INFINITY, -INFINITY};
      if (busy) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          tmem_ld16x256_x4(tbase + (t & 1) * kUKeys + half * kUHalf + 32 * b + lane_off, sv[b]);
#pragma unroll
          for (int r = 0; r < 16; ++r) {
            const int key = kb + 32 * b + 8 * (r >> 2) + 2 * tq + (r & 1);
            sv[b][r] = key < key1 ? sv[b][r] * sl2 : -INFINITY;
            mx[(r >> 1) & 1] = fmaxf(mx[(r >> 1) & 1], sv[b][r]);
          }
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {  // the row's four threads
          mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
          mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
        }
        if (tq == 0) {
          xmax[half * 128 + rr[0]] = mx[0];
          xmax[half * 128 + rr[1]] = mx[1];
        }
      }
      bar_sync(1, 256);  // both halves' maxima
      char* pb = pbuf + (t & 1) * kUP;
      if (busy) {
        bool grow[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          mx[i] = fmaxf(xmax[rr[i]], xmax[128 + rr[i]]);
          // the same decision in both halves of the row; padding rows never move
          grow[i] = valid[i] && mx[i] > mref[i] + 8.f;
        }
        if (__any_sync(0xffffffffu, grow[0] || grow[1])) {  // tcgen05.ld/st are warp-wide
          float alpha[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const float nref = grow[i] ? mx[i] : mref[i];
            alpha[i] = grow[i] ? exp2f(mref[i] - nref) : 1.f;  // 0 while nothing is accumulated
            lrow[i] *= alpha[i];
            mref[i] = nref;
          }
          if (t > 0) {
            // O holds every P V up to tile t - 1
            ok = ok && mbar_wait(&bO[(t - 1) & 1], ((t - 1) >> 1) & 1);
            tc_fence_after();
#pragma unroll 1
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
              float v[16];
              tmem_ld16x256_x4(tO + lane_off + c0, v);
#pragma unroll
              for (int r = 0; r < 16; ++r) v[r] *= alpha[(r >> 1) & 1];
              tmem_st16x256_x4(tO + lane_off + c0, v);
            }
          }
        }
        // P = 2^(s - mref) <= 2^8 in bf16, [64 rows][128 keys] K-major (two
        // atoms of 64 keys), swizzled, one 4-byte store per key pair; l adds
        // the rounded weights
#pragma unroll
        for (int b = 0; b < 2; ++b) {
#pragma unroll
          for (int r = 0; r < 16; r += 2) {
            const int i = (r >> 1) & 1;
            const uint32_t pw = pack_bf16x2(ex2_approx(sv[b][r] - mref[i]),
                                            ex2_approx(sv[b][r + 1] - mref[i]));
            lrow[i] += __uint_as_float(pw << 16) + __uint_as_float(pw & 0xffff0000u);
            *reinterpret_cast<uint32_t*>(
                pb + sw128_off(rr[i], half * kUHalf + 32 * b + 8 * (r >> 2) + 2 * tq, MR)) = pw;
          }
        }
      }
      if (key0 + (t + 1) * kUKeys > key1) zero_v_tail(t);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bP[t & 1]);
    }
    ok = ok && mbar_wait(&bO[(n - 1) & 1], ((n - 1) >> 1) & 1);
    tc_fence_after();
    if (!__all_sync(0xffffffffu, ok) && lane == 0) *s_fail = 1;
#pragma unroll
    for (int i = 0; i < 2; ++i) {  // the row's four threads' shares of this half's sum
      lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 1);
      lrow[i] += __shfl_xor_sync(0xffffffffu, lrow[i], 2);
    }
    if (busy && half == 1 && tq == 0) {  // the second half's row sums
      xmax[rr[0]] = lrow[0];
      xmax[rr[1]] = lrow[1];
    }
    bar_sync(1, 256);
    if (!*s_fail && busy) {
      float* dst0 = part + ((static_cast<size_t>(sg) * d.nsplit + split) * rows) * kPartStride;
#pragma unroll 1
      for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
        float v[16];
        tmem_ld16x256_x4(tO + lane_off + c0, v);
#pragma unroll
        for (int r = 0; r < 16; r += 2) {
          const int i = (r >> 1) & 1;
          if (valid[i])
            *reinterpret_cast<float2*>(dst0 + rr[i] * kPartStride + 4 + c0 + 8 * (r >> 2) +
                                       2 * tq) = make_float2(v[r], v[r + 1]);
        }
      }
      if (half == 0 && tq == 0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          if (!valid[i]) continue;
          float* dst = dst0 + rr[i] * kPartStride;
          dst[0] = mref[i];
          dst[1] = lrow[i] + xmax[rr[i]];
        }
      }
    }
  } else {
    // ---- softmax warps: warp w reads TMEM lanes 32 (w % 4) .. (its
    // sub-partition), where the accumulator rows (M = 128) 32 (w % 4) + lane
    // or (M = 64) 16 (w % 4) + lane, lane < 16, live; a thread owns its row's
    // w / 4 half of each S tile's keys and of O
    constexpr int RPW = MR / 4;  // accumulator rows per sub-partition
    const int row = (warp & 3) * RPW + lane, half = warp >> 2;
    const bool mine = lane < RPW && row < rows;  // this thread's row is a real query row
    const bool busy = (warp & 3) * RPW < rows;   // (warp-uniform) some row of this warp is real
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = d.scale_log2;
    float mref = -INFINITY, lrow = 0.f;  // lrow: this half's share of the row sum
#pragma unroll 1
    for (int t = 0; t < n; ++t) {
      ok = ok && mbar_wait(&bS[t & 1], (t >> 1) & 1);
      // the P buffers of this parity are free once P V of two tiles back is done
      ok = ok && (t < 2 || mbar_wait(&bO[t & 1], ((t - 2) >> 1) & 1));
      tc_fence_after();
      const int kb = key0 + t * kUKeys + half * kUHalf;
      float sv[2][32];
      float mx = -INFINITY;
      if (busy) {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          tmem_ld32(tbase + (t & 1) * kUKeys + half * kUHalf + 32 * b + lane_off, sv[b]);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            sv[b][i] = kb + 32 * b + i < key1 ? sv[b][i] * sl2 : -INFINITY;
            mx = fmaxf(mx, sv[b][i]);
          }
        }
        if (lane < RPW) xmax[half * 128 + row] = mx;
      }
      bar_sync(1, 256);  // both halves' maxima
      char* pb = pbuf + (t & 1) * kUP;
      if (busy) {
        if (lane < RPW) mx = fmaxf(xmax[row], xmax[128 + row]);
        // the same decision in both halves of the row; padding lanes never move
        const bool grow = mine && mx > mref + 8.f;
        if (__any_sync(0xffffffffu, grow)) {  // tcgen05.ld/st are warp-wide
          const float nref = grow ? mx : mref;
          const float alpha = grow ? exp2f(mref - nref) : 1.f;  // 0 while nothing is accumulated
          lrow *= alpha;
          if (t > 0) {
            // O holds every P V up to tile t - 1
            ok = ok && mbar_wait(&bO[(t - 1) & 1], ((t - 1) >> 1) & 1);
            tc_fence_after();
#pragma unroll 1
            for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
              float v[32];
              tmem_ld32(tO + lane_off + c0, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tmem_st32(tO + lane_off + c0, v);
            }
          }
          mref = nref;
        }
        // P = 2^(s - mref) <= 2^8 in bf16, [128 rows][128 keys] K-major (two
        // atoms of 64 keys), swizzled; l adds the rounded weights
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t pw[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            pw[u] = pack_bf16x2(ex2_approx(sv[c8 >> 2][(c8 & 3) * 8 + 2 * u] - mref),
                                ex2_approx(sv[c8 >> 2][(c8 & 3) * 8 + 2 * u + 1] - mref));
            lrow += __uint_as_float(pw[u] << 16) + __uint_as_float(pw[u] & 0xffff0000u);
          }
          if (lane < RPW)
            *reinterpret_cast<uint4*>(pb + sw128_off(row, half * kUHalf + c8 * 8, MR)) =
                make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
      }
      if (key0 + (t + 1) * kUKeys > key1) zero_v_tail(t);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bP[t & 1]);
    }
    ok = ok && mbar_wait(&bO[(n - 1) & 1], ((n - 1) >> 1) & 1);
    tc_fence_after();
    if (!__all_sync(0xffffffffu, ok) && lane == 0) *s_fail = 1;
    if (half == 1 && lane < RPW) xmax[row] = lrow;  // the second half's row sum
    bar_sync(1, 256);
    if (!*s_fail && busy) {
      float* dst = part + ((static_cast<size_t>(sg) * d.nsplit + split) * rows + row) * kPartStride;
#pragma unroll 1
      for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {
        float v[32];
        tmem_ld32(tO + lane_off + c0, v);
        if (mine) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + 4 + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
        }
      }
      if (mine && half == 0) {
        dst[0] = mref;
        dst[1] = lrow + xmax[row];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *s_fail) atomicCAS(status, 0, LOSA_ERR_DEVICE_TIMEOUT);
  if (warp == 0) tmem_dealloc(tbase, kUCols);
}

}  // namespace
}  // namespace losa

extern "C" int losa_dense_prefix(const losa_shape* shape, const void* q, const void* k_prefix,
                                 const void* v_prefix, const void* k_blk, const void* v_blk,
                                 float* o_p, float* l_p, float* out, float* out_lse,
                                 void* workspace, size_t ws_bytes, void* stream) {
  using namespace losa;
  Dims d;
  int rc = make_dims(shape, LOSA_WS_DENSE, &d);
  if (rc != LOSA_OK) return rc;
  if (bad_ptr(q) || bad_ptr(k_prefix) || bad_ptr(v_prefix) || bad_ptr(k_blk) || bad_ptr(v_blk) ||
      bad_ptr(o_p) || bad_ptr(l_p) || bad_ptr(out) || bad_opt_ptr(out_lse) || !workspace ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return LOSA_ERR_INVALID_ARG;
  if (ws_bytes < d.total) return LOSA_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(d.S) * d.Hq * d.B;
  const size_t SG = static_cast<size_t>(d.S) * d.Hkv;
  const size_t qb = rows * kD * d.esz, ob = rows * kD * sizeof(float), lb = rows * sizeof(float);
  const size_t kvb = SG * d.Lc * kD * d.esz, kbb = SG * d.B * kD * d.esz;
  const Region reg[] = {{q, qb, false},       {k_prefix, kvb, false}, {v_prefix, kvb, false},
                        {k_blk, kbb, false},  {v_blk, kbb, false},    {o_p, ob, true},
                        {l_p, lb, true},      {out, ob, true},        {out_lse, lb, true},
                        {workspace, d.total, true}};
  if (any_write_alias(reg, static_cast<int>(sizeof(reg) / sizeof(reg[0]))))
    return LOSA_ERR_INVALID_ARG;
  if (d.S * d.Hkv > 65535) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = reinterpret_cast<float*>(static_cast<char*>(workspace) + d.off_part);
  int* status = reinterpret_cast<int*>(static_cast<char*>(workspace) + d.off_status);
  if (d.dtype == LOSA_BF16) {
    if (d.G * d.B > 128) return LOSA_ERR_UNSUPPORTED;
    static bool attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !attr_done[dev]) {
      cudaError_t e0 = cudaFuncSetAttribute(
          dense_umma_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, UPlan<64>::smem);
      if (e0 == cudaSuccess)
        e0 = cudaFuncSetAttribute(dense_umma_kernel<128>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, UPlan<128>::smem);
      if (e0 != cudaSuccess) return record_cuda_error(e0);
      attr_done[dev] = true;
    }
    const bool m64 = d.G * d.B <= 64;
    CUtensorMap qmap, kmap, vmap;
    if (make_tmap(&qmap, q, rows, m64 ? 64 : 128) != LOSA_OK ||
        make_tmap(&kmap, k_prefix, static_cast<unsigned long long>(d.S) * d.Hkv * d.Lc, kUKeys) != LOSA_OK ||
        make_tmap(&vmap, v_prefix, static_cast<unsigned long long>(d.S) * d.Hkv * d.Lc, kUKeys) != LOSA_OK)
      return record_cuda_error(cudaErrorInvalidValue);
    if (m64)
      dense_umma_kernel<64><<<dim3(d.nsplit, d.S * d.Hkv), 288, UPlan<64>::smem, st>>>(
          qmap, kmap, vmap, part, status, d);
    else
      dense_umma_kernel<128><<<dim3(d.nsplit, d.S * d.Hkv), 288, UPlan<128>::smem, st>>>(
          qmap, kmap, vmap, part, status, d);
  } else {
    dense_partial_kernel<<<dim3(d.nsplit, d.S * d.Hkv), kDenseWarps * 32, 0, st>>>(
        q, k_prefix, v_prefix, part, status, d);
  }
  {
    // behind the split kernel with programmatic dependent launch: the finish
    // CTAs stage the block's K/V while the split kernel drains
    cudaLaunchConfig_t cf = {};
    cudaLaunchAttribute at[1];
    cf.gridDim = dim3(d.S * d.Hq, (d.B + kFinishWarps - 1) / kFinishWarps, 1);
    cf.blockDim = dim3(kFinishWarps * 32, 1, 1);
    cf.dynamicSmemBytes = 2u * ((d.B + kPS - 1) / kPS * kPS) * kD * sizeof(float);
    cf.stream = st;
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cf.attrs = at;
    cf.numAttrs = 1;
    const cudaError_t ef = cudaLaunchKernelEx(&cf, dense_finish_kernel, q, k_blk, v_blk,
                                              static_cast<const float*>(part), o_p, l_p, out,
                                              out_lse, d);
    if (ef != cudaSuccess) return record_cuda_error(ef);
  }
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
