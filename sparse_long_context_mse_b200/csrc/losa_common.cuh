// losa_common.cuh -- shared definitions of the LoSA CUDA library (sm_100a).
//
// Host-side shape derivation and workspace layout, plus the small device
// helpers every kernel uses (element loads, warp reductions, order-preserving
// selection keys).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "losa.h"

namespace losa {

constexpr int kD = 128;         // head dimension the kernels implement
constexpr int kPS = 16;         // tokens per page
constexpr int kMaxB = 32;       // block tokens (one warp lane per token)
constexpr int kMaxRowsPerGroup = 128;  // G*B (and hence G*A) per KV head
constexpr int kMaxK = 64;       // pages per active row unless every page is taken
constexpr int kPartStride = kD + 4;    // floats per split-softmax partial: m, l, pad, pad, acc[d]
constexpr int kMaxDevices = 64;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Shape-derived sizes and workspace layout (host computed, passed by value).
// ---------------------------------------------------------------------------
struct Dims {
  int S, Hq, Hkv, G, L, P, B, A, k, R, MW, Umax, dtype, esz;
  int Lc, Pc;             // prefix capacity: tokens (K/V row stride) and page records per (s, g)
  int all_pages;          // k == P: every page is selected, no scoring needed
  int attend_union;       // LOSA_STEP_ATTEND_UNION: active rows attend to the group's union
  const int32_t* lens;    // per-sequence prefix lengths (device, [S]) or null: every one is L
  float scale;            // softmax scale (natural-log units)
  float scale_log2;       // scale * log2(e): scores in base-2 units
  // prefix splits (dense pass)
  int nsplit, split_pages;
  // workspace byte offsets
  size_t off_status, off_part, total;
};

// Element load as float (bf16 -> f32 is exact).
__device__ __forceinline__ float ld_elem(const void* base, size_t idx, int dtype) {
  if (dtype == LOSA_BF16) {
    const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(base);
    return __bfloat162float(p[idx]);
  }
  return static_cast<const float*>(base)[idx];
}

// Four consecutive elements starting at idx (idx % 4 == 0) as floats.
__device__ __forceinline__ float4 ld4(const void* base, size_t idx, int dtype) {
  if (dtype == LOSA_BF16) {
    uint2 raw = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(base) + idx);
    float4 r;
    r.x = __uint_as_float(raw.x << 16);
    r.y = __uint_as_float(raw.x & 0xffff0000u);
    r.z = __uint_as_float(raw.y << 16);
    r.w = __uint_as_float(raw.y & 0xffff0000u);
    return r;
  }
  return *reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
    v = w > v ? w : v;
  }
  return v;
}

// Order-preserving map of a float to uint32 (larger float -> larger uint);
// -0 is folded onto +0 so that equal values tie.
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Selection key: larger score first, then lower index.  Never 0 for a real
// candidate (the low word is ~idx with idx < 2^31), so 0 marks "empty".
__device__ __forceinline__ unsigned long long sel_key(float score, int idx) {
  return (static_cast<unsigned long long>(ordered_bits(score)) << 32) |
         static_cast<unsigned long long>(~static_cast<uint32_t>(idx));
}
__device__ __forceinline__ int key_index(unsigned long long key) {
  return static_cast<int>(~static_cast<uint32_t>(key & 0xffffffffull));
}

// Physical byte offset, inside a page-metadata record, of logical byte b
// (16-byte chunks XOR-swizzled by the page index).
__host__ __device__ __forceinline__ uint32_t meta_swz(uint32_t b, int page) {
  return ((((b >> 4) ^ static_cast<uint32_t>(page & 7)) << 4) | (b & 15u));
}

// The page-norm section of the page metadata, after the S*Hkv*Pc records:
// for every (s, g) a row of meta_norm_stride(d) float2 entries, entry p =
// (||kmin||_2, ||kmax||_2) of page p over the d channels, each rounded up (an
// upper bound of the exact norm).  The row stride is a multiple of 8 entries
// so that every 8-page run starts on a 64-byte boundary.
__host__ __device__ __forceinline__ size_t meta_norm_offset(const Dims& d) {
  return static_cast<size_t>(d.S) * d.Hkv * d.Pc * 2 * kD * d.esz;
}
__host__ __device__ __forceinline__ int meta_norm_stride(const Dims& d) {
  return (d.Pc + 7) / 8 * 8;
}

// Prefix length of sequence s: its entry of the per-sequence lengths, clamped
// into [1, L] (so that every access stays inside the buffers), else L.
__device__ __forceinline__ int seq_len(const Dims& d, int s) {
  return d.lens ? min(max(d.lens[s], 1), d.L) : d.L;
}
// The entry of sequence s lies outside [1, L] (seq_len clamped it).
__device__ __forceinline__ bool seq_len_bad(const Dims& d, int s) {
  return d.lens && (d.lens[s] < 1 || d.lens[s] > d.L);
}

__device__ __forceinline__ void set_status(void* ws, int code) {
  atomicCAS(static_cast<int*>(ws), 0, code);
}

// ---------------------------------------------------------------------------
// Online softmax over one page (<= 16 keys) for one query row, one warp.
//
// Lane l owns channels [4l, 4l+4).  q: the lane's query channels; Ks/Vs:
// [16][kD] floats in shared memory (rows >= ntok ignored).  State (m in
// base-2 units of the scaled score, l = sum of 2^(s - m), acc = the lane's
// channels of sum 2^(s - m) v) is updated in place.  Ps: 16 floats of
// per-warp shared scratch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void attend_page_row(float4 q, const float* Ks, const float* Vs,
                                                int ntok, float scale_log2, float& m, float& l,
                                                float4& acc, float* Ps) {
  const int lane = threadIdx.x & 31;
  float v[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    float4 k = *reinterpret_cast<const float4*>(Ks + j * kD + 4 * lane);
    v[j] = q.x * k.x + q.y * k.y + q.z * k.z + q.w * k.w;
  }
  // reduce-scatter across the warp: after the butterfly lanes 2j and 2j+1
  // hold the full dot product of key j
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = lane & 16;
    float send = hi ? v[i] : v[i + 8];
    float keep = hi ? v[i + 8] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = lane & 8;
    float send = hi ? v[i] : v[i + 4];
    float keep = hi ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = lane & 4;
    float send = hi ? v[i] : v[i + 2];
    float keep = hi ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool hi = lane & 2;
    float send = hi ? v[0] : v[1];
    float keep = hi ? v[1] : v[0];
    v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
  const int key = lane >> 1;
  float sc = key < ntok ? v[0] * scale_log2 : -INFINITY;
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
    const float pj = Ps[j];
    psum += pj;
    float4 vv = *reinterpret_cast<const float4*>(Vs + j * kD + 4 * lane);
    o.x += pj * vv.x;
    o.y += pj * vv.y;
    o.z += pj * vv.z;
    o.w += pj * vv.w;
  }
  acc = o;
  l = l * alpha + psum;
  m = m_new;
}

// Log-sum-exp merge of two normalised partial attentions given as
// (o, L) with L in natural-log units.
__device__ __forceinline__ void lse_merge(float4 o1, float L1, float4 o2, float L2, float4& o,
                                          float& L) {
  const float m = fmaxf(L1, L2);
  const float a = __expf(L1 - m), b = __expf(L2 - m);
  const float inv = __frcp_rn(a + b);
  o.x = (a * o1.x + b * o2.x) * inv;
  o.y = (a * o1.y + b * o2.y) * inv;
  o.z = (a * o1.z + b * o2.z) * inv;
  o.w = (a * o1.w + b * o2.w) * inv;
  L = m + __logf(a + b);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
inline bool bad_ptr(const void* p) {
  return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) != 0;
}
inline bool bad_opt_ptr(const void* p) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) != 0;
}
inline bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// A buffer an entry point reads or writes: base, bytes, whether it is written.
struct Region {
  const void* p;
  size_t n;
  bool w;
};
// Whether two of the regions overlap where at least one of the two is written
// (read-only inputs may alias each other; a null region is skipped).
inline bool any_write_alias(const Region* r, int n) {
  for (int i = 0; i < n; ++i)
    for (int j = i + 1; j < n; ++j)
      if ((r[i].w || r[j].w) && overlaps(r[i].p, r[i].n, r[j].p, r[j].n)) return true;
  return false;
}

int make_dims(const losa_shape* sh, int which, Dims* d);
// Whether the fused step kernel's shared-memory plan fits in `max_dyn` bytes.
bool fused_step_fits(const Dims& d, int max_dyn);
// Dynamic shared memory a B200 CTA may opt in to (227 KB).
constexpr int kB200MaxDynSmem = 232448;
// The fused step kernel (step_fused.cu); arguments already validated.
int launch_fused_step(const Dims& d, const void* q_cur, const void* q_prev, const void* k_prefix,
                      const void* v_prefix, const void* page_meta, const void* k_blk,
                      const void* v_blk, float* o_p, float* l_p, float* out, float* out_lse,
                      int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                      void* workspace, cudaStream_t st, void* q_ref_out = nullptr);
int record_cuda_error(cudaError_t e);  // stores the message, returns LOSA_ERR_CUDA
// 2-D tensor map over a [nrows][128] bf16 tensor at `base`, for
// 128-byte-swizzled boxes of 64 channels x box_rows rows (rows past nrows
// read as zero).  LOSA_OK, or LOSA_ERR_CUDA if the driver refuses it.
int make_tmap(CUtensorMap* map, const void* base, unsigned long long nrows, unsigned box_rows);
// A 3-D map over the same [nrows][kD] bf16 rows whose box is one page of
// kPS rows, both 64-channel halves: dims (channel within the half, row,
// half), so that one copy lands the page as [half][row][64 channels] with
// the 128-byte swizzle (the layout of two 2-D boxes at offsets 0 and
// kPS * 128).  LOSA_ERR_CUDA if the driver refuses the map.
int make_page_tmap(CUtensorMap* map, const void* base, unsigned long long nrows);
int num_sms();

}  // namespace losa
