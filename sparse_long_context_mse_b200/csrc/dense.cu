// dense.cu -- cold-start dense prefix pass (first denoising step of a block).
//
// LoSA needs the full prefix attention of every block token once per block
// to seed the reuse cache (LoSA paper, limitations: the first denoising
// iteration of each block stays dense).  Flash-decode layout: the prefix of
// each (sequence, KV head) is split into page ranges; one CTA streams one
// range for all G*B query rows of the group and writes an unnormalised
// online-softmax partial per row; the finish kernel merges the partials, adds
// the dense suffix over the block's own keys and writes cache and output.
#include "losa_common.cuh"

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
                         const void* __restrict__ V, float* __restrict__ part, Dims d) {
  __shared__ __align__(16) float Ks[kPS * kD];
  __shared__ __align__(16) float Vs[kPS * kD];
  __shared__ float Ps[kDenseWarps][kPS];
  const int sg = blockIdx.y, split = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = d.G * d.B;
  const int p0 = split * d.split_pages;
  const int p1 = min(d.P, p0 + d.split_pages);
  const size_t kv0 = static_cast<size_t>(sg) * d.L * kD;

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
      const int ntok = min(kPS, d.L - p * kPS);
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

__global__ void __launch_bounds__(128)
    dense_finish_kernel(const void* __restrict__ Q, const void* __restrict__ Kb,
                        const void* __restrict__ Vb, const float* __restrict__ part,
                        float* __restrict__ o_p, float* __restrict__ l_p, float* __restrict__ out,
                        float* __restrict__ out_lse, Dims d) {
  __shared__ __align__(16) float Ksb[kMaxB * kD];
  __shared__ __align__(16) float Vsb[kMaxB * kD];
  __shared__ float Ps[4][kPS];
  const int sh = blockIdx.x;  // s * Hq + h
  const int s = sh / d.Hq, h = sh % d.Hq, g = h / d.G;
  const int sg = s * d.Hkv + g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = d.G * d.B;
  const int Bpad = (d.B + kPS - 1) / kPS * kPS;
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
  for (int t = warp; t < d.B; t += 4) {
    const size_t row = static_cast<size_t>(sh) * d.B + t;
    const int r = (h - g * d.G) * d.B + t;
    // merge the prefix partials (base-2 units) of every split
    float M = -INFINITY;
    for (int sp = 0; sp < d.nsplit; ++sp)
      M = fmaxf(M, part[((static_cast<size_t>(sg) * d.nsplit + sp) * rows + r) * kPartStride]);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < d.nsplit; ++sp) {
      const float* src = part + ((static_cast<size_t>(sg) * d.nsplit + sp) * rows + r) * kPartStride;
      const float w = exp2f(src[0] - M);
      lsum += w * src[1];
      const float4 a = *reinterpret_cast<const float4*>(src + 4 + 4 * lane);
      acc.x += w * a.x;
      acc.y += w * a.y;
      acc.z += w * a.z;
      acc.w += w * a.w;
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
  const size_t qb = rows * kD * d.esz;
  if (overlaps(out, rows * kD * 4, q, qb) || overlaps(out, rows * kD * 4, o_p, rows * kD * 4))
    return LOSA_ERR_INVALID_ARG;
  if (d.S * d.Hkv > 65535) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* part = reinterpret_cast<float*>(static_cast<char*>(workspace) + d.off_part);
  dense_partial_kernel<<<dim3(d.nsplit, d.S * d.Hkv), kDenseWarps * 32, 0, st>>>(
      q, k_prefix, v_prefix, part, d);
  dense_finish_kernel<<<d.S * d.Hq, 128, 0, st>>>(q, k_blk, v_blk, part, o_p, l_p, out, out_lse,
                                                  d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
