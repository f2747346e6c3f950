// meta.cu -- page min/max metadata build (once per prefix).
//
// QUEST's bound needs, per page and channel, the min and max key value over
// the page's tokens (LoSA paper, methodology: QUEST-style selection over KV
// pages).  One warp per page; lane l owns channels [4l, 4l+4).  Min/max are
// exact, so the result is bit-identical to any correct implementation.
#include "losa_common.cuh"

namespace losa {
namespace {

constexpr int kMetaWarps = 8;

__global__ void __launch_bounds__(kMetaWarps * 32)
    meta_build_kernel(const void* __restrict__ K, void* __restrict__ meta, Dims d) {
  const int sg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * kMetaWarps + warp;
  if (p >= d.P) return;
  const int j0 = p * kPS;
  const int n = min(kPS, d.L - j0);
  const size_t base = (static_cast<size_t>(sg) * d.L + j0) * kD + 4 * lane;
  float4 lo = ld4(K, base, d.dtype), hi = lo;
  for (int j = 1; j < n; ++j) {
    const float4 x = ld4(K, base + static_cast<size_t>(j) * kD, d.dtype);
    // strict comparisons: the first of equal values (e.g. -0 vs +0) is kept
    lo.x = x.x < lo.x ? x.x : lo.x;
    lo.y = x.y < lo.y ? x.y : lo.y;
    lo.z = x.z < lo.z ? x.z : lo.z;
    lo.w = x.w < lo.w ? x.w : lo.w;
    hi.x = x.x > hi.x ? x.x : hi.x;
    hi.y = x.y > hi.y ? x.y : hi.y;
    hi.z = x.z > hi.z ? x.z : hi.z;
    hi.w = x.w > hi.w ? x.w : hi.w;
  }
  char* rec = static_cast<char*>(meta) + (static_cast<size_t>(sg) * d.P + p) * (2 * kD * d.esz);
  if (d.dtype == LOSA_BF16) {
    // the values are bf16 numbers held in fp32: the top 16 bits are exact
    uint2 mn, mx;
    mn.x = (__float_as_uint(lo.x) >> 16) | (__float_as_uint(lo.y) & 0xffff0000u);
    mn.y = (__float_as_uint(lo.z) >> 16) | (__float_as_uint(lo.w) & 0xffff0000u);
    mx.x = (__float_as_uint(hi.x) >> 16) | (__float_as_uint(hi.y) & 0xffff0000u);
    mx.y = (__float_as_uint(hi.z) >> 16) | (__float_as_uint(hi.w) & 0xffff0000u);
    *reinterpret_cast<uint2*>(rec + meta_swz(8u * lane, p)) = mn;
    *reinterpret_cast<uint2*>(rec + meta_swz(2u * kD + 8u * lane, p)) = mx;
  } else {
    *reinterpret_cast<float4*>(rec + meta_swz(16u * lane, p)) = lo;
    *reinterpret_cast<float4*>(rec + meta_swz(4u * kD + 16u * lane, p)) = hi;
  }
}

}  // namespace
}  // namespace losa

extern "C" int losa_build_page_meta(const losa_shape* shape, const void* k_prefix,
                                    void* page_meta, void* stream) {
  using namespace losa;
  Dims d;
  int rc = make_dims(shape, LOSA_WS_DENSE, &d);
  if (rc != LOSA_OK) return rc;
  if (bad_ptr(k_prefix) || bad_ptr(page_meta)) return LOSA_ERR_INVALID_ARG;
  const size_t kbytes = static_cast<size_t>(d.S) * d.Hkv * d.L * kD * d.esz;
  if (overlaps(k_prefix, kbytes, page_meta, losa_page_meta_size(shape))) return LOSA_ERR_INVALID_ARG;
  dim3 grid((d.P + kMetaWarps - 1) / kMetaWarps, d.S * d.Hkv);
  if (grid.y > 65535u) return LOSA_ERR_UNSUPPORTED;
  meta_build_kernel<<<grid, kMetaWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      k_prefix, page_meta, d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
