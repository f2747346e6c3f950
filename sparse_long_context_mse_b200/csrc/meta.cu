// meta.cu -- page min/max metadata: the build (once per prefix) and prefix
// growth (a committed block appended, its pages' records rebuilt).
//
// QUEST's bound needs, per page and channel, the min and max key value over
// the page's tokens (LoSA paper, methodology: QUEST-style selection over KV
// pages).  One warp per page; lane l owns channels [4l, 4l+4).  Min/max are
// exact, so the records are bit-identical to any correct implementation.
// Each page also gets the norms of its kmin and kmax rows, rounded up: the
// scoring kernel bounds the error of its tensor-core sums with them.
#include "losa_common.cuh"

namespace losa {
namespace {

constexpr int kMetaWarps = 8;

// Min and max over n >= 1 tokens of channels [4 lane, 4 lane + 4) (key4(j):
// token j's four channels as floats), stored as page p's record of group sg.
template <typename Key4>
__device__ __forceinline__ void page_record(Key4 key4, int n, void* meta, int sg, int p,
                                            const Dims& d, int lane) {
  float4 lo = key4(0), hi = lo;
  for (int j = 1; j < n; ++j) {
    const float4 x = key4(j);
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
  // the norms of kmin and kmax, every operation rounded up (all terms are
  // non-negative, so each partial sum bounds the exact one from above)
  float sl = 0.f, sh = 0.f;
  sl = __fmaf_ru(lo.x, lo.x, sl);
  sl = __fmaf_ru(lo.y, lo.y, sl);
  sl = __fmaf_ru(lo.z, lo.z, sl);
  sl = __fmaf_ru(lo.w, lo.w, sl);
  sh = __fmaf_ru(hi.x, hi.x, sh);
  sh = __fmaf_ru(hi.y, hi.y, sh);
  sh = __fmaf_ru(hi.z, hi.z, sh);
  sh = __fmaf_ru(hi.w, hi.w, sh);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sl = __fadd_ru(sl, __shfl_xor_sync(0xffffffffu, sl, o));
    sh = __fadd_ru(sh, __shfl_xor_sync(0xffffffffu, sh, o));
  }
  if (lane == 0) {
    float2* nrm = reinterpret_cast<float2*>(static_cast<char*>(meta) + meta_norm_offset(d));
    nrm[static_cast<size_t>(sg) * meta_norm_stride(d) + p] = make_float2(__fsqrt_ru(sl), __fsqrt_ru(sh));
  }
  char* rec = static_cast<char*>(meta) + (static_cast<size_t>(sg) * d.Pc + p) * (2 * kD * d.esz);
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

__global__ void __launch_bounds__(kMetaWarps * 32)
    meta_build_kernel(const void* __restrict__ K, void* __restrict__ meta, Dims d) {
  const int sg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p = blockIdx.x * kMetaWarps + warp;
  const int L = seq_len(d, sg / d.Hkv);  // this sequence's prefix length
  if (p * kPS >= L) return;
  const int j0 = p * kPS;
  const size_t base = (static_cast<size_t>(sg) * d.Lc + j0) * kD + 4 * lane;
  page_record([&](int j) { return ld4(K, base + static_cast<size_t>(j) * kD, d.dtype); },
              min(kPS, L - j0), meta, sg, p, d, lane);
}

// Prefix growth: one warp per page touched by tokens L .. L+B-1 (pages
// L/ps .. (L+B-1)/ps, L the sequence's own length): the page's block tokens
// are copied into the prefix K and V (16-byte chunks), and its record is
// rebuilt over its tokens < L+B, each read from where it lives before the
// copy (old prefix below L, the block from L on), so no thread reads what
// another writes.
__global__ void __launch_bounds__(kMetaWarps * 32)
    append_kernel(const void* __restrict__ kb, const void* __restrict__ vb, void* __restrict__ K,
                  void* __restrict__ V, void* __restrict__ meta, Dims d) {
  const int sg = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = seq_len(d, sg / d.Hkv);
  const int p0 = L / kPS, np = (L + d.B - 1) / kPS - p0 + 1;
  const int i = blockIdx.x * kMetaWarps + warp;
  if (i >= np) return;
  const int p = p0 + i;
  const int L1 = L + d.B;
  const int j0 = p * kPS, j1 = min(j0 + kPS, L1);
  const size_t rowb = static_cast<size_t>(kD) * d.esz;
  const int c16 = static_cast<int>(rowb / 16);  // 16-byte chunks per token row
  const char* kbs = static_cast<const char*>(kb) + static_cast<size_t>(sg) * d.B * rowb;
  const char* vbs = static_cast<const char*>(vb) + static_cast<size_t>(sg) * d.B * rowb;
  char* Kd = static_cast<char*>(K) + static_cast<size_t>(sg) * d.Lc * rowb;
  char* Vd = static_cast<char*>(V) + static_cast<size_t>(sg) * d.Lc * rowb;
  const int jb = max(j0, L);
  for (int e = lane; e < (j1 - jb) * c16; e += 32) {
    const int j = jb + e / c16, c = e % c16;
    const size_t src = static_cast<size_t>(j - L) * rowb + 16 * c;
    const size_t dst = static_cast<size_t>(j) * rowb + 16 * c;
    *reinterpret_cast<uint4*>(Kd + dst) = *reinterpret_cast<const uint4*>(kbs + src);
    *reinterpret_cast<uint4*>(Vd + dst) = *reinterpret_cast<const uint4*>(vbs + src);
  }
  const size_t kbase = (static_cast<size_t>(sg) * d.Lc) * kD + 4 * lane;
  const size_t bbase = (static_cast<size_t>(sg) * d.B) * kD + 4 * lane;
  page_record(
      [&](int t) {
        const int j = j0 + t;
        return j < L ? ld4(K, kbase + static_cast<size_t>(j) * kD, d.dtype)
                     : ld4(kb, bbase + static_cast<size_t>(j - L) * kD, d.dtype);
      },
      j1 - j0, meta, sg, p, d, lane);
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
  const size_t kbytes = static_cast<size_t>(d.S) * d.Hkv * d.Lc * kD * d.esz;
  if (overlaps(k_prefix, kbytes, page_meta, losa_page_meta_size(shape))) return LOSA_ERR_INVALID_ARG;
  dim3 grid((d.P + kMetaWarps - 1) / kMetaWarps, d.S * d.Hkv);
  if (grid.y > 65535u) return LOSA_ERR_UNSUPPORTED;
  meta_build_kernel<<<grid, kMetaWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      k_prefix, page_meta, d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}

extern "C" int losa_append_block(const losa_shape* shape, const void* k_blk, const void* v_blk,
                                 void* k_prefix, void* v_prefix, void* page_meta, void* stream) {
  using namespace losa;
  Dims d;
  int rc = make_dims(shape, LOSA_WS_DENSE, &d);
  if (rc != LOSA_OK) return rc;
  if (bad_ptr(k_blk) || bad_ptr(v_blk) || bad_ptr(k_prefix) || bad_ptr(v_prefix) ||
      bad_ptr(page_meta))
    return LOSA_ERR_INVALID_ARG;
  if (static_cast<long long>(d.L) + d.B > d.Lc) return LOSA_ERR_INVALID_ARG;  // no room
  const size_t pb = static_cast<size_t>(d.S) * d.Hkv * d.Lc * kD * d.esz;
  const size_t bb = static_cast<size_t>(d.S) * d.Hkv * d.B * kD * d.esz;
  const size_t mb = losa_page_meta_size(shape);
  if (overlaps(k_prefix, pb, v_prefix, pb) || overlaps(k_prefix, pb, page_meta, mb) ||
      overlaps(v_prefix, pb, page_meta, mb) || overlaps(k_blk, bb, k_prefix, pb) ||
      overlaps(k_blk, bb, v_prefix, pb) || overlaps(v_blk, bb, k_prefix, pb) ||
      overlaps(v_blk, bb, v_prefix, pb) || overlaps(k_blk, bb, page_meta, mb) ||
      overlaps(v_blk, bb, page_meta, mb))
    return LOSA_ERR_INVALID_ARG;
  // pages touched: (L+B-1)/ps - L/ps + 1 <= (B-1)/ps + 2, whatever L is
  const int np = (d.B - 1) / kPS + 2;
  dim3 grid((np + kMetaWarps - 1) / kMetaWarps, d.S * d.Hkv);
  if (grid.y > 65535u) return LOSA_ERR_UNSUPPORTED;
  append_kernel<<<grid, kMetaWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      k_blk, v_blk, k_prefix, v_prefix, page_meta, d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
