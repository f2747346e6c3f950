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
#include "ptx.cuh"

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

__global__ void __launch_bounds__(256)
    dense_finish_kernel(const void* __restrict__ Q, const void* __restrict__ Kb,
                        const void* __restrict__ Vb, const float* __restrict__ part,
                        float* __restrict__ o_p, float* __restrict__ l_p, float* __restrict__ out,
                        float* __restrict__ out_lse, Dims d) {
  __shared__ __align__(16) float Ksb[kMaxB * kD];
  __shared__ __align__(16) float Vsb[kMaxB * kD];
  __shared__ float Ps[8][kPS];
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
  // one warp per row: rows blockIdx.y * 8 + warp of head h
  for (int t = blockIdx.y * 8 + warp; t < min(d.B, blockIdx.y * 8 + 8); t += 8) {
    const size_t row = static_cast<size_t>(sh) * d.B + t;
    const int r = (h - g * d.G) * d.B + t;
    // merge the prefix partials (base-2 units) of every split: the splits'
    // maxima over the lanes, then the weighted sums with eight splits' loads
    // in flight at a time
    const float* p0 = part + (static_cast<size_t>(sg) * d.nsplit * rows + r) * kPartStride;
    const size_t pstride = static_cast<size_t>(rows) * kPartStride;
    float M = -INFINITY;
    for (int sp = lane; sp < d.nsplit; sp += 32) M = fmaxf(M, __ldcg(p0 + sp * pstride));
    M = warp_max(M);
    float lsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int sp = 0; sp < d.nsplit; ++sp) {
      const float* src = p0 + sp * pstride;
      const float w = exp2f(__ldcg(src) - M);
      lsum += w * __ldcg(src + 1);
      const float4 a = __ldcg(reinterpret_cast<const float4*>(src + 4) + lane);
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

// ---------------------------------------------------------------------------
// bf16: tensor cores.  CTA = (split, group); warp w owns query rows
// [16w, 16w + 16) of the group's G*B rows.  Keys stream through a 3-stage
// cp.async ring of 64-key K/V tiles (16-byte chunks XOR-swizzled by row, so
// ldmatrix is conflict-free).  S = Q K^T and O += P V with mma.sync
// m16n8k16 (bf16 operands, fp32 accumulation); P is split into a bf16 high
// part and a bf16 remainder so the weights keep ~16 bits.  Online softmax in
// base 2, one partial (m, l, acc) per row and split, as the fp32 kernel.
// ---------------------------------------------------------------------------
constexpr int kDKeys = 64;
constexpr size_t kMaxDenseSmem = 128 * 256 + 3 * 2 * 64 * 128 * 2;
constexpr int kDStages = 3;
constexpr int kDTileBytes = kDKeys * kD * 2;

__global__ void __launch_bounds__(256) dense_mma_kernel(const __nv_bfloat16* __restrict__ Q,
                                                        const __nv_bfloat16* __restrict__ K,
                                                        const __nv_bfloat16* __restrict__ V,
                                                        float* __restrict__ part, Dims d) {
  extern __shared__ __align__(1024) char dsm[];
  const int sg = blockIdx.y, split = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int rows = d.G * d.B;
  const int M16 = (rows + 15) / 16 * 16;
  const int nthr = blockDim.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  char* qs = dsm;                 // [M16][256 B]
  char* kvs = dsm + M16 * 256;    // stages x (K tile, V tile)
  const int key0 = split * d.split_pages * kPS;
  const int key1 = min(d.L, key0 + d.split_pages * kPS);
  const int ntile = (key1 - key0 + kDKeys - 1) / kDKeys;
  const size_t kvbase = static_cast<size_t>(sg) * d.L * kD;
  const size_t qbase = (static_cast<size_t>(s) * d.Hq + g * d.G) * d.B * kD;

#pragma unroll 1
  for (int e = tid; e < M16 * 16; e += nthr) {
    const int r = e >> 4, c = e & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < rows) v = *reinterpret_cast<const uint4*>(Q + qbase + static_cast<size_t>(r) * kD + c * 8);
    *reinterpret_cast<uint4*>(qs + r * 256 + ((c ^ (r & 7)) << 4)) = v;
  }
  auto load_tile = [&](int t, int stage) {
    char* kt = kvs + stage * 2 * kDTileBytes;
    char* vt = kt + kDTileBytes;
    const int kb = key0 + t * kDKeys;
#pragma unroll 1
    for (int e = tid; e < kDKeys * 16; e += nthr) {
      const int j = e >> 4, c = e & 15;
      const int key = kb + j;
      const bool ok = key < key1;
      const size_t off = kvbase + static_cast<size_t>(ok ? key : key0) * kD + c * 8;
      const uint32_t o = j * 256 + ((c ^ (j & 7)) << 4);
      cp_async16(su32(kt + o), K + off, ok ? 16u : 0u);
      cp_async16(su32(vt + o), V + off, ok ? 16u : 0u);
    }
  };
#pragma unroll 1
  for (int st = 0; st < kDStages - 1; ++st) {
    if (st < ntile) load_tile(st, st);
    cp_async_commit();
  }
  __syncthreads();
  uint32_t qa[8][4];
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int mi = lane >> 3, row = warp * 16 + (mi & 1) * 8 + (lane & 7);
    const int ch = ks * 2 + (mi >> 1);
    ldsm_x4(su32(qs + row * 256 + ((ch ^ (row & 7)) << 4)), qa[ks][0], qa[ks][1], qa[ks][2],
            qa[ks][3]);
  }
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  const float sl2 = d.scale_log2;

#pragma unroll 1
  for (int t = 0; t < ntile; ++t) {
    cp_async_wait<kDStages - 2>();
    __syncthreads();
    {
      const int tn = t + kDStages - 1;
      if (tn < ntile) load_tile(tn, tn % kDStages);
      cp_async_commit();
    }
    const char* kt = kvs + (t % kDStages) * 2 * kDTileBytes;
    const char* vt = kt + kDTileBytes;
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        uint32_t b0, b1, b2, b3;
        const int key = nt * 8 + (lane & 7), ch = ks * 2 + (lane >> 3);
        ldsm_x4(su32(kt + key * 256 + ((ch ^ (key & 7)) << 4)), b0, b1, b2, b3);
        mma_bf16(sc[nt], qa[ks], b0, b1);
        mma_bf16(sc[nt], qa[ks + 1], b2, b3);
      }
    }
    const int kb = key0 + t * kDKeys;
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const bool ok = kb + nt * 8 + 2 * t4 + c < key1;
        sc[nt][c] = ok ? sc[nt][c] * sl2 : -INFINITY;
        sc[nt][2 + c] = ok ? sc[nt][2 + c] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, sc[nt][c]);
        mx1 = fmaxf(mx1, sc[nt][2 + c]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      sc[nt][0] = exp2f(sc[nt][0] - mn0);
      sc[nt][1] = exp2f(sc[nt][1] - mn0);
      sc[nt][2] = exp2f(sc[nt][2] - mn1);
      sc[nt][3] = exp2f(sc[nt][3] - mn1);
      ps0 += sc[nt][0] + sc[nt][1];
      ps1 += sc[nt][2] + sc[nt][3];
    }
    l0 = l0 * al0 + ps0;
    l1 = l1 * al1 + ps1;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      o[n][0] *= al0;
      o[n][1] *= al0;
      o[n][2] *= al1;
      o[n][3] *= al1;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      // P as the A operand: high bf16 part and the bf16 remainder
      uint32_t ah[4], al[4];
      const float* p0 = sc[2 * kk];
      const float* p1 = sc[2 * kk + 1];
      const float pv[8] = {p0[0], p0[1], p0[2], p0[3], p1[0], p1[1], p1[2], p1[3]};
      float rem[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float hi = __bfloat162float(__float2bfloat16_rn(pv[i]));
        rem[i] = pv[i] - hi;
      }
      ah[0] = pack_bf16x2(pv[0], pv[1]);
      ah[1] = pack_bf16x2(pv[2], pv[3]);
      ah[2] = pack_bf16x2(pv[4], pv[5]);
      ah[3] = pack_bf16x2(pv[6], pv[7]);
      al[0] = pack_bf16x2(rem[0], rem[1]);
      al[1] = pack_bf16x2(rem[2], rem[3]);
      al[2] = pack_bf16x2(rem[4], rem[5]);
      al[3] = pack_bf16x2(rem[6], rem[7]);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = 16 * kk + ((lane >> 3) & 1) * 8 + (lane & 7);
        const int ch = 2 * np + (lane >> 4);
        ldsm_x4_trans(su32(vt + key * 256 + ((ch ^ (key & 7)) << 4)), b0, b1, b2, b3);
        mma_bf16(o[2 * np], ah, b0, b1);
        mma_bf16(o[2 * np + 1], ah, b2, b3);
        mma_bf16(o[2 * np], al, b0, b1);
        mma_bf16(o[2 * np + 1], al, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const int r0 = warp * 16 + g4, r1 = r0 + 8;
  const size_t pb = (static_cast<size_t>(sg) * d.nsplit + split) * rows;
  if (r0 < rows) {
    float* dst = part + (pb + r0) * kPartStride;
    if (t4 == 0) {
      dst[0] = m0;
      dst[1] = l0;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(dst + 4 + n * 8 + 2 * t4) = make_float2(o[n][0], o[n][1]);
  }
  if (r1 < rows) {
    float* dst = part + (pb + r1) * kPartStride;
    if (t4 == 0) {
      dst[0] = m1;
      dst[1] = l1;
    }
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(dst + 4 + n * 8 + 2 * t4) = make_float2(o[n][2], o[n][3]);
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
  if (d.dtype == LOSA_BF16) {
    const int M16 = (d.G * d.B + 15) / 16 * 16;
    const size_t smem = static_cast<size_t>(M16) * 256 + kDStages * 2 * kDTileBytes;
    static bool attr_done[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < kMaxDevices && !attr_done[dev]) {
      cudaError_t e0 = cudaFuncSetAttribute(dense_mma_kernel,
                                            cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            static_cast<int>(kMaxDenseSmem));
      if (e0 != cudaSuccess) return record_cuda_error(e0);
      attr_done[dev] = true;
    }
    dense_mma_kernel<<<dim3(d.nsplit, d.S * d.Hkv), 32 * (M16 / 16), smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k_prefix),
        static_cast<const __nv_bfloat16*>(v_prefix), part, d);
  } else {
    dense_partial_kernel<<<dim3(d.nsplit, d.S * d.Hkv), kDenseWarps * 32, 0, st>>>(
        q, k_prefix, v_prefix, part, d);
  }
  dense_finish_kernel<<<dim3(d.S * d.Hq, (d.B + 7) / 8), 256, 0, st>>>(q, k_blk, v_blk, part, o_p,
                                                                        l_p, out, out_lse, d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
