// step.cu -- one LoSA denoising step (LoSA paper, methodology).
//
//   active_kernel   locality score (MSE of Q_t vs Q_{t-1}) and top-|A| per
//                   query head
//   score_kernel    QUEST bound of every page of a chunk for the active rows
//                   of one KV group; chunk-local top-k per row
//   select_kernel   merge of the chunk candidates into each row's top-k,
//                   union of the group's pages with a row mask per page
//   gather_kernel   one warp per union page: load K/V once, online-softmax
//                   partial for every row whose mask holds the page
//   finish_kernel   per query head: dense suffix over the block, split merge
//                   for active rows (cache write-back), reuse for stable rows,
//                   log-sum-exp merge, output
#include <mutex>

#include "losa_common.cuh"

namespace losa {
namespace {

// ---------------------------------------------------------------------------
// 1. locality + active set.  One CTA per (sequence, query head).
// mse in fp32 with one rounding per operation and channels summed in order
// (the order the selection is defined in), so the active set is exact.
// ---------------------------------------------------------------------------
constexpr int kQPad = kD + 1;  // padded row: thread t walks row t conflict-free

__global__ void __launch_bounds__(128)
    active_kernel(const void* __restrict__ Qc, const void* __restrict__ Qp,
                  int32_t* __restrict__ act_tok, int32_t* __restrict__ act_slot,
                  int32_t* __restrict__ active_idx_out, Dims d) {
  __shared__ float qc[kMaxB * kQPad];
  __shared__ float qp[kMaxB * kQPad];
  __shared__ float mse[kMaxB];
  const int sh = blockIdx.x;
  const size_t q0 = static_cast<size_t>(sh) * d.B * kD;
  for (int e = threadIdx.x; e < d.B * kD / 4; e += blockDim.x) {
    const int t = e / (kD / 4), c = (e % (kD / 4)) * 4;
    const float4 a = ld4(Qc, q0 + static_cast<size_t>(t) * kD + c, d.dtype);
    const float4 b = ld4(Qp, q0 + static_cast<size_t>(t) * kD + c, d.dtype);
    float* x = qc + t * kQPad + c;
    float* y = qp + t * kQPad + c;
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    y[0] = b.x; y[1] = b.y; y[2] = b.z; y[3] = b.w;
  }
  __syncthreads();
  const int t = threadIdx.x;
  if (t < d.B) {
    float acc = 0.f;
    for (int i = 0; i < kD; ++i) {
      const float delta = __fsub_rn(qc[t * kQPad + i], qp[t * kQPad + i]);
      acc = __fadd_rn(acc, __fmul_rn(delta, delta));
    }
    mse[t] = __fdiv_rn(acc, static_cast<float>(kD));
  }
  __syncthreads();
  if (t < 32) {
    int slot = -1;
    bool is_active = false;
    if (t < d.B) {
      const float x = mse[t];
      int rank = 0;
      for (int u = 0; u < d.B; ++u) {
        const float y = mse[u];
        rank += (y > x) || (y == x && u < t);
      }
      is_active = rank < d.A;
    }
    const unsigned mask = __ballot_sync(0xffffffffu, is_active);
    if (is_active) slot = __popc(mask & ((1u << t) - 1u));
    if (t < d.B) act_slot[static_cast<size_t>(sh) * d.B + t] = slot;
    if (is_active) {
      act_tok[static_cast<size_t>(sh) * d.A + slot] = t;
      if (active_idx_out) active_idx_out[static_cast<size_t>(sh) * d.A + slot] = t;
    }
  }
}

// ---------------------------------------------------------------------------
// 2. bound scoring.  CTA = (chunk of pages, (s, g)); thread = page.
// U = sum_i max(q_i*kmax_i, q_i*kmin_i) in fp32, channels in order, with
// explicit round-to-nearest multiplies and adds (no contraction): the exact
// arithmetic the selection is defined in.
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 128;  // == chunk_pages

__device__ __forceinline__ void load_meta_chunk(const char* rec, int page, uint32_t lbyte,
                                                int dtype, float* out8, int& n) {
  // returns the channels held by one 16-byte logical chunk: 8 (bf16) or 4 (f32)
  const uint4 raw = *reinterpret_cast<const uint4*>(rec + meta_swz(lbyte, page));
  if (dtype == LOSA_BF16) {
    out8[0] = __uint_as_float(raw.x << 16);
    out8[1] = __uint_as_float(raw.x & 0xffff0000u);
    out8[2] = __uint_as_float(raw.y << 16);
    out8[3] = __uint_as_float(raw.y & 0xffff0000u);
    out8[4] = __uint_as_float(raw.z << 16);
    out8[5] = __uint_as_float(raw.z & 0xffff0000u);
    out8[6] = __uint_as_float(raw.w << 16);
    out8[7] = __uint_as_float(raw.w & 0xffff0000u);
    n = 8;
  } else {
    out8[0] = __uint_as_float(raw.x);
    out8[1] = __uint_as_float(raw.y);
    out8[2] = __uint_as_float(raw.z);
    out8[3] = __uint_as_float(raw.w);
    n = 4;
  }
}

__global__ void __launch_bounds__(kScoreThreads)
    score_kernel(const void* __restrict__ Qc, const void* __restrict__ meta,
                 const int32_t* __restrict__ act_tok, unsigned long long* __restrict__ cand,
                 Dims d) {
  extern __shared__ __align__(16) float sm[];
  float* qs = sm;                       // [R][kD]
  float* sc = sm + d.R * kD;            // [R][kScoreThreads]
  const int sg = blockIdx.y, chunk = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int tid = threadIdx.x;
  for (int e = tid; e < d.R * kD / 4; e += blockDim.x) {
    const int r = e / (kD / 4), c = (e % (kD / 4)) * 4;
    const int h = g * d.G + r / d.A, a = r % d.A;
    const int t = act_tok[(static_cast<size_t>(s) * d.Hq + h) * d.A + a];
    const float4 v = ld4(Qc, ((static_cast<size_t>(s) * d.Hq + h) * d.B + t) * kD + c, d.dtype);
    *reinterpret_cast<float4*>(qs + r * kD + c) = v;
  }
  __syncthreads();
  const int p = chunk * kScoreThreads + tid;
  if (p < d.P) {
    const char* rec = static_cast<const char*>(meta) +
                      (static_cast<size_t>(sg) * d.P + p) * (2 * kD * d.esz);
    const uint32_t half = kD * d.esz;  // bytes of the kmin row
    for (int r = 0; r < d.R; ++r) {
      float acc = 0.f;
      for (uint32_t b = 0; b < half; b += 16) {
        float mn[8], mx[8];
        int n;
        load_meta_chunk(rec, p, b, d.dtype, mn, n);
        load_meta_chunk(rec, p, half + b, d.dtype, mx, n);
        const int i0 = b / d.esz;
        for (int j = 0; j < n; ++j) {
          const float q = qs[r * kD + i0 + j];
          const float hi = __fmul_rn(q, mx[j]);
          const float lo = __fmul_rn(q, mn[j]);
          acc = __fadd_rn(acc, fmaxf(hi, lo));
        }
      }
      sc[r * kScoreThreads + tid] = acc;
    }
  }
  __syncthreads();
  // chunk-local top-k per row: warp per row, k rounds of warp argmax
  const int warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int kc = d.k;
  for (int r = warp; r < d.R; r += nw) {
    unsigned long long key[kScoreThreads / 32];
#pragma unroll
    for (int i = 0; i < kScoreThreads / 32; ++i) {
      const int pl = i * 32 + lane;
      const int pp = chunk * kScoreThreads + pl;
      key[i] = pp < d.P ? sel_key(sc[r * kScoreThreads + pl], pp) : 0ull;
    }
    unsigned long long* dst = cand + ((static_cast<size_t>(sg) * d.nchunk + chunk) * d.R + r) * kc;
    for (int j = 0; j < kc; ++j) {
      unsigned long long best = 0;
#pragma unroll
      for (int i = 0; i < kScoreThreads / 32; ++i) best = key[i] > best ? key[i] : best;
      best = warp_max_u64(best);
#pragma unroll
      for (int i = 0; i < kScoreThreads / 32; ++i)
        if (key[i] == best) key[i] = 0;
      if (lane == 0) dst[j] = best;
    }
  }
}

// ---------------------------------------------------------------------------
// 3. selection merge + union.  One CTA per (s, g).
// ---------------------------------------------------------------------------
constexpr int kSelectThreads = 256;

__global__ void __launch_bounds__(kSelectThreads)
    select_kernel(const unsigned long long* __restrict__ cand, int32_t* __restrict__ sel,
                  int32_t* __restrict__ uni, uint32_t* __restrict__ umask,
                  int32_t* __restrict__ ucount, int32_t* __restrict__ page_idx_out,
                  int32_t* __restrict__ union_count_out, Dims d, void* status) {
  extern __shared__ __align__(16) uint32_t smu[];
  const int nwords = (d.P + 31) / 32;
  uint32_t* bitmap = smu;             // [nwords]
  uint32_t* wbase = smu + nwords;     // [nwords] exclusive prefix of popcounts
  __shared__ int32_t picked[kMaxK * 8];  // per-warp scratch (k <= 64, 8 warps)
  __shared__ int32_t s_total;
  const int sg = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nw = blockDim.x >> 5;
  const int k = d.k;
  int32_t* selg = sel + static_cast<size_t>(sg) * d.R * k;

  // (a) each row's top-k pages, ascending
  for (int r = warp; r < d.R; r += nw) {
    int32_t* pk = picked + warp * kMaxK;
    if (d.all_pages) {
      for (int j = lane; j < k; j += 32) selg[static_cast<size_t>(r) * k + j] = j;
      continue;
    }
    const int ncand = d.nchunk * k;
    const unsigned long long* cr = cand + static_cast<size_t>(sg) * d.nchunk * d.R * k;
    // candidate c of row r: chunk c / k, slot c % k
    for (int j = 0; j < k; ++j) {
      unsigned long long best = 0;
      for (int c = lane; c < ncand; c += 32) {
        const unsigned long long x =
            cr[(static_cast<size_t>(c / k) * d.R + r) * k + (c % k)];
        bool taken = false;
        for (int u = 0; u < j; ++u) taken |= (key_index(x) == pk[u]);
        if (!taken && x > best) best = x;
      }
      best = warp_max_u64(best);
      if (lane == 0) pk[j] = best ? key_index(best) : -1;
      __syncwarp();
    }
    // ascending order by rank
    for (int j = lane; j < k; j += 32) {
      const int x = pk[j];
      int rank = 0;
      for (int u = 0; u < k; ++u) rank += pk[u] < x;
      if (x < 0 || x >= d.P) set_status(status, LOSA_ERR_DEVICE_BOUNDS);
      selg[static_cast<size_t>(r) * k + rank] = x;
    }
    __syncwarp();
  }
  // (b) union bitmap
  for (int w = tid; w < nwords; w += blockDim.x) bitmap[w] = 0;
  __syncthreads();
  for (int e = tid; e < d.R * k; e += blockDim.x) {
    const int p = selg[e];
    if (p >= 0 && p < d.P) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < nwords; ++w) {
      wbase[w] = run;
      run += __popc(bitmap[w]);
    }
    s_total = run;
  }
  __syncthreads();
  const int U = s_total;
  int32_t* ug = uni + static_cast<size_t>(sg) * d.Umax;
  uint32_t* mg = umask + static_cast<size_t>(sg) * d.Umax * d.MW;
  for (int w = tid; w < nwords; w += blockDim.x) {
    uint32_t bits = bitmap[w];
    int pos = wbase[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < d.Umax) ug[pos] = w * 32 + b;
      ++pos;
    }
  }
  for (int e = tid; e < U * d.MW; e += blockDim.x) mg[e] = 0;
  __syncthreads();
  for (int e = tid; e < d.R * k; e += blockDim.x) {
    const int r = e / k, p = selg[e];
    if (p < 0 || p >= d.P) continue;
    const int w = p >> 5;
    const int u = wbase[w] + __popc(bitmap[w] & ((1u << (p & 31)) - 1u));
    if (u < d.Umax) atomicOr(&mg[static_cast<size_t>(u) * d.MW + (r >> 5)], 1u << (r & 31));
    else set_status(status, LOSA_ERR_DEVICE_BOUNDS);
  }
  if (tid == 0) {
    ucount[sg] = U;
    if (union_count_out) union_count_out[sg] = U;
  }
  if (page_idx_out)
    for (int e = tid; e < d.R * k; e += blockDim.x)
      page_idx_out[static_cast<size_t>(sg) * d.R * k + e] = selg[e];
}

// ---------------------------------------------------------------------------
// 4. union gather.  One warp per union page; K/V of the page are read once and
// serve every active row of the group whose mask holds the page.
// ---------------------------------------------------------------------------
constexpr int kGatherWarps = 4;

__global__ void __launch_bounds__(kGatherWarps * 32)
    gather_kernel(const void* __restrict__ Qc, const void* __restrict__ K,
                  const void* __restrict__ V, const int32_t* __restrict__ act_tok,
                  const int32_t* __restrict__ sel, const int32_t* __restrict__ uni,
                  const uint32_t* __restrict__ umask, const int32_t* __restrict__ ucount,
                  float* __restrict__ part, Dims d, void* status) {
  extern __shared__ __align__(16) float smg[];
  __shared__ float Ps[kGatherWarps][kPS];
  const int sg = blockIdx.x;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.y * kGatherWarps + warp;
  if (u >= ucount[sg]) return;
  float* Ks = smg + warp * (2 * kPS * kD);
  float* Vs = Ks + kPS * kD;
  const int p = uni[static_cast<size_t>(sg) * d.Umax + u];
  if (p < 0 || p >= d.P) {
    set_status(status, LOSA_ERR_DEVICE_BOUNDS);
    return;
  }
  const int ntok = min(kPS, d.L - p * kPS);
  const size_t kv0 = (static_cast<size_t>(sg) * d.L + static_cast<size_t>(p) * kPS) * kD;
  for (int j = 0; j < kPS; ++j) {
    float4 kv = make_float4(0.f, 0.f, 0.f, 0.f), vv = kv;
    if (j < ntok) {
      kv = ld4(K, kv0 + static_cast<size_t>(j) * kD + 4 * lane, d.dtype);
      vv = ld4(V, kv0 + static_cast<size_t>(j) * kD + 4 * lane, d.dtype);
    }
    *reinterpret_cast<float4*>(Ks + j * kD + 4 * lane) = kv;
    *reinterpret_cast<float4*>(Vs + j * kD + 4 * lane) = vv;
  }
  __syncwarp();
  const uint32_t* mk = umask + (static_cast<size_t>(sg) * d.Umax + u) * d.MW;
  const int32_t* selg = sel + static_cast<size_t>(sg) * d.R * d.k;
  for (int w = 0; w < d.MW; ++w) {
    uint32_t bits = mk[w];
    while (bits) {
      const int r = w * 32 + __ffs(bits) - 1;
      bits &= bits - 1;
      const int h = g * d.G + r / d.A, a = r % d.A;
      const int t = act_tok[(static_cast<size_t>(s) * d.Hq + h) * d.A + a];
      const float4 q = ld4(Qc, ((static_cast<size_t>(s) * d.Hq + h) * d.B + t) * kD + 4 * lane,
                           d.dtype);
      float m = -INFINITY, l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      attend_page_row(q, Ks, Vs, ntok, d.scale_log2, m, l, acc, Ps[warp]);
      // slot of page p in row r's ascending list
      const int32_t* lst = selg + static_cast<size_t>(r) * d.k;
      int lo = 0, hi = d.k;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (lst[mid] < p) lo = mid + 1; else hi = mid;
      }
      if (lo >= d.k || lst[lo] != p) {
        set_status(status, LOSA_ERR_DEVICE_BOUNDS);
        continue;
      }
      float* dst = part + ((static_cast<size_t>(sg) * d.R + r) * d.k + lo) * kPartStride;
      if (lane == 0) {
        dst[0] = m;
        dst[1] = l;
      }
      *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// 5. finish.  One CTA per (s, h): suffix for every token, split merge and cache
// write-back for active tokens, cached state for stable tokens, LSE merge.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void suffix_row_s(float4 q, const float* Kb, const float* Vb, int B,
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
    finish_kernel(const void* __restrict__ Qc, const void* __restrict__ Kb,
                  const void* __restrict__ Vb, const int32_t* __restrict__ act_slot,
                  const float* __restrict__ part, float* __restrict__ o_p,
                  float* __restrict__ l_p, float* __restrict__ out, float* __restrict__ out_lse,
                  Dims d) {
  __shared__ __align__(16) float Ksb[kMaxB * kD];
  __shared__ __align__(16) float Vsb[kMaxB * kD];
  __shared__ float Ps[4][kPS];
  const int sh = blockIdx.x;
  const int s = sh / d.Hq, h = sh % d.Hq, g = h / d.G;
  const int sg = s * d.Hkv + g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    const int a = act_slot[row];
    float4 op;
    float Lp;
    if (a >= 0) {
      const int r = (h - g * d.G) * d.A + a;
      const float* src0 = part + (static_cast<size_t>(sg) * d.R + r) * d.k * kPartStride;
      float M = -INFINITY;
      for (int j = 0; j < d.k; ++j) M = fmaxf(M, src0[static_cast<size_t>(j) * kPartStride]);
      float lsum = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < d.k; ++j) {
        const float* src = src0 + static_cast<size_t>(j) * kPartStride;
        const float w = exp2f(src[0] - M);
        lsum += w * src[1];
        const float4 x = *reinterpret_cast<const float4*>(src + 4 + 4 * lane);
        acc.x += w * x.x;
        acc.y += w * x.y;
        acc.z += w * x.z;
        acc.w += w * x.w;
      }
      const float inv = 1.f / lsum;
      op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      Lp = (M + __log2f(lsum)) * kLn2;
      *reinterpret_cast<float4*>(o_p + row * kD + 4 * lane) = op;
      if (lane == 0) l_p[row] = Lp;
    } else {
      op = *reinterpret_cast<const float4*>(o_p + row * kD + 4 * lane);
      Lp = l_p[row];
    }
    const float4 q = ld4(Qc, row * kD + 4 * lane, d.dtype);
    float4 os;
    float Ls;
    suffix_row_s(q, Ksb, Vsb, d.B, d.scale_log2, Ps[warp], os, Ls);
    float4 o;
    float L;
    lse_merge(op, Lp, os, Ls, o, L);
    *reinterpret_cast<float4*>(out + row * kD + 4 * lane) = o;
    if (out_lse && lane == 0) out_lse[row] = L;
  }
}

// Raises the dynamic shared-memory limit of the kernels that need more than
// 48 KB, once per device (the first call on a device should come before any
// stream capture).
int g_max_dyn[kMaxDevices] = {};  // smallest dynamic-smem limit granted, per device

int set_kernel_attributes(size_t* max_dyn) {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return LOSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) {
    *max_dyn = static_cast<size_t>(g_max_dyn[dev]);
    return LOSA_OK;
  }
  const void* fns[] = {reinterpret_cast<const void*>(score_kernel),
                       reinterpret_cast<const void*>(select_kernel),
                       reinterpret_cast<const void*>(gather_kernel)};
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  for (const void* f : fns) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, f);
    if (e != cudaSuccess) return record_cuda_error(e);
    const int dyn = optin - static_cast<int>(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
    if (e != cudaSuccess) return record_cuda_error(e);
    g_max_dyn[dev] = dyn < g_max_dyn[dev] || g_max_dyn[dev] == 0 ? dyn : g_max_dyn[dev];
  }
  done[dev] = true;
  *max_dyn = static_cast<size_t>(g_max_dyn[dev]);
  return LOSA_OK;
}

}  // namespace
}  // namespace losa

extern "C" int losa_step(const losa_shape* shape, const void* q_cur, const void* q_prev,
                         const void* k_prefix, const void* v_prefix, const void* page_meta,
                         const void* k_blk, const void* v_blk, float* o_p, float* l_p,
                         float* out, float* out_lse, int32_t* active_idx, int32_t* page_idx,
                         int32_t* union_count, void* workspace, size_t ws_bytes, void* stream) {
  using namespace losa;
  Dims d;
  int rc = make_dims(shape, LOSA_WS_STEP, &d);
  if (rc != LOSA_OK) return rc;
  if (bad_ptr(q_cur) || bad_ptr(q_prev) || bad_ptr(k_prefix) || bad_ptr(v_prefix) ||
      bad_ptr(page_meta) || bad_ptr(k_blk) || bad_ptr(v_blk) || bad_ptr(o_p) || bad_ptr(l_p) ||
      bad_ptr(out) || bad_opt_ptr(out_lse) || bad_opt_ptr(active_idx) ||
      bad_opt_ptr(page_idx) || bad_opt_ptr(union_count) || !workspace ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return LOSA_ERR_INVALID_ARG;
  if (ws_bytes < d.total) return LOSA_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(d.S) * d.Hq * d.B;
  const size_t ob = rows * kD * sizeof(float), qb = rows * kD * d.esz;
  if (overlaps(out, ob, q_cur, qb) || overlaps(out, ob, q_prev, qb) || overlaps(out, ob, o_p, ob) ||
      overlaps(out, ob, l_p, rows * sizeof(float)))
    return LOSA_ERR_INVALID_ARG;
  if (d.S * d.Hkv > 65535 || d.nchunk > 65535) return LOSA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  void* status = ws + d.off_status;
  int32_t* act_tok = reinterpret_cast<int32_t*>(ws + d.off_act_tok);
  int32_t* act_slot = reinterpret_cast<int32_t*>(ws + d.off_act_slot);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(ws + d.off_cand);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + d.off_sel);
  int32_t* uni = reinterpret_cast<int32_t*>(ws + d.off_union);
  uint32_t* umask = reinterpret_cast<uint32_t*>(ws + d.off_mask);
  int32_t* ucount = reinterpret_cast<int32_t*>(ws + d.off_ucount);
  float* part = reinterpret_cast<float*>(ws + d.off_part);

  size_t max_dyn = 0;
  rc = set_kernel_attributes(&max_dyn);
  if (rc != LOSA_OK) return rc;
  // every limit is checked before the first launch
  const size_t smem_score = static_cast<size_t>(d.R) * (kD + kScoreThreads) * sizeof(float);
  const size_t smem_sel = 2 * static_cast<size_t>((d.P + 31) / 32) * sizeof(uint32_t);
  const size_t smem_g = static_cast<size_t>(kGatherWarps) * 2 * kPS * kD * sizeof(float);
  const int ublocks = (d.Umax + kGatherWarps - 1) / kGatherWarps;
  if (smem_score > max_dyn || smem_sel > max_dyn || smem_g > max_dyn || ublocks > 65535)
    return LOSA_ERR_UNSUPPORTED;

  active_kernel<<<d.S * d.Hq, 128, 0, st>>>(q_cur, q_prev, act_tok, act_slot, active_idx, d);
  if (d.A > 0) {
    if (!d.all_pages)
      score_kernel<<<dim3(d.nchunk, d.S * d.Hkv), kScoreThreads, smem_score, st>>>(
          q_cur, page_meta, act_tok, cand, d);
    select_kernel<<<d.S * d.Hkv, kSelectThreads, smem_sel, st>>>(
        cand, sel, uni, umask, ucount, page_idx, union_count, d, status);
    gather_kernel<<<dim3(d.S * d.Hkv, ublocks), kGatherWarps * 32, smem_g, st>>>(
        q_cur, k_prefix, v_prefix, act_tok, sel, uni, umask, ucount, part, d, status);
  } else if (union_count) {
    cudaMemsetAsync(union_count, 0, static_cast<size_t>(d.S) * d.Hkv * sizeof(int32_t), st);
  }
  finish_kernel<<<d.S * d.Hq, 128, 0, st>>>(q_cur, k_blk, v_blk, act_slot, part, o_p, l_p, out,
                                            out_lse, d);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}
