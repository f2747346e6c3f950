// step_fused.cu -- one LoSA denoising step as a single kernel launch.
//
// LoSA paper, methodology: locality pruning (MSE of Q_t vs Q_{t-1}, top-|A|
// per head), reuse of the cached prefix state for stable tokens, QUEST page
// selection for active queries only, union of the selected pages, sparse
// prefix attention, dense intra-block suffix, online-softmax merge, cache
// update.
//
// One thread-block cluster of CL CTAs serves one (sequence, KV head) group;
// CTA `rank` of the cluster owns pages [rank*chunk, (rank+1)*chunk) of the
// group's prefix.  Phases (one CTA's view):
//
//   P0  issue bulk (TMA) copies of this CTA's page-metadata chunk into a
//       shared-memory ring; meanwhile compute the group's active set (every
//       CTA computes it, identically), the suffix of the stable rows this CTA
//       owns (written out at once) and of its active rows (kept in smem);
//   P1  QUEST bound of every page of the chunk for the group's R active rows:
//       bf16 -- tensor cores, U = [q-|q+] . [kmin;kmax] (mma.sync m16n8k16,
//       exact products, fp32 accumulation); fp32 -- CUDA cores, the sum in
//       channel order with one rounding per operation;
//   P2  chunk-local top-k per row (selection keys: score, then lower page);
//   --  cluster barrier
//   P3  rows are dealt to CTAs (r % CL); each merges its rows' CL candidate
//       lists through distributed shared memory into the row's top-k pages;
//   --  cluster barrier
//   P4  every CTA reads all rows' page lists, builds the group's union
//       (bitmap, ascending) and the row mask of each union page; union slot u
//       belongs to CTA u % CL;
//   P5  each CTA bulk-copies its union pages' K and V (each page read once
//       for the whole GQA group) and writes an online-softmax partial
//       (m, l, acc) for every row whose mask holds the page;
//   --  cluster barrier
//   P6  each CTA combines the partials of its active rows, writes their new
//       o_p / L_p to the cache and merges them with their suffix.
//
// Every wait on a bulk copy is bounded (clock64); a wait that gives up sets
// LOSA_ERR_DEVICE_TIMEOUT in the status word and the CTA keeps going through
// every cluster barrier without doing further work, so the cluster never
// deadlocks.  There is no other cross-CTA wait.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "losa_common.cuh"

namespace cg = cooperative_groups;

namespace losa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRingBytes = 128 * 1024;
constexpr int kStageBytes = 32 * 1024;
constexpr int kMaxStages = kMaxRingBytes / kStageBytes;
constexpr int kCandCap = 64;                     // per-warp compaction buffer
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 2 GHz
constexpr int kMaxCluster = 16;

struct Layout {  // dynamic shared-memory byte offsets
  int ring, scores, qrows, kbv, cand, sel_own, sel_all, bitmap, wbase, lpages, masks, sfx, cbuf,
      ps, misc, mbar, total;
};

struct Params {
  const void* qc;
  const void* qp;
  const void* K;
  const void* V;
  const char* meta;
  const void* kb;
  const void* vb;
  float* o_p;
  float* l_p;
  float* out;
  float* out_lse;
  int32_t* active_idx;
  int32_t* page_idx;
  int32_t* union_count;
  float* part;
  int* status;
  Dims d;
  int CL;           // CTAs per cluster (per group)
  int chunk;        // pages per CTA (multiple of 8)
  int tile;         // pages per ring stage
  int rec;          // bytes per metadata record
  int sc_stride;    // floats per score row
  int stages;       // metadata ring stages (ring = stages * 32 KiB)
  int gslots;       // gather slots per gathering warp
  int gwarps;       // warps that gather union pages
  int max_lp;       // max union pages per CTA
  Layout lo;
};

// ---------------------------------------------------------------------------
// PTX wrappers: mbarrier, bulk copy, ldmatrix, mma
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(bar)),
               "r"(bytes)
               : "memory");
}
// Non-multicast bulk copy global -> this CTA's shared memory.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(su32(dst)),
      "l"(src), "r"(bytes), "r"(su32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for phase `parity` of `bar`; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

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

// ---------------------------------------------------------------------------
// Warp top-k over n selection keys key(i), i in [0, n): writes the k largest
// keys, descending, to out[0..k) (0 = empty slot when n < k).  Fast path:
// threshold = k-th largest of the lanes' local maxima (a lower bound of the
// true k-th largest), compaction of the keys at or above it, rank sort.
// Fallback (k > 32 or too many survivors): k rounds of warp argmax.
// ---------------------------------------------------------------------------
template <typename KeyFn>
__device__ void warp_topk(KeyFn key, int n, int k, unsigned long long* out,
                          unsigned long long* cbuf) {
  const int lane = threadIdx.x & 31;
  unsigned long long lmax = 0;
  for (int i = lane; i < n; i += 32) lmax = umax64(lmax, key(i));
  bool done = false;
  if (k <= 32) {
    // bitonic sort of the 32 local maxima, descending (lane 0 largest)
    unsigned long long v = lmax;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
        const bool dir = (lane & size) == 0;
        const bool lower = (lane & stride) == 0;
        v = (lower == dir) ? umax64(v, o) : (v < o ? v : o);
      }
    }
    const unsigned long long tau = __shfl_sync(0xffffffffu, v, k - 1);
    int cnt = 0;
    for (int i = lane; i < n; i += 32) cnt += key(i) >= tau && key(i) != 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= kCandCap) {
      int pos = incl - cnt;
      for (int i = lane; i < n; i += 32) {
        const unsigned long long x = key(i);
        if (x >= tau && x != 0) cbuf[pos++] = x;
      }
      __syncwarp();
      for (int j = lane; j < total; j += 32) {
        const unsigned long long x = cbuf[j];
        int rank = 0;
        for (int m = 0; m < total; ++m) rank += cbuf[m] > x;
        if (rank < k) out[rank] = x;
      }
      for (int j = total + lane; j < k; j += 32) out[j] = 0;
      __syncwarp();
      done = true;
    }
  }
  if (!done) {
    unsigned long long last = ~0ull;
    for (int j = 0; j < k; ++j) {
      unsigned long long best = 0;
      for (int i = lane; i < n; i += 32) {
        const unsigned long long x = key(i);
        if (x < last && x > best) best = x;
      }
      best = warp_max_u64(best);
      if (lane == 0) out[j] = best;
      last = best ? best : 1ull;  // once empty, stay empty
    }
    __syncwarp();
  }
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int DT>
__global__ void __launch_bounds__(kThreads, 1) losa_step_kernel(const Params prm) {
  extern __shared__ __align__(1024) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const Dims& d = prm.d;
  const Layout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster.block_rank());
  const int CL = prm.CL;
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int esz = DT == LOSA_BF16 ? 2 : 4;

  char* ring = smem + lo.ring;
  float* sc = reinterpret_cast<float*>(smem + lo.scores);
  char* qrows = smem + lo.qrows;
  char* kbv = smem + lo.scores;  // [Bpad][kD] K then V, element type (aliases sc)
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + lo.cand);
  int32_t* sel_own = reinterpret_cast<int32_t*>(smem + lo.sel_own);
  int32_t* sel_all = reinterpret_cast<int32_t*>(smem + lo.sel_all);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + lo.bitmap);
  int32_t* wbase = reinterpret_cast<int32_t*>(smem + lo.wbase);
  int32_t* lpages = reinterpret_cast<int32_t*>(smem + lo.lpages);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + lo.masks);
  float* sfx = reinterpret_cast<float*>(smem + lo.sfx);
  unsigned long long* cbuf = reinterpret_cast<unsigned long long*>(smem + lo.cbuf);
  float* Ps = reinterpret_cast<float*>(smem + lo.ps);
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  // misc: [0] failed flag, [1] union size, [2] local pages, [3..3+kMaxB*? ) act
  int32_t* s_fail = misc;
  int32_t* s_U = misc + 1;
  int32_t* s_nlp = misc + 2;
  float* s_mse = reinterpret_cast<float*>(misc + 4);   // [G*B]
  int32_t* act_slot = misc + 4 + kMaxRowsPerGroup;     // [G*B] slot or -1
  int32_t* act_tok = act_slot + kMaxRowsPerGroup;      // [G][A] -> [R]

  const int p0 = rank * prm.chunk;
  const int npages = max(0, min(d.P, p0 + prm.chunk) - p0);
  const int ntiles = (npages + prm.tile - 1) / prm.tile;
  const bool scan = A > 0 && !d.all_pages;
  const char* meta_g = prm.meta + static_cast<size_t>(sg) * d.P * prm.rec;

  // ---- P0: barriers, first metadata copies --------------------------------
  if (tid == 0) {
    for (int i = 0; i < kMaxStages + kWarps * 2; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
    *s_fail = 0;
  }
  __syncthreads();
  if (tid == 0 && scan) {
    for (int t = 0; t < min(ntiles, prm.stages); ++t) {
      const int np = min(prm.tile, npages - t * prm.tile);
      const uint32_t bytes = static_cast<uint32_t>(np * prm.rec);
      mbar_expect_tx(&mbar[t], bytes);
      bulk_g2s(ring + t * kStageBytes, meta_g + static_cast<size_t>(p0 + t * prm.tile) * prm.rec,
               bytes, &mbar[t]);
    }
  }

  // ---- P0: locality score and active set (every CTA, identical) -----------
  const int GB = G * B;
  if (tid < GB) {
    const int hl = tid / B, t = tid % B;
    const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
    float acc = 0.f;
    if (DT == LOSA_BF16) {
      const uint4* a4 = reinterpret_cast<const uint4*>(static_cast<const char*>(prm.qc) + row * kD * 2);
      const uint4* b4 = reinterpret_cast<const uint4*>(static_cast<const char*>(prm.qp) + row * kD * 2);
#pragma unroll 4
      for (int c = 0; c < kD / 8; ++c) {
        const uint4 x = a4[c], y = b4[c];
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float d0 = __fsub_rn(__uint_as_float(xs[u] << 16), __uint_as_float(ys[u] << 16));
          acc = __fadd_rn(acc, __fmul_rn(d0, d0));
          const float d1 = __fsub_rn(__uint_as_float(xs[u] & 0xffff0000u),
                                     __uint_as_float(ys[u] & 0xffff0000u));
          acc = __fadd_rn(acc, __fmul_rn(d1, d1));
        }
      }
    } else {
      const float4* a4 = reinterpret_cast<const float4*>(static_cast<const float*>(prm.qc) + row * kD);
      const float4* b4 = reinterpret_cast<const float4*>(static_cast<const float*>(prm.qp) + row * kD);
      for (int c = 0; c < kD / 4; ++c) {
        const float4 x = a4[c], y = b4[c];
        const float xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float d0 = __fsub_rn(xs[u], ys[u]);
          acc = __fadd_rn(acc, __fmul_rn(d0, d0));
        }
      }
    }
    s_mse[tid] = __fdiv_rn(acc, static_cast<float>(kD));
  }
  // block K/V of the group -> smem in the element type, rows >= B zero (this
  // area is reused for the bound scores once the suffix is done)
  const int Bpad = (B + kPS - 1) / kPS * kPS;
  {
    const int chunks = Bpad * kD * esz / 16;  // 16-byte chunks per tensor
    const char* kg = static_cast<const char*>(prm.kb) + static_cast<size_t>(sg) * B * kD * esz;
    const char* vg = static_cast<const char*>(prm.vb) + static_cast<size_t>(sg) * B * kD * esz;
    char* kd = reinterpret_cast<char*>(kbv);
    char* vd = kd + Bpad * kD * esz;
    const int valid = B * kD * esz / 16;
    for (int e = tid; e < chunks; e += kThreads) {
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (e < valid) {
        a = reinterpret_cast<const uint4*>(kg)[e];
        b = reinterpret_cast<const uint4*>(vg)[e];
      }
      reinterpret_cast<uint4*>(kd)[e] = a;
      reinterpret_cast<uint4*>(vd)[e] = b;
    }
  }
  __syncthreads();
  if (tid < GB) {  // rank within the head: ties go to the lower token index
    const int hl = tid / B, t = tid % B;
    const float x = s_mse[tid];
    int rk = 0;
    for (int u = 0; u < B; ++u) {
      const float y = s_mse[hl * B + u];
      rk += (y > x) || (y == x && u < t);
    }
    act_slot[tid] = rk < A ? 1 : 0;
  }
  __syncthreads();
  int my_slot = -1;
  if (tid < GB && act_slot[tid]) {  // slot = active tokens before t in the head
    const int hl = tid / B, t = tid % B;
    my_slot = 0;
    for (int u = 0; u < t; ++u) my_slot += act_slot[hl * B + u];
  }
  __syncthreads();
  if (tid < GB) act_slot[tid] = my_slot;
  __syncthreads();
  if (tid < GB && act_slot[tid] >= 0) {
    const int hl = tid / B, t = tid % B;
    act_tok[hl * A + act_slot[tid]] = t;
    if (rank == 0 && prm.active_idx)
      prm.active_idx[(static_cast<size_t>(s) * d.Hq + g * G + hl) * A + act_slot[tid]] = t;
  }
  __syncthreads();

  // active rows' query vectors for the bound: bf16 -> [R16][256] = [q- | q+]
  // (swizzled 16-byte chunks for ldmatrix); fp32 -> [R][128] plain
  const int R16 = (R + 15) / 16 * 16;
  if (scan) {
    if (DT == LOSA_BF16) {
      for (int e = tid; e < R16 * 32; e += kThreads) {
        const int r = e / 32, c = e % 32;  // 16-byte chunk c of row r (8 bf16)
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < R) {
          const int hl = r / A, t = act_tok[r];
          const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
          const uint4 q = *reinterpret_cast<const uint4*>(
              static_cast<const char*>(prm.qc) + row * kD * 2 + (c & 15) * 16);
          const uint32_t w[4] = {q.x, q.y, q.z, q.w};
          uint32_t o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint32_t lo16 = w[u] & 0xffffu, hi16 = w[u] >> 16;
            const bool neg_lo = lo16 & 0x8000u, neg_hi = hi16 & 0x8000u;
            if (c < 16) {  // q- = min(q, 0)
              lo16 = neg_lo ? lo16 : 0u;
              hi16 = neg_hi ? hi16 : 0u;
            } else {       // q+ = max(q, 0)
              lo16 = neg_lo ? 0u : lo16;
              hi16 = neg_hi ? 0u : hi16;
            }
            o[u] = lo16 | (hi16 << 16);
          }
          v = make_uint4(o[0], o[1], o[2], o[3]);
        }
        *reinterpret_cast<uint4*>(qrows + r * 512 + ((c ^ (r & 7)) << 4)) = v;
      }
    } else {
      for (int e = tid; e < R * kD / 4; e += kThreads) {
        const int r = e / (kD / 4), c = (e % (kD / 4)) * 4;
        const int hl = r / A, t = act_tok[r];
        const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
        *reinterpret_cast<float4*>(qrows + (r * kD + c) * 4) = ld4(prm.qc, row * kD + c, DT);
      }
    }
  }

  // suffix of this CTA's rows: stable token-rows i with i % CL == rank are
  // finished here; active rows r with r % CL == rank keep (o_s, L_s) in smem
  // for the final merge
  {
    float* psw = Ps + warp * 16;
    const char* kbs = reinterpret_cast<const char*>(kbv);
    const char* vbs = kbs + Bpad * kD * esz;
    const int nstable_mine = (GB - rank + CL - 1) / CL;
    const int nactive_mine = R > rank ? (R - rank + CL - 1) / CL : 0;
    for (int job = warp; job < nstable_mine + nactive_mine; job += kWarps) {
      int hl, t, r = -1;
      if (job < nstable_mine) {
        const int i = rank + job * CL;
        if (act_slot[i] >= 0) continue;
        hl = i / B;
        t = i % B;
      } else {
        r = rank + (job - nstable_mine) * CL;
        hl = r / A;
        t = act_tok[r];
      }
      const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
      const float4 q = ld4(prm.qc, row * kD + 4 * lane, DT);
      float m = -INFINITY, l = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j0 = 0; j0 < B; j0 += kPS)
        attend_page<DT>(q, kbs + j0 * kD * esz, vbs + j0 * kD * esz, min(kPS, B - j0),
                        d.scale_log2, m, l, acc, psw);
      const float inv = 1.f / l;
      const float4 os = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      const float Ls = (m + __log2f(l)) * kLn2;
      if (r < 0) {
        const float4 op = *reinterpret_cast<const float4*>(prm.o_p + row * kD + 4 * lane);
        const float Lp = prm.l_p[row];
        float4 o;
        float L;
        lse_merge(op, Lp, os, Ls, o, L);
        *reinterpret_cast<float4*>(prm.out + row * kD + 4 * lane) = o;
        if (prm.out_lse && lane == 0) prm.out_lse[row] = L;
      } else {
        float* dst = sfx + (r / CL) * kPartStride;
        if (lane == 0) dst[0] = Ls;
        *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = os;
      }
    }
  }
  __syncthreads();

  // ---- P1: bound scores of the chunk --------------------------------------
  if (scan) {
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % prm.stages;
      const uint32_t parity = (t / prm.stages) & 1;
      if (!mbar_wait(&mbar[st], parity)) {
        atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
        *s_fail = 1;
      }
      __syncthreads();
      if (*s_fail) break;
      const char* tile = ring + st * kStageBytes;
      const int np = min(prm.tile, npages - t * prm.tile);
      const int pl0 = t * prm.tile;  // chunk-local index of the tile's first page
      if (DT == LOSA_BF16) {
        const int ntn = (np + 7) / 8, ntm = R16 / 16;
        const int g4 = lane >> 2, t4 = lane & 3;
        for (int job = warp; job < ntn * ntm; job += kWarps) {
          const int nt = job % ntn, mt = job / ntn;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ks = 0; ks < 16; ks += 2) {
            uint32_t b[4];
            {
              const int mi = lane >> 3, pg = nt * 8 + (lane & 7);
              const int ch = ks * 2 + mi;
              ldsm_x4(su32(tile + pg * 512 + ((ch ^ (pg & 7)) << 4)), b[0], b[1], b[2], b[3]);
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
              uint32_t a[4];
              const int mi = lane >> 3;
              const int row = mt * 16 + (mi & 1) * 8 + (lane & 7);
              const int ch = (ks + kk) * 2 + (mi >> 1);
              ldsm_x4(su32(qrows + row * 512 + ((ch ^ (row & 7)) << 4)), a[0], a[1], a[2], a[3]);
              mma_bf16(acc, a, b[2 * kk], b[2 * kk + 1]);
            }
          }
          const int r0 = mt * 16 + g4, pc = pl0 + nt * 8 + 2 * t4;
          if (r0 < R) {
            sc[r0 * prm.sc_stride + pc] = acc[0];
            sc[r0 * prm.sc_stride + pc + 1] = acc[1];
          }
          if (r0 + 8 < R) {
            sc[(r0 + 8) * prm.sc_stride + pc] = acc[2];
            sc[(r0 + 8) * prm.sc_stride + pc + 1] = acc[3];
          }
        }
      } else {
        // fp32: exact sum in channel order, one rounding per operation
        for (int e = tid; e < np * R; e += kThreads) {
          const int pl = e % np, r = e / np;
          const int pg = p0 + pl0 + pl;
          const char* recp = tile + pl * prm.rec;
          const float* q = reinterpret_cast<const float*>(qrows) + r * kD;
          float acc = 0.f;
          for (int c = 0; c < kD / 4; ++c) {
            const float4 mn = *reinterpret_cast<const float4*>(recp + meta_swz(16u * c, pg));
            const float4 mx =
                *reinterpret_cast<const float4*>(recp + meta_swz(16u * (c + kD / 4), pg));
            const float mns[4] = {mn.x, mn.y, mn.z, mn.w}, mxs[4] = {mx.x, mx.y, mx.z, mx.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float qi = q[4 * c + u];
              acc = __fadd_rn(acc, fmaxf(__fmul_rn(qi, mxs[u]), __fmul_rn(qi, mns[u])));
            }
          }
          sc[r * prm.sc_stride + pl0 + pl] = acc;
        }
      }
      __syncthreads();
      if (tid == 0 && t + prm.stages < ntiles) {  // refill the stage just consumed
        const int tn = t + prm.stages;
        const int npn = min(prm.tile, npages - tn * prm.tile);
        const uint32_t bytes = static_cast<uint32_t>(npn * prm.rec);
        mbar_expect_tx(&mbar[st], bytes);
        bulk_g2s(ring + st * kStageBytes,
                 meta_g + static_cast<size_t>(p0 + tn * prm.tile) * prm.rec, bytes, &mbar[st]);
      }
    }
    // ---- P2: chunk-local top-k per row ------------------------------------
    if (!*s_fail) {
      for (int r = warp; r < R; r += kWarps) {
        const float* row = sc + r * prm.sc_stride;
        warp_topk([&](int i) { return sel_key(row[i], p0 + i); }, npages, k, cand + r * k,
                  cbuf + warp * kCandCap);
      }
    }
  }
  __syncthreads();
  cluster.sync();

  // ---- P3: merge of the CL candidate lists of this CTA's rows --------------
  if (A > 0) {
    if (!d.all_pages) {
      for (int r = rank + CL * warp; r < R; r += CL * kWarps) {
        unsigned long long* best = cbuf + (kWarps + warp) * kCandCap;  // k <= 64
        const unsigned long long* remote[kMaxCluster];
        for (int c = 0; c < CL; ++c) remote[c] = cluster.map_shared_rank(cand, c) + r * k;
        warp_topk([&](int i) { return remote[i / k][i % k]; }, CL * k, k, best,
                  cbuf + warp * kCandCap);
        // the k pages in ascending order
        int32_t* dst = sel_own + (r / CL) * k;
        for (int j = lane; j < k; j += 32) {
          const int pj = key_index(best[j]);
          int rk = 0;
          for (int u = 0; u < k; ++u) rk += key_index(best[u]) < pj;
          dst[rk] = pj;
          if (prm.page_idx) {
            const int hl = r / A, a = r % A;
            prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + a) * k + rk] = pj;
          }
        }
        __syncwarp();
      }
    } else if (prm.page_idx) {
      for (int e = tid; e < R * k; e += kThreads) {
        const int r = e / k;
        if (r % CL != rank) continue;
        const int hl = r / A, a = r % A;
        prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + a) * k + e % k] = e % k;
      }
    }
  }
  __syncthreads();
  cluster.sync();

  // ---- P4: union of the group's pages and this CTA's share ------------------
  const int nwords = (d.P + 31) / 32;
  if (A > 0 && d.all_pages) {
    // every row takes every page: the union is the whole prefix
    const int U = d.P;
    const int nlp = U > rank ? (U - rank + CL - 1) / CL : 0;
    if (tid == 0) {
      *s_nlp = nlp;
      if (rank == 0 && prm.union_count) prm.union_count[sg] = U;
    }
    for (int j = tid; j < min(nlp, prm.max_lp); j += kThreads) lpages[j] = rank + j * CL;
    for (int e = tid; e < min(nlp, prm.max_lp) * d.MW; e += kThreads) {
      const int w = e % d.MW;
      const int nb = min(32, R - 32 * w);
      masks[e] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
    }
  } else if (A > 0) {
    for (int e = tid; e < R * k; e += kThreads) {
      const int r = e / k, j = e % k;
      sel_all[e] = cluster.map_shared_rank(sel_own, r % CL)[(r / CL) * k + j];
    }
    for (int w = tid; w < nwords; w += kThreads) bitmap[w] = 0u;
    __syncthreads();
    for (int e = tid; e < R * k; e += kThreads) {
      const int p = sel_all[e];
      if (p >= 0 && p < d.P) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
      else atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
    }
    __syncthreads();
    // exclusive prefix of word popcounts (warp 0; words dealt in runs per lane)
    if (warp == 0) {
      const int per = (nwords + 31) / 32;
      const int w0 = lane * per, w1 = min(nwords, w0 + per);
      int sum = 0;
      for (int w = w0; w < w1; ++w) sum += __popc(bitmap[w]);
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
      for (int w = w0; w < w1; ++w) {
        wbase[w] = run;
        run += __popc(bitmap[w]);
      }
      if (lane == 31) *s_U = incl;
    }
    __syncthreads();
    const int U = *s_U;
    const int nlp = U > rank ? (U - rank + CL - 1) / CL : 0;
    if (tid == 0) {
      *s_nlp = nlp;
      if (rank == 0 && prm.union_count) prm.union_count[sg] = U;
    }
    for (int w = tid; w < nwords; w += kThreads) {
      uint32_t bits = bitmap[w];
      int pos = wbase[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos % CL == rank && pos / CL < prm.max_lp) lpages[pos / CL] = w * 32 + b;
        ++pos;
      }
    }
    for (int e = tid; e < min(nlp, prm.max_lp) * d.MW; e += kThreads) masks[e] = 0u;
    __syncthreads();
    for (int e = tid; e < R * k; e += kThreads) {
      const int p = sel_all[e];
      if (p < 0 || p >= d.P) continue;
      const int w = p >> 5;
      const int u = wbase[w] + __popc(bitmap[w] & ((1u << (p & 31)) - 1u));
      if (u % CL != rank) continue;
      const int r = e / k;
      if (u / CL < prm.max_lp) atomicOr(&masks[(u / CL) * d.MW + (r >> 5)], 1u << (r & 31));
      else atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
    }
  } else if (tid == 0 && rank == 0 && prm.union_count) {
    prm.union_count[sg] = 0;
  }
  __syncthreads();

  // ---- P5: gather this CTA's union pages ------------------------------------
  if (A > 0 && !*s_fail && warp < prm.gwarps) {
    const int nlp = min(*s_nlp, prm.max_lp);
    const int gw = prm.gwarps;
    const int pbytes = kPS * kD * esz;  // one of K, V of a full page
    char* slots = ring + warp * prm.gslots * 2 * pbytes;
    uint64_t* wbar = mbar + kMaxStages + warp * 2;
    const int mine = warp < nlp ? (nlp - warp + gw - 1) / gw : 0;
    auto issue = [&](int i) {  // i-th page of this warp into slot i % gslots
      const int p = lpages[warp + i * gw];
      const int ntok = min(kPS, d.L - p * kPS);
      const uint32_t bytes = static_cast<uint32_t>(ntok * kD * esz);
      char* dst = slots + (i % prm.gslots) * 2 * pbytes;
      const size_t off = (static_cast<size_t>(sg) * d.L + static_cast<size_t>(p) * kPS) * kD * esz;
      mbar_expect_tx(&wbar[i % prm.gslots], 2 * bytes);
      bulk_g2s(dst, static_cast<const char*>(prm.K) + off, bytes, &wbar[i % prm.gslots]);
      bulk_g2s(dst + pbytes, static_cast<const char*>(prm.V) + off, bytes, &wbar[i % prm.gslots]);
    };
    if (lane == 0)
      for (int i = 0; i < min(mine, prm.gslots); ++i) issue(i);
    float* psw = Ps + warp * 16;
    for (int i = 0; i < mine; ++i) {
      const int ul = warp + i * gw;
      const int p = lpages[ul];
      const int ntok = min(kPS, d.L - p * kPS);
      // every lane waits on the slot's barrier (acquire by each reader)
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&wbar[i % prm.gslots], (i / prm.gslots) & 1));
      if (!ok) {
        if (lane == 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
        break;
      }
      const char* Ks = slots + (i % prm.gslots) * 2 * pbytes;
      const char* Vs = Ks + pbytes;
      const uint32_t* mk = masks + ul * d.MW;
      for (int w = 0; w < d.MW; ++w) {
        uint32_t bits = mk[w];
        while (bits) {
          const int r = w * 32 + __ffs(bits) - 1;
          bits &= bits - 1;
          const int hl = r / A, t = act_tok[r];
          const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
          const float4 q = ld4(prm.qc, row * kD + 4 * lane, DT);
          float m = -INFINITY, l = 0.f;
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          // zero rows beyond ntok are masked by attend_page (score -inf, p = 0)
          attend_page<DT>(q, Ks, Vs, ntok, d.scale_log2, m, l, acc, psw);
          // slot of page p in row r's ascending list
          int lo_ = p;
          if (!d.all_pages) {
            const int32_t* lst = sel_all + r * k;
            int hi_ = k;
            lo_ = 0;
            while (lo_ < hi_) {
              const int mid = (lo_ + hi_) >> 1;
              if (lst[mid] < p) lo_ = mid + 1;
              else hi_ = mid;
            }
            if (lo_ < k && lst[lo_] != p) lo_ = k;
          }
          if (lo_ >= k) {
            if (lane == 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
            continue;
          }
          float* dst = prm.part + ((static_cast<size_t>(sg) * R + r) * k + lo_) * kPartStride;
          if (lane == 0) {
            dst[0] = m;
            dst[1] = l;
          }
          *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = acc;
        }
      }
      __syncwarp();
      if (lane == 0 && i + prm.gslots < mine) issue(i + prm.gslots);
    }
  }
  __threadfence();
  __syncthreads();
  cluster.sync();

  // ---- P6: combine, cache write-back, merge with the suffix ----------------
  if (A > 0 && !*s_fail) {
    for (int r = rank + CL * warp; r < R; r += CL * kWarps) {
      const float* src0 = prm.part + (static_cast<size_t>(sg) * R + r) * k * kPartStride;
      float M = -INFINITY;
      for (int j = 0; j < k; ++j) M = fmaxf(M, __ldcg(src0 + static_cast<size_t>(j) * kPartStride));
      float lsum = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {
        const float* src = src0 + static_cast<size_t>(j) * kPartStride;
        const float w = exp2f(__ldcg(src) - M);
        lsum += w * __ldcg(src + 1);
        const float4 x = __ldcg(reinterpret_cast<const float4*>(src + 4 + 4 * lane));
        acc.x += w * x.x;
        acc.y += w * x.y;
        acc.z += w * x.z;
        acc.w += w * x.w;
      }
      const float inv = 1.f / lsum;
      const float4 op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      const float Lp = (M + __log2f(lsum)) * kLn2;
      const int hl = r / A, t = act_tok[r];
      const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
      *reinterpret_cast<float4*>(prm.o_p + row * kD + 4 * lane) = op;
      if (lane == 0) prm.l_p[row] = Lp;
      const float* sx = sfx + (r / CL) * kPartStride;
      const float4 os = *reinterpret_cast<const float4*>(sx + 4 + 4 * lane);
      float4 o;
      float L;
      lse_merge(op, Lp, os, sx[0], o, L);
      *reinterpret_cast<float4*>(prm.out + row * kD + 4 * lane) = o;
      if (prm.out_lse && lane == 0) prm.out_lse[row] = L;
    }
  }
}

// ---------------------------------------------------------------------------
// host side: launch geometry, shared-memory layout, attributes
// ---------------------------------------------------------------------------
int align_up(int x, int a) { return (x + a - 1) / a * a; }

bool plan_with_ring(const Dims& d, Params* prm, int ring_bytes, int max_dyn, int max_cluster) {
  prm->d = d;
  prm->rec = 2 * kD * d.esz;
  prm->tile = kStageBytes / prm->rec;  // 64 (bf16) or 32 (fp32) pages per stage
  const int chunk = align_up((d.P + max_cluster - 1) / max_cluster, 8);
  const int CL = (d.P + chunk - 1) / chunk;
  prm->chunk = chunk;
  prm->CL = CL;
  prm->stages = ring_bytes / kStageBytes;
  prm->sc_stride = align_up(chunk, 4) + 4;
  const int pbytes = kPS * kD * d.esz;
  prm->gwarps = std::min(kWarps, ring_bytes / (2 * pbytes));
  if (prm->gwarps < 1) return false;
  prm->gslots = std::min(2, ring_bytes / (prm->gwarps * 2 * pbytes));
  prm->max_lp = (d.Umax + CL - 1) / CL;
  const bool scan = d.A > 0 && !d.all_pages;
  if (scan && d.k > kCandCap) return false;
  const int R16 = (d.R + 15) / 16 * 16;
  const int Bpad = (d.B + kPS - 1) / kPS * kPS;
  const int nwords = (d.P + 31) / 32;
  const int rows_per_cta = (d.R + CL - 1) / CL;
  Layout& lo = prm->lo;
  int off = 0;
  auto take = [&](long long bytes, int align) {
    off = align_up(off, align);
    const int o = off;
    off += static_cast<int>(std::min<long long>(bytes, 1 << 30));
    return o;
  };
  lo.ring = take(ring_bytes, 1024);
  lo.scores = take(std::max<long long>(scan ? 4LL * d.R * prm->sc_stride : 0,
                                       2LL * Bpad * kD * d.esz), 16);
  lo.qrows = take(scan ? R16 * 512 : 0, 128);
  lo.kbv = lo.scores;
  lo.cand = take(scan ? 8LL * d.R * d.k : 0, 16);
  lo.sel_own = take(scan ? 4LL * rows_per_cta * d.k : 0, 16);
  lo.sel_all = take(d.all_pages ? 0 : 4LL * d.R * d.k, 16);
  lo.bitmap = take(nwords * 4, 16);
  lo.wbase = take(nwords * 4, 16);
  lo.lpages = take(prm->max_lp * 4, 16);
  lo.masks = take(4LL * prm->max_lp * d.MW, 16);
  lo.sfx = take(4LL * rows_per_cta * kPartStride, 16);
  lo.cbuf = take(2 * kWarps * kCandCap * 8, 16);
  lo.ps = take(kWarps * 16 * 4, 16);
  lo.misc = take((4 + 3 * kMaxRowsPerGroup) * 4, 16);
  lo.mbar = take((kMaxStages + kWarps * 2) * 8, 8);
  lo.total = off;
  return lo.total <= max_dyn;
}

// Largest metadata ring (128, 96 or 64 KiB) whose plan fits.
bool plan(const Dims& d, Params* prm, int max_dyn, int max_cluster = kMaxCluster) {
  for (int ring = kMaxRingBytes; ring >= 64 * 1024; ring -= 32 * 1024)
    if (plan_with_ring(d, prm, ring, max_dyn, max_cluster)) return true;
  return false;
}

}  // namespace

// Whether the fused step's shared-memory plan fits `max_dyn` bytes.
bool fused_step_fits(const Dims& d, int max_dyn) {
  Params prm;
  return plan(d, &prm, max_dyn);
}

namespace {

std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices] = {};
int g_attr_dyn[kMaxDevices] = {};
int g_attr_cluster[kMaxDevices] = {};

// Largest cluster size (16 or 8) of which at least one cluster of
// full-shared-memory CTAs can be resident on the device.
int probe_cluster(int dyn) {
  for (int cl = kMaxCluster; cl >= 8; cl /= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(dyn);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, losa_step_kernel<LOSA_BF16>, &cfg) == cudaSuccess &&
        n > 0)
      return cl;
    cudaGetLastError();  // clear a refused query
  }
  return 8;
}

int ensure_attributes(int* max_dyn, int* max_cluster) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return LOSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_attr_mu);
  if (!g_attr_done[dev]) {
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return record_cuda_error(e);
    const void* fns[] = {reinterpret_cast<const void*>(losa_step_kernel<LOSA_BF16>),
                         reinterpret_cast<const void*>(losa_step_kernel<LOSA_F32>)};
    int dyn = optin;
    for (const void* f : fns) {
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, f);
      if (e != cudaSuccess) return record_cuda_error(e);
      const int mine = optin - static_cast<int>(fa.sharedSizeBytes);
      e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, mine);
      if (e != cudaSuccess) return record_cuda_error(e);
      e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return record_cuda_error(e);
      dyn = mine < dyn ? mine : dyn;
    }
    g_attr_dyn[dev] = dyn;
    g_attr_cluster[dev] = probe_cluster(dyn);
    g_attr_done[dev] = true;
  }
  *max_dyn = g_attr_dyn[dev];
  *max_cluster = g_attr_cluster[dev];
  return LOSA_OK;
}

}  // namespace

// Plans and launches the fused step (host validation already done).
int launch_fused_step(const Dims& d, const void* q_cur, const void* q_prev, const void* k_prefix,
                      const void* v_prefix, const void* page_meta, const void* k_blk,
                      const void* v_blk, float* o_p, float* l_p, float* out, float* out_lse,
                      int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                      void* workspace, cudaStream_t st) {
  int max_dyn = 0, max_cluster = kMaxCluster;
  int rc = ensure_attributes(&max_dyn, &max_cluster);
  if (rc != LOSA_OK) return rc;
  Params prm;
  if (!plan(d, &prm, max_dyn, max_cluster)) return LOSA_ERR_UNSUPPORTED;
  if (d.S * d.Hkv > 65535) return LOSA_ERR_UNSUPPORTED;
  char* ws = static_cast<char*>(workspace);
  prm.qc = q_cur;
  prm.qp = q_prev;
  prm.K = k_prefix;
  prm.V = v_prefix;
  prm.meta = static_cast<const char*>(page_meta);
  prm.kb = k_blk;
  prm.vb = v_blk;
  prm.o_p = o_p;
  prm.l_p = l_p;
  prm.out = out;
  prm.out_lse = out_lse;
  prm.active_idx = active_idx;
  prm.page_idx = page_idx;
  prm.union_count = union_count;
  prm.part = reinterpret_cast<float*>(ws + d.off_part);
  prm.status = reinterpret_cast<int*>(ws + d.off_status);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(prm.CL, d.S * d.Hkv, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(prm.lo.total);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = prm.CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = d.dtype == LOSA_BF16 ? cudaLaunchKernelEx(&cfg, losa_step_kernel<LOSA_BF16>, prm)
                                       : cudaLaunchKernelEx(&cfg, losa_step_kernel<LOSA_F32>, prm);
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}

}  // namespace losa
