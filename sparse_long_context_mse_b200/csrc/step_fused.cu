// step_fused.cu -- one LoSA denoising step in two kernel launches.
//
// LoSA paper, methodology: locality pruning (MSE of Q_t vs Q_{t-1}, top-|A|
// per head), reuse of the cached prefix state for stable tokens, QUEST page
// selection for active queries only, union of the selected pages, sparse
// prefix attention, dense intra-block suffix, online-softmax merge, cache
// update.
//
// K1 `losa_scan_kernel` -- a flat grid over every SM: each CTA owns one chunk
//    of one (sequence, KV head) group's pages.  It bulk-copies (TMA) the
//    chunk's page metadata into a shared-memory ring and meanwhile computes
//    the group's active set (every CTA of the group computes it, identically)
//    and the suffix attention over the block of its share of the group's
//    token rows: stable rows are finished here (merge with the untouched
//    cache), active rows leave their suffix partial in the workspace.  With
//    no active row (or k = P) that is all.  Otherwise the QUEST bound of the
//    chunk's pages for the group's R active rows -- bf16: tensor cores,
//    U = [q- | q+] . [kmin ; kmax] with mma.sync m16n8k16 (exact products,
//    fp32 accumulation); fp32: CUDA cores, the sum in channel order with one
//    rounding per operation -- and a chunk-local top-k per row, written to the
//    workspace.
// K2 `losa_gather_kernel` -- one thread-block cluster per group, launched
//    with programmatic dependent launch behind K1.  Rows are dealt to the
//    cluster's CTAs; each merges its rows' chunk candidates into the row's
//    top-k pages; every CTA then builds the group's page union (bitmap,
//    ascending, with a row mask per page) from the rows' lists in
//    distributed shared memory; union slot u belongs to CTA u % CL, which
//    bulk-copies the page's K and V once for the whole GQA group and folds
//    the page into an online-softmax partial per row; finally each CTA
//    combines its rows' partials from every CTA of the cluster (distributed
//    shared memory), writes the new o_p / L_p to the cache and merges them
//    with the suffix partial.  K2 is launched only when some row is active.
//
// Every wait on a bulk copy is bounded (clock64); a wait that gives up sets
// LOSA_ERR_DEVICE_TIMEOUT in the status word and the CTA skips the rest of
// its work but still takes part in every cluster barrier, so the cluster
// never deadlocks.  There is no other cross-CTA wait.
#include <cooperative_groups.h>

#include <algorithm>
#include <mutex>

#include "losa_common.cuh"
#include "ptx.cuh"

namespace cg = cooperative_groups;

namespace losa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRingBytes = 128 * 1024;
constexpr int kStageBytes = 32 * 1024;
constexpr int kMaxStages = kMaxRingBytes / kStageBytes;
constexpr int kCandCap = 64;                     // per-warp compaction buffer
constexpr int kMaxCluster = 16;
constexpr int kMaxGatherPages = 16;              // pages in flight per K2 CTA

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
__device__ __noinline__ void attend_page(float4 q, const char* Ks, const char* Vs, int ntok,
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
// Register top-k: KP (power of two) selection keys per thread, descending.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cas_desc(unsigned long long& a, unsigned long long& b) {
  const bool sw = a < b;
  const unsigned long long hi = sw ? b : a, lo = sw ? a : b;
  a = hi;
  b = lo;
}

template <int KP>
__device__ __forceinline__ void bitonic_sort_desc(unsigned long long (&x)[KP]) {
#pragma unroll
  for (int size = 2; size <= KP; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
#pragma unroll
      for (int i = 0; i < KP; ++i) {
        const int j = i ^ stride;
        if (j > i) {
          if ((i & size) == 0) cas_desc(x[i], x[j]);
          else cas_desc(x[j], x[i]);
        }
      }
    }
  }
}

// x <- the KP largest of x and y (both descending); result descending.  The
// element-wise max of x and reversed y is bitonic and holds exactly the top
// KP; half-cleaners sort it.
template <int KP>
__device__ __forceinline__ void merge_top(unsigned long long (&x)[KP],
                                          const unsigned long long (&y)[KP]) {
#pragma unroll
  for (int i = 0; i < KP; ++i) x[i] = umax64(x[i], y[KP - 1 - i]);
#pragma unroll
  for (int stride = KP >> 1; stride > 0; stride >>= 1) {
#pragma unroll
    for (int i = 0; i < KP; ++i) {
      const int j = i ^ stride;
      if (j > i) cas_desc(x[i], x[j]);
    }
  }
}

// Merge the lists of `width` consecutive lanes (power of two <= 32); every
// lane of the group ends with the group's top KP.
template <int KP>
__device__ __forceinline__ void group_merge(unsigned long long (&x)[KP], int width) {
  for (int off = 1; off < width; off <<= 1) {
    unsigned long long y[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i) y[i] = __shfl_xor_sync(0xffffffffu, x[i], off);
    merge_top<KP>(x, y);
  }
}

// Top-KP of the keys key(i), i = j, j + stride, j + 2*stride, ... < n, held by
// one thread (descending, 0 = empty).
template <int KP, typename KeyFn>
__device__ __forceinline__ void thread_topk(KeyFn key, int j, int stride, int n,
                                            unsigned long long (&x)[KP]) {
#pragma unroll
  for (int i = 0; i < KP; ++i) x[i] = 0ull;
  for (int base = j; base < n; base += stride * KP) {
    unsigned long long y[KP];
#pragma unroll
    for (int i = 0; i < KP; ++i) {
      const int idx = base + i * stride;
      y[i] = idx < n ? key(idx) : 0ull;
    }
    bitonic_sort_desc<KP>(y);
    merge_top<KP>(x, y);
  }
}

// Top-k (k <= W) of the keys held by a group of W lanes (W a power of two;
// groups are aligned inside the warp).  Lane j of a group holds the keys
// key(i) for i = j, j + W, ... < n (0 = no key).  The threshold tau is the
// k-th largest of the group's lane maxima: at least k keys reach it, so every
// key of the top k does too.  The keys >= tau (at most `cap`) are compacted
// into buf and rank-sorted into out[0..k).  Returns false, for every lane of
// the warp and before writing anything, if an active group of the warp had
// more than `cap` survivors.
template <typename KeyFn>
__device__ bool group_topk_filter(KeyFn key, int n, int W, int k, unsigned long long* buf,
                                  unsigned long long* out, int cap, bool active) {
  constexpr int kNV = 32;  // keys a lane keeps in registers
  const int lane = threadIdx.x & 31;
  const int j = lane & (W - 1);
  if (n > W * kNV) return false;  // (uniform) the caller's other path handles it
  unsigned long long kx[kNV];
  unsigned long long lmax = 0ull;
#pragma unroll
  for (int t = 0; t < kNV; ++t) {
    const int i = j + t * W;
    kx[t] = i < n ? key(i) : 0ull;
    lmax = umax64(lmax, kx[t]);
  }
  unsigned long long v = lmax;  // bitonic sort of the lane maxima, descending
#pragma unroll 1
  for (int size = 2; size <= W; size <<= 1) {
#pragma unroll 1
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
      const bool dir = (j & size) == 0, lower = (j & stride) == 0;
      v = (lower == dir) ? umax64(v, o) : (v < o ? v : o);
    }
  }
  const unsigned long long tau = __shfl_sync(0xffffffffu, v, k - 1, W);
  int cnt = 0;
#pragma unroll
  for (int t = 0; t < kNV; ++t) cnt += (kx[t] >= tau && kx[t] != 0ull);
  int incl = cnt;
#pragma unroll 1
  for (int o = 1; o < W; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o, W);
    if (j >= o) incl += y;
  }
  const int total = __shfl_sync(0xffffffffu, incl, W - 1, W);
  if (!__all_sync(0xffffffffu, !active || total <= cap)) return false;
  if (active) {
    int pos = incl - cnt;
#pragma unroll
    for (int t = 0; t < kNV; ++t)
      if (kx[t] >= tau && kx[t] != 0ull) buf[pos++] = kx[t];
  }
  __syncwarp();
  if (active) {
#pragma unroll 1
    for (int t = j; t < total; t += W) {
      const unsigned long long x = buf[t];
      int rank = 0;
#pragma unroll 8
      for (int m = 0; m < total; ++m) rank += buf[m] > x;
      if (rank < k) out[rank] = x;
    }
#pragma unroll 1
    for (int t = total + j; t < k; t += W) out[t] = 0ull;
  }
  __syncwarp();
  return true;
}

int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}
int align_up(int x, int a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// K1: scan
// ---------------------------------------------------------------------------
struct ScanLayout {
  int ring, scores, kbv, qrows, misc, ps, fbuf, cbuf, mbar, total;
};

struct ScanParams {
  const void* qc;
  const void* qp;
  const char* meta;
  const void* kb;
  const void* vb;
  const float* o_p;
  const float* l_p;
  float* out;
  float* out_lse;
  int32_t* active_idx;
  int32_t* union_count;
  int32_t* act_tok_g;              // workspace [S*Hkv][R]
  float* sfx_g;                    // workspace [S*Hkv][R][kPartStride]: active rows' suffix
  unsigned long long* cand;        // workspace [S*Hkv][nchunk][R][k]
  int* status;
  Dims d;
  int rec;        // bytes per metadata record
  int tile;       // pages per ring stage
  int stages;     // ring stages
  int sc_stride;  // floats per score row
  int qw;         // 32-bit words per staged query row (padded)
  int kp;         // register top-k width (2..16), 0 = warp fallback
  int tpr;        // threads per row for the chunk top-k
  ScanLayout lo;
};

// Chunk-local top-k of every active row -> dst_base[r][0..k).  Fast path
// (k <= 16): the threshold filter over a group of W >= k lanes per row, rows
// in passes of kThreads / W; a warp whose groups overflow the filter buffer
// falls back to register sort-and-merge.  k > 16: one warp per row.
template <int DT, int KP>
__device__ __forceinline__ void chunk_topk(const ScanParams& prm, const float* sc, int R, int k,
                                           int npages, int p0, unsigned long long* dst_base,
                                           unsigned long long* fbuf, unsigned long long* cbuf) {
  const int tid = threadIdx.x;
  if (KP > 0) {
    const int W = prm.tpr;
    const int rows_per_pass = kThreads / W;
#pragma unroll 1
    for (int r0 = 0; r0 < R; r0 += rows_per_pass) {
      const int r = r0 + tid / W;
      const bool active = r < R;
      const float* row = sc + (active ? r : 0) * prm.sc_stride;
      unsigned long long* out = dst_base + static_cast<size_t>(active ? r : 0) * k;
      auto key = [&](int i) { return sel_key(row[i], p0 + i); };
      if (!group_topk_filter(key, npages, W, k, fbuf + (tid / W) * kCandCap, out, kCandCap,
                             active)) {
        unsigned long long x[KP > 0 ? KP : 1];
        thread_topk<(KP > 0 ? KP : 1)>(key, tid & (W - 1), W, npages, x);
        group_merge<(KP > 0 ? KP : 1)>(x, W);
        if (active && (tid & (W - 1)) == 0) {
#pragma unroll
          for (int i = 0; i < (KP > 0 ? KP : 1); ++i)
            if (i < k) out[i] = x[i];
        }
      }
    }
  } else {
    const int warp = tid >> 5, lane = tid & 31;
#pragma unroll 1
    for (int r = warp; r < R; r += kWarps) {
      const float* row = sc + r * prm.sc_stride;
      warp_topk([&](int i) { return sel_key(row[i], p0 + i); }, npages, k,
                cbuf + (kWarps + warp) * kCandCap, cbuf + warp * kCandCap);
      __syncwarp();
#pragma unroll 1
      for (int i = lane; i < k; i += 32)
        dst_base[static_cast<size_t>(r) * k + i] = cbuf[(kWarps + warp) * kCandCap + i];
      __syncwarp();
    }
  }
}

template <int DT, int KP>
__global__ void __launch_bounds__(kThreads, 1) losa_scan_kernel(const ScanParams prm) {
  extern __shared__ __align__(1024) char smem[];
  const Dims& d = prm.d;
  const ScanLayout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, nchunk = gridDim.x;
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int GB = G * B;
  const int qw = prm.qw;
  const int esz = DT == LOSA_BF16 ? 2 : 4;
  const int Bpad = (B + kPS - 1) / kPS * kPS;

  // let the gather kernel start its own preparation now; it waits for this
  // grid's completion before it reads anything written here
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  char* ring = smem + lo.ring;
  float* sc = reinterpret_cast<float*>(smem + lo.scores);
  uint32_t* qcs = reinterpret_cast<uint32_t*>(smem + lo.scores);  // staging; aliases sc
  uint32_t* qps = qcs + GB * qw;
  char* kbv = smem + lo.kbv;  // the block's own K then V (element type)
  char* qrows = smem + lo.qrows;
  float* Ps = reinterpret_cast<float*>(smem + lo.ps);
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  unsigned long long* fbuf = reinterpret_cast<unsigned long long*>(smem + lo.fbuf);
  unsigned long long* cbuf = reinterpret_cast<unsigned long long*>(smem + lo.cbuf);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  int32_t* s_fail = misc;
  float* s_mse = reinterpret_cast<float*>(misc + 4);
  int32_t* act_slot = misc + 4 + kMaxRowsPerGroup;
  int32_t* act_tok = act_slot + kMaxRowsPerGroup;

  const int p0 = chunk * d.chunk_pages;
  const int npages = max(0, min(d.P, p0 + d.chunk_pages) - p0);
  const int ntiles = (npages + prm.tile - 1) / prm.tile;
  const char* meta_g = prm.meta + static_cast<size_t>(sg) * d.P * prm.rec;
  const bool scan = A > 0 && !d.all_pages && npages > 0;
  // token-rows of the group whose suffix this CTA computes: i = chunk + n * nchunk
  const int n_mine = GB > chunk ? (GB - chunk + nchunk - 1) / nchunk : 0;
  const uint32_t blk_bytes = static_cast<uint32_t>(B * kD * esz);

  if (tid == 0) {
    for (int i = 0; i < kMaxStages + 1; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
    *s_fail = 0;
    if (n_mine > 0) {
      mbar_expect_tx(&mbar[kMaxStages], 2 * blk_bytes);
      const size_t off = static_cast<size_t>(sg) * B * kD * esz;
      bulk_g2s(kbv, static_cast<const char*>(prm.kb) + off, blk_bytes, &mbar[kMaxStages]);
      bulk_g2s(kbv + Bpad * kD * esz, static_cast<const char*>(prm.vb) + off, blk_bytes,
               &mbar[kMaxStages]);
    }
#pragma unroll 1
    for (int t = 0; scan && t < min(ntiles, prm.stages); ++t) {
      const int np = min(prm.tile, npages - t * prm.tile);
      const uint32_t bytes = static_cast<uint32_t>(np * prm.rec);
      mbar_expect_tx(&mbar[t], bytes);
      bulk_g2s(ring + t * kStageBytes, meta_g + static_cast<size_t>(p0 + t * prm.tile) * prm.rec,
               bytes, &mbar[t]);
    }
  }

  // ---- stage the group's current / previous queries (coalesced), padded
  // rows so that one thread walking its row in channel order hits every bank
  {
    const int cpr = kD * esz / 16;  // 16-byte chunks per row
    const size_t base = (static_cast<size_t>(s) * d.Hq + g * G) * B * kD * esz;
    const uint4* gc = reinterpret_cast<const uint4*>(static_cast<const char*>(prm.qc) + base);
    const uint4* gp = reinterpret_cast<const uint4*>(static_cast<const char*>(prm.qp) + base);
#pragma unroll 2
    for (int e = tid; e < GB * cpr; e += kThreads) {
      const int row = e / cpr, c = e % cpr;
      const uint4 a = gc[e], b = gp[e];
      uint32_t* x = qcs + row * qw + 4 * c;
      uint32_t* y = qps + row * qw + 4 * c;
      x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
      y[0] = b.x; y[1] = b.y; y[2] = b.z; y[3] = b.w;
    }
  }
  __syncthreads();

  // ---- locality score: fp32, one rounding per operation, channels in order
  if (tid < GB) {
    const uint32_t* x = qcs + tid * qw;
    const uint32_t* y = qps + tid * qw;
    float acc = 0.f;
    if (DT == LOSA_BF16) {
#pragma unroll 8
      for (int w = 0; w < kD / 2; ++w) {
        const uint32_t a = x[w], b = y[w];
        const float d0 = __fsub_rn(__uint_as_float(a << 16), __uint_as_float(b << 16));
        acc = __fadd_rn(acc, __fmul_rn(d0, d0));
        const float d1 = __fsub_rn(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u));
        acc = __fadd_rn(acc, __fmul_rn(d1, d1));
      }
    } else {
#pragma unroll 8
      for (int w = 0; w < kD; ++w) {
        const float d0 = __fsub_rn(__uint_as_float(x[w]), __uint_as_float(y[w]));
        acc = __fadd_rn(acc, __fmul_rn(d0, d0));
      }
    }
    s_mse[tid] = acc * (1.0f / kD);  // exact: kD is a power of two
  }
  __syncthreads();
  if (tid < GB) {  // rank within the head: ties go to the lower token index
    const int hl = tid / B, t = tid % B;
    const float x = s_mse[tid];
    int rk = 0;
#pragma unroll 4
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
#pragma unroll 1
    for (int u = 0; u < t; ++u) my_slot += act_slot[hl * B + u];
  }
  __syncthreads();
  if (tid < GB) act_slot[tid] = my_slot;
  __syncthreads();
  if (tid < GB && act_slot[tid] >= 0) {
    const int hl = tid / B, r = hl * A + act_slot[tid];
    act_tok[r] = tid % B;
    if (chunk == 0) {
      prm.act_tok_g[static_cast<size_t>(sg) * R + r] = tid % B;
      if (prm.active_idx)
        prm.active_idx[(static_cast<size_t>(s) * d.Hq + g * G + hl) * A + act_slot[tid]] = tid % B;
    }
  }
  if (chunk == 0 && tid == 0 && A == 0 && prm.union_count) prm.union_count[sg] = 0;
  __syncthreads();

  // ---- suffix over the block of this CTA's token-rows (hidden under the
  // metadata stream): stable rows are finished here (merge with their
  // untouched cache); active rows leave (o_s, L_s) in the workspace
  if (n_mine > 0) {
    if (!mbar_wait(&mbar[kMaxStages], 0)) {
      if (tid == 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
    } else {
      float* psw = Ps + warp * 16;
#pragma unroll 1
      for (int n = warp; n < n_mine; n += kWarps) {
        const int i = chunk + n * nchunk;
        const int slot = act_slot[i];
        const size_t grow = (static_cast<size_t>(s) * d.Hq + g * G) * B + i;
        float4 q;
        if (DT == LOSA_BF16) {
          const uint32_t w0 = qcs[i * qw + 2 * lane], w1 = qcs[i * qw + 2 * lane + 1];
          q = make_float4(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xffff0000u),
                          __uint_as_float(w1 << 16), __uint_as_float(w1 & 0xffff0000u));
        } else {
          const uint32_t* w = qcs + i * qw + 4 * lane;
          q = make_float4(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]),
                          __uint_as_float(w[3]));
        }
        float m = -INFINITY, l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int j0 = 0; j0 < B; j0 += kPS)
          attend_page<DT>(q, kbv + j0 * kD * esz, kbv + (Bpad + j0) * kD * esz, min(kPS, B - j0),
                          d.scale_log2, m, l, acc, psw);
        const float inv = __frcp_rn(l);
        const float4 os = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        const float Ls = (m + __log2f(l)) * kLn2;
        if (slot < 0) {
          const float4 op = *reinterpret_cast<const float4*>(prm.o_p + grow * kD + 4 * lane);
          float4 o;
          float L;
          lse_merge(op, prm.l_p[grow], os, Ls, o, L);
          *reinterpret_cast<float4*>(prm.out + grow * kD + 4 * lane) = o;
          if (prm.out_lse && lane == 0) prm.out_lse[grow] = L;
        } else {
          float* dst = prm.sfx_g + (static_cast<size_t>(sg) * R + (i / B) * A + slot) * kPartStride;
          if (lane == 0) dst[0] = Ls;
          *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = os;
        }
      }
    }
  }
  if (!scan) return;

  // ---- active rows' queries for the bound: bf16 -> [R16][256] = [q- | q+]
  // in swizzled 16-byte chunks (ldmatrix); fp32 -> [R][128]
  const int R16 = (R + 15) / 16 * 16;
  if (DT == LOSA_BF16) {
#pragma unroll 1
    for (int e = tid; e < R16 * 32; e += kThreads) {
      const int r = e / 32, c = e % 32;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < R) {
        const int row = (r / A) * B + act_tok[r];
        const uint32_t* src = qcs + row * qw + 4 * (c & 15);
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t w = src[u];
          uint32_t lo16 = w & 0xffffu, hi16 = w >> 16;
          const bool nl = lo16 & 0x8000u, nh = hi16 & 0x8000u;
          if (c < 16) {  // q- = min(q, 0)
            lo16 = nl ? lo16 : 0u;
            hi16 = nh ? hi16 : 0u;
          } else {  // q+ = max(q, 0)
            lo16 = nl ? 0u : lo16;
            hi16 = nh ? 0u : hi16;
          }
          o[u] = lo16 | (hi16 << 16);
        }
        v = make_uint4(o[0], o[1], o[2], o[3]);
      }
      *reinterpret_cast<uint4*>(qrows + r * 512 + ((c ^ (r & 7)) << 4)) = v;
    }
  } else {
#pragma unroll 1
    for (int e = tid; e < R * kD; e += kThreads) {
      const int r = e / kD, c = e % kD;
      const int row = (r / A) * B + act_tok[r];
      reinterpret_cast<uint32_t*>(qrows)[r * kD + c] = qcs[row * qw + c];
    }
  }
  __syncthreads();  // the staging area becomes the score area below

  // ---- bound scores of the chunk
  const int ntm = R16 / 16;
#pragma unroll 1
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % prm.stages;
    const uint32_t parity = (t / prm.stages) & 1;
    if (!mbar_wait(&mbar[st], parity)) {
      atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
      *s_fail = 1;
    }
    __syncthreads();
    if (*s_fail) return;  // no cluster here: leaving early is safe
    const char* tile = ring + st * kStageBytes;
    const int np = min(prm.tile, npages - t * prm.tile);
    const int pl0 = t * prm.tile;
    if (DT == LOSA_BF16) {
      const int ntn = (np + 7) / 8;
      const int g4 = lane >> 2, t4 = lane & 3;
#pragma unroll 1
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
#pragma unroll 1
      for (int e = tid; e < np * R; e += kThreads) {
        const int pl = e % np, r = e / np;
        const int pg = p0 + pl0 + pl;
        const char* recp = tile + pl * prm.rec;
        const float* q = reinterpret_cast<const float*>(qrows) + r * kD;
        float acc = 0.f;
#pragma unroll 1
        for (int c = 0; c < kD / 4; ++c) {
          const float4 mn = *reinterpret_cast<const float4*>(recp + meta_swz(16u * c, pg));
          const float4 mx = *reinterpret_cast<const float4*>(recp + meta_swz(16u * (c + kD / 4), pg));
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
      bulk_g2s(ring + st * kStageBytes, meta_g + static_cast<size_t>(p0 + tn * prm.tile) * prm.rec,
               bytes, &mbar[st]);
    }
  }

  // ---- chunk-local top-k per row -> workspace
  unsigned long long* dst = prm.cand + (static_cast<size_t>(sg) * nchunk + chunk) * R * k;
  chunk_topk<DT, KP>(prm, sc, R, k, npages, p0, dst, fbuf, cbuf);
}

// ---------------------------------------------------------------------------
// K2: select, union, gather, combine
// ---------------------------------------------------------------------------
struct GatherLayout {
  int stage, qa, sel_own, sel_all, bitmap, wbase, lpages, masks, part, misc, ps, mbuf, mbar,
      total;
};

struct GatherParams {
  const void* qc;
  const void* K;
  const void* V;
  float* o_p;
  float* l_p;
  float* out;
  float* out_lse;
  int32_t* active_idx;
  int32_t* page_idx;
  int32_t* union_count;
  const int32_t* act_tok_g;
  const float* sfx_g;
  const unsigned long long* cand;
  int* status;
  Dims d;
  int CL;        // CTAs per cluster
  int max_lp;    // max union pages per CTA
  int ngp;       // pages in flight per CTA
  int qw;        // 32-bit words per staged query row (padded)
  GatherLayout lo;
};

// The k best chunk candidates of row r (keys, descending) -> out[0..k).
// Fast path: lane c holds chunk c's sorted list; threshold = k-th largest
// list head; the survivors are rank-sorted.  Fallback: sort-and-merge trees
// or k rounds of warp argmax.
template <int KP>
__device__ __forceinline__ void merge_row(const GatherParams& prm, int r, int sg,
                                          unsigned long long* out, unsigned long long* fb) {
  const Dims& d = prm.d;
  const int lane = threadIdx.x & 31, k = d.k, nc = d.nchunk, R = d.R;
  const unsigned long long* base = prm.cand + static_cast<size_t>(sg) * nc * R * k;
  if (KP > 0) {
    constexpr int KQ = KP > 0 ? KP : 1;
    unsigned long long x[KQ];
    {
      const unsigned long long* lst = base + (static_cast<size_t>(lane) * R + r) * k;
#pragma unroll
      for (int i = 0; i < KQ; ++i) x[i] = (lane < nc && i < k) ? __ldcg(lst + i) : 0ull;
    }
#pragma unroll 1
    for (int c = lane + 32; c < nc; c += 32) {  // more than 32 chunks: fold lists
      unsigned long long y[KQ];
      const unsigned long long* lst = base + (static_cast<size_t>(c) * R + r) * k;
#pragma unroll
      for (int i = 0; i < KQ; ++i) y[i] = i < k ? __ldcg(lst + i) : 0ull;
      merge_top<KQ>(x, y);
    }
    // threshold from the list heads (every list is sorted, descending)
    unsigned long long v = x[0];
#pragma unroll 1
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll 1
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, stride);
        const bool dir = (lane & size) == 0, lower = (lane & stride) == 0;
        v = (lower == dir) ? umax64(v, o) : (v < o ? v : o);
      }
    }
    const unsigned long long tau = __shfl_sync(0xffffffffu, v, k - 1);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < KQ; ++i) cnt += (x[i] >= tau && x[i] != 0ull);
    int incl = cnt;
#pragma unroll 1
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= kCandCap) {
      int pos = incl - cnt;
#pragma unroll
      for (int i = 0; i < KQ; ++i)
        if (x[i] >= tau && x[i] != 0ull) fb[pos++] = x[i];
      __syncwarp();
#pragma unroll 1
      for (int t = lane; t < total; t += 32) {
        const unsigned long long y = fb[t];
        int rank = 0;
#pragma unroll 4
        for (int m = 0; m < total; ++m) rank += fb[m] > y;
        if (rank < k) out[rank] = y;
      }
#pragma unroll 1
      for (int t = total + lane; t < k; t += 32) out[t] = 0ull;
    } else {
      group_merge<KQ>(x, 32);
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < KQ; ++i)
          if (i < k) out[i] = x[i];
      }
    }
    __syncwarp();
  } else {
    warp_topk([&](int i) { return __ldcg(base + (static_cast<size_t>(i / k) * R + r) * k + i % k); },
              nc * k, k, out, fb);
    __syncwarp();
  }
}

template <int DT>
__device__ __forceinline__ float4 qrow4(const uint32_t* qs, int row, int qw, int lane) {
  if (DT == LOSA_BF16) {
    const uint32_t w0 = qs[row * qw + 2 * lane], w1 = qs[row * qw + 2 * lane + 1];
    return make_float4(__uint_as_float(w0 << 16), __uint_as_float(w0 & 0xffff0000u),
                       __uint_as_float(w1 << 16), __uint_as_float(w1 & 0xffff0000u));
  }
  const uint32_t* w = qs + row * qw + 4 * lane;
  return make_float4(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]),
                     __uint_as_float(w[3]));
}

template <int DT, int KP>
__global__ void __launch_bounds__(kThreads, 2) losa_gather_kernel(const GatherParams prm) {
  extern __shared__ __align__(1024) char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const Dims& d = prm.d;
  const GatherLayout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = static_cast<int>(cluster.block_rank());
  const int CL = prm.CL;
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int esz = DT == LOSA_BF16 ? 2 : 4;
  const int pbytes = kPS * kD * esz;
  const int nwords = (d.P + 31) / 32;

  char* slots = smem + lo.stage;  // gather pages
  char* qa = smem + lo.qa;  // [R][kD] active rows' queries, element type
  int32_t* sel_own = reinterpret_cast<int32_t*>(smem + lo.sel_own);
  int32_t* sel_all = reinterpret_cast<int32_t*>(smem + lo.sel_all);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + lo.bitmap);
  int32_t* wbase = reinterpret_cast<int32_t*>(smem + lo.wbase);
  int32_t* lpages = reinterpret_cast<int32_t*>(smem + lo.lpages);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + lo.masks);
  float* part = reinterpret_cast<float*>(smem + lo.part);  // [R][kPartStride]
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  float* Ps = reinterpret_cast<float*>(smem + lo.ps);
  unsigned long long* mbuf = reinterpret_cast<unsigned long long*>(smem + lo.mbuf);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  int32_t* s_fail = misc;
  int32_t* s_U = misc + 1;
  int32_t* s_nlp = misc + 2;
  int32_t* act_tok = misc + 4;  // [R]
  float* psw = Ps + warp * 16;

  if (tid == 0) {
    for (int i = 0; i < kMaxGatherPages; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
    *s_fail = 0;
  }
#pragma unroll 1
  for (int e = tid; e < R * kPartStride; e += kThreads)  // empty partials
    part[e] = (e % kPartStride) == 0 ? -INFINITY : 0.f;

  // everything below reads what the scan kernel wrote
  asm volatile("griddepcontrol.wait;" ::: "memory");

#pragma unroll 1
  for (int r = tid; r < R; r += kThreads)
    act_tok[r] = __ldcg(prm.act_tok_g + static_cast<size_t>(sg) * R + r);
  __syncthreads();
  {  // active rows' queries (element type)
    const int cpr = kD * esz / 16;
#pragma unroll 1
    for (int e = tid; e < R * cpr; e += kThreads) {
      const int r = e / cpr, c = e - r * cpr;
      const size_t row = (static_cast<size_t>(s) * d.Hq + g * G + r / A) * B + act_tok[r];
      reinterpret_cast<uint4*>(qa)[e] =
          reinterpret_cast<const uint4*>(static_cast<const char*>(prm.qc) + row * kD * esz)[c];
    }
  }

  // ---- this CTA's rows (r % CL == rank): the row's k pages
  if (!d.all_pages) {
#pragma unroll 1
    for (int r = rank + CL * warp; r < R; r += CL * kWarps) {
      unsigned long long* best = mbuf + (kWarps + warp) * kCandCap;
      merge_row<KP>(prm, r, sg, best, mbuf + warp * kCandCap);
      int32_t* dst = sel_own + (r / CL) * k;
#pragma unroll 1
      for (int j = lane; j < k; j += 32) {  // pages in ascending order
        const int pj = key_index(best[j]);
        int rk = 0;
#pragma unroll 4
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
#pragma unroll 1
    for (int r = rank; r < R; r += CL) {
      const int hl = r / A, a = r % A;
#pragma unroll 1
      for (int j = tid; j < k; j += kThreads)
        prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + a) * k + j] = j;
    }
  }
  __syncthreads();
  cluster.sync();

  // ---- union of the group's pages and this CTA's share
  if (d.all_pages) {
    const int U = d.P;
    const int nlp = U > rank ? (U - rank + CL - 1) / CL : 0;
    if (tid == 0) {
      *s_nlp = nlp;
      if (rank == 0 && prm.union_count) prm.union_count[sg] = U;
    }
#pragma unroll 1
    for (int j = tid; j < min(nlp, prm.max_lp); j += kThreads) lpages[j] = rank + j * CL;
#pragma unroll 1
    for (int e = tid; e < min(nlp, prm.max_lp) * d.MW; e += kThreads) {
      const int w = e % d.MW;
      const int nb = min(32, R - 32 * w);
      masks[e] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
    }
  } else {
    const int rows_own = (R + CL - 1) / CL;
#pragma unroll 1
    for (int e = tid; e < R * k; e += kThreads) {
      const int r = e / k, j = e - r * k;
      sel_all[e] = cluster.map_shared_rank(sel_own, r % CL)[(r / CL) * k + j];
    }
    (void)rows_own;
#pragma unroll 1
    for (int w = tid; w < nwords; w += kThreads) bitmap[w] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int e = tid; e < R * k; e += kThreads) {
      const int p = sel_all[e];
      if (p >= 0 && p < d.P) atomicOr(&bitmap[p >> 5], 1u << (p & 31));
      else atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of word popcounts
      const int per = (nwords + 31) / 32;
      const int w0 = lane * per, w1 = min(nwords, w0 + per);
      int sum = 0;
#pragma unroll 1
      for (int w = w0; w < w1; ++w) sum += __popc(bitmap[w]);
      int incl = sum;
#pragma unroll 1
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
#pragma unroll 1
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
#pragma unroll 1
    for (int w = tid; w < nwords; w += kThreads) {
      uint32_t bits = bitmap[w];
      int pos = wbase[w];
#pragma unroll 1
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos % CL == rank && pos / CL < prm.max_lp) lpages[pos / CL] = w * 32 + b;
        ++pos;
      }
    }
#pragma unroll 1
    for (int e = tid; e < min(nlp, prm.max_lp) * d.MW; e += kThreads) masks[e] = 0u;
    __syncthreads();
#pragma unroll 1
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
  }
  __syncthreads();

  // ---- gather: this CTA's union pages, in batches of ngp; warp w folds the
  // pages of rows r = w, w + 8, ... into their partials (one writer per row)
  {
    const int nlp = min(*s_nlp, prm.max_lp);
#pragma unroll 1
    for (int b0 = 0; b0 < nlp && !*s_fail; b0 += prm.ngp) {
      const int nb = min(prm.ngp, nlp - b0);
      const int batch = b0 / prm.ngp;
      if (tid == 0) {
#pragma unroll 1
        for (int i = 0; i < nb; ++i) {
          const int p = lpages[b0 + i];
          const int ntok = min(kPS, d.L - p * kPS);
          const uint32_t bytes = static_cast<uint32_t>(ntok * kD * esz);
          const size_t off = (static_cast<size_t>(sg) * d.L + static_cast<size_t>(p) * kPS) * kD * esz;
          char* dst = slots + i * 2 * pbytes;
          mbar_expect_tx(&mbar[i], 2 * bytes);
          bulk_g2s(dst, static_cast<const char*>(prm.K) + off, bytes, &mbar[i]);
          bulk_g2s(dst + pbytes, static_cast<const char*>(prm.V) + off, bytes, &mbar[i]);
        }
      }
#pragma unroll 1
      for (int r = warp; r < R; r += kWarps) {
        bool have = false;
#pragma unroll 1
        for (int i = 0; i < nb; ++i) have |= (masks[(b0 + i) * d.MW + (r >> 5)] >> (r & 31)) & 1u;
        if (!have) continue;
        const float4 q = row4<DT>(qa, r, lane);
        float* pr = part + r * kPartStride;
        float m = pr[0], l = pr[1];
        float4 acc = *reinterpret_cast<const float4*>(pr + 4 + 4 * lane);
#pragma unroll 1
        for (int i = 0; i < nb; ++i) {
          if (!((masks[(b0 + i) * d.MW + (r >> 5)] >> (r & 31)) & 1u)) continue;
          if (!__all_sync(0xffffffffu, mbar_wait(&mbar[i], batch & 1))) {
            if (lane == 0) {
              atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
              *s_fail = 1;
            }
            break;
          }
          const int p = lpages[b0 + i];
          const char* Ks = slots + i * 2 * pbytes;
          attend_page<DT>(q, Ks, Ks + pbytes, min(kPS, d.L - p * kPS), d.scale_log2, m, l, acc,
                          psw);
        }
        __syncwarp();
        if (lane == 0) {
          pr[0] = m;
          pr[1] = l;
        }
        *reinterpret_cast<float4*>(pr + 4 + 4 * lane) = acc;
      }
      // every copy of this batch has landed before the slots are refilled
#pragma unroll 1
      for (int i = tid; i < nb; i += kThreads)
        if (!mbar_wait(&mbar[i], batch & 1)) *s_fail = 1;
      __syncthreads();
    }
  }
  __syncthreads();
  cluster.sync();

  // ---- combine every CTA's partial of this CTA's rows, cache write-back,
  // merge with the suffix
  if (!*s_fail) {
#pragma unroll 1
    for (int r = rank + CL * warp; r < R; r += CL * kWarps) {
      float M = -INFINITY;
#pragma unroll 1
      for (int c = 0; c < CL; ++c) M = fmaxf(M, cluster.map_shared_rank(part, c)[r * kPartStride]);
      float lsum = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (int c = 0; c < CL; ++c) {  // fixed order: deterministic
        const float* pr = cluster.map_shared_rank(part, c) + r * kPartStride;
        const float mc = pr[0];
        if (mc == -INFINITY) continue;  // this CTA held none of the row's pages
        const float w = exp2f(mc - M);
        lsum += w * pr[1];
        const float4 a = *reinterpret_cast<const float4*>(pr + 4 + 4 * lane);
        acc.x += w * a.x;
        acc.y += w * a.y;
        acc.z += w * a.z;
        acc.w += w * a.w;
      }
      const float inv = __frcp_rn(lsum);
      const float4 op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      const float Lp = (M + __log2f(lsum)) * kLn2;
      const int hl = r / A, t = act_tok[r];
      const size_t grow = (static_cast<size_t>(s) * d.Hq + g * G + hl) * B + t;
      *reinterpret_cast<float4*>(prm.o_p + grow * kD + 4 * lane) = op;
      if (lane == 0) prm.l_p[grow] = Lp;
      const float* sx = prm.sfx_g + (static_cast<size_t>(sg) * R + r) * kPartStride;
      const float4 os = __ldcg(reinterpret_cast<const float4*>(sx + 4 + 4 * lane));
      float4 o;
      float L;
      lse_merge(op, Lp, os, __ldcg(sx), o, L);
      *reinterpret_cast<float4*>(prm.out + grow * kD + 4 * lane) = o;
      if (prm.out_lse && lane == 0) prm.out_lse[grow] = L;
    }
  }
  // no CTA may leave while others can still read its shared memory
  cluster.sync();
}

// ---------------------------------------------------------------------------
// host side: launch geometry, shared-memory layouts, attributes
// ---------------------------------------------------------------------------
constexpr int kGatherSmemTarget = 110 * 1024;  // two gather CTAs per SM

int topk_width(int k) {
  if (k <= 2) return 2;
  if (k <= 4) return 4;
  if (k <= 8) return 8;
  if (k <= 16) return 16;
  return 0;  // warp fallback
}

bool plan_scan(const Dims& d, ScanParams* prm, int max_dyn) {
  prm->d = d;
  prm->rec = 2 * kD * d.esz;
  prm->tile = kStageBytes / prm->rec;  // 64 (bf16) or 32 (fp32) pages per stage
  prm->sc_stride = align_up(d.chunk_pages, 4) + 4;
  prm->qw = d.esz == 2 ? kD / 2 + 1 : kD + 1;
  prm->kp = topk_width(d.k);
  // a row's top-k group: at least k lanes, and enough lanes to cover the
  // CTA's rows in few passes
  prm->tpr = std::min(32, std::max(pow2_floor(std::max(1, kThreads / std::max(d.R, 1))),
                                   d.k <= 1 ? 1 : pow2_floor(2 * d.k - 1)));
  const bool selects = d.A > 0 && !d.all_pages;
  if (selects && prm->kp > 0 && prm->tpr < d.k) return false;
  if (selects && prm->kp == 0 && d.k > kCandCap) return false;
  const int R16 = (d.R + 15) / 16 * 16;
  const int GB = d.G * d.B;
  for (int ring = kMaxRingBytes; ring >= 64 * 1024; ring -= 32 * 1024) {
    ScanLayout& lo = prm->lo;
    int off = 0;
    auto take = [&](long long bytes, int align) {
      off = align_up(off, align);
      const int o = off;
      off += static_cast<int>(std::min<long long>(bytes, 1 << 30));
      return o;
    };
    lo.ring = take(ring, 1024);
    // scores, or (before the scan) the staged queries
    lo.scores = take(std::max(4LL * d.R * prm->sc_stride, 2LL * GB * prm->qw * 4), 16);
    lo.kbv = take(2LL * ((d.B + kPS - 1) / kPS * kPS) * kD * d.esz, 16);
    lo.qrows = take(R16 * 512, 128);
    lo.misc = take((4 + 3 * kMaxRowsPerGroup) * 4, 16);
    lo.ps = take(kWarps * 16 * 4, 16);
    lo.fbuf = take(prm->kp > 0 ? 8LL * (kThreads / prm->tpr) * kCandCap : 0, 16);
    lo.cbuf = take(prm->kp == 0 ? 2 * kWarps * kCandCap * 8 : 0, 16);
    lo.mbar = take((kMaxStages + 1) * 8, 8);
    lo.total = off;
    prm->stages = ring / kStageBytes;
    if (lo.total <= max_dyn) return true;
  }
  return false;
}

bool plan_gather(const Dims& d, GatherParams* prm, int max_dyn, int max_cluster) {
  prm->d = d;
  const int CL = std::min(max_cluster, std::max(1, std::max(d.Umax, 1)));
  prm->CL = CL;
  prm->max_lp = (d.Umax + CL - 1) / CL;
  prm->qw = d.esz == 2 ? kD / 2 + 1 : kD + 1;
  if (!d.all_pages && d.A > 0 && topk_width(d.k) == 0 && d.k > kCandCap) return false;
  const int nwords = (d.P + 31) / 32;
  const int pbytes = kPS * kD * d.esz;
  const int rows_per_cta = (d.R + CL - 1) / CL;
  for (int ngp = std::min(kMaxGatherPages, std::max(1, prm->max_lp)); ngp >= 1; ngp /= 2) {
    GatherLayout& lo = prm->lo;
    int off = 0;
    auto take = [&](long long bytes, int align) {
      off = align_up(off, align);
      const int o = off;
      off += static_cast<int>(std::min<long long>(bytes, 1 << 30));
      return o;
    };
    lo.stage = take(2LL * ngp * pbytes, 1024);
    lo.qa = take(1LL * d.R * kD * d.esz, 16);
    lo.sel_own = take(d.all_pages ? 0 : 4LL * rows_per_cta * d.k, 16);
    lo.sel_all = take(d.all_pages ? 0 : 4LL * d.R * d.k, 16);
    lo.bitmap = take(nwords * 4, 16);
    lo.wbase = take(nwords * 4, 16);
    lo.lpages = take(prm->max_lp * 4, 16);
    lo.masks = take(4LL * prm->max_lp * d.MW, 16);
    lo.part = take(4LL * d.R * kPartStride, 16);
    lo.misc = take((4 + kMaxRowsPerGroup) * 4, 16);
    lo.ps = take(kWarps * 16 * 4, 16);
    lo.mbuf = take(2 * kWarps * kCandCap * 8, 16);
    lo.mbar = take(kMaxGatherPages * 8, 8);
    lo.total = off;
    prm->ngp = ngp;
    if (lo.total <= std::min(max_dyn, kGatherSmemTarget) || (ngp == 1 && lo.total <= max_dyn))
      return true;
  }
  return false;
}

std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices] = {};
int g_attr_dyn[kMaxDevices] = {};
int g_attr_cluster[kMaxDevices] = {};

// Largest cluster size (16, 8, 4) of which at least one cluster of gather
// CTAs can be resident on the device.
int probe_cluster() {
  for (int cl = kMaxCluster; cl >= 4; cl /= 2) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cl, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(kGatherSmemTarget);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, losa_gather_kernel<LOSA_BF16, 8>, &cfg) == cudaSuccess &&
        n > 0)
      return cl;
    cudaGetLastError();  // clear a refused query
  }
  return 4;
}

template <int DT, int KP>
cudaError_t set_attrs_one(int optin, int* dyn) {
  const void* fns[2] = {reinterpret_cast<const void*>(losa_scan_kernel<DT, KP>),
                        reinterpret_cast<const void*>(losa_gather_kernel<DT, KP>)};
  for (int i = 0; i < 2; ++i) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, fns[i]);
    if (e != cudaSuccess) return e;
    const int mine = optin - static_cast<int>(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, mine);
    if (e != cudaSuccess) return e;
    if (i == 1) {
      e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    *dyn = std::min(*dyn, mine);
  }
  return cudaSuccess;
}

template <int DT>
cudaError_t set_attrs_dt(int optin, int* dyn) {
  cudaError_t e;
  if ((e = set_attrs_one<DT, 0>(optin, dyn)) != cudaSuccess) return e;
  if ((e = set_attrs_one<DT, 2>(optin, dyn)) != cudaSuccess) return e;
  if ((e = set_attrs_one<DT, 4>(optin, dyn)) != cudaSuccess) return e;
  if ((e = set_attrs_one<DT, 8>(optin, dyn)) != cudaSuccess) return e;
  return set_attrs_one<DT, 16>(optin, dyn);
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
    int dyn = optin;
    if ((e = set_attrs_dt<LOSA_BF16>(optin, &dyn)) != cudaSuccess) return record_cuda_error(e);
    if ((e = set_attrs_dt<LOSA_F32>(optin, &dyn)) != cudaSuccess) return record_cuda_error(e);
    g_attr_dyn[dev] = dyn;
    g_attr_cluster[dev] = probe_cluster();
    g_attr_done[dev] = true;
  }
  *max_dyn = g_attr_dyn[dev];
  *max_cluster = g_attr_cluster[dev];
  return LOSA_OK;
}

template <int DT, int KP>
cudaError_t launch_pair(const cudaLaunchConfig_t& c1, const ScanParams& sp,
                        const cudaLaunchConfig_t* c2, const GatherParams& gp) {
  const cudaError_t e = cudaLaunchKernelEx(&c1, losa_scan_kernel<DT, KP>, sp);
  if (e != cudaSuccess || !c2) return e;
  return cudaLaunchKernelEx(c2, losa_gather_kernel<DT, KP>, gp);
}

template <int DT>
cudaError_t launch_dt(int kp, const cudaLaunchConfig_t& c1, const ScanParams& sp,
                      const cudaLaunchConfig_t* c2, const GatherParams& gp) {
  switch (kp) {
    case 2: return launch_pair<DT, 2>(c1, sp, c2, gp);
    case 4: return launch_pair<DT, 4>(c1, sp, c2, gp);
    case 8: return launch_pair<DT, 8>(c1, sp, c2, gp);
    case 16: return launch_pair<DT, 16>(c1, sp, c2, gp);
    default: return launch_pair<DT, 0>(c1, sp, c2, gp);
  }
}

}  // namespace

bool fused_step_fits(const Dims& d, int max_dyn) {
  ScanParams sp;
  GatherParams gp;
  return plan_scan(d, &sp, max_dyn) && (d.A == 0 || plan_gather(d, &gp, max_dyn, kMaxCluster));
}

int launch_fused_step(const Dims& d, const void* q_cur, const void* q_prev, const void* k_prefix,
                      const void* v_prefix, const void* page_meta, const void* k_blk,
                      const void* v_blk, float* o_p, float* l_p, float* out, float* out_lse,
                      int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                      void* workspace, cudaStream_t st) {
  int max_dyn = 0, max_cluster = kMaxCluster;
  int rc = ensure_attributes(&max_dyn, &max_cluster);
  if (rc != LOSA_OK) return rc;
  ScanParams sp;
  GatherParams gp;
  if (!plan_scan(d, &sp, max_dyn)) return LOSA_ERR_UNSUPPORTED;
  if (d.A > 0 && !plan_gather(d, &gp, max_dyn, max_cluster)) return LOSA_ERR_UNSUPPORTED;
  if (d.S * d.Hkv > 65535 || d.nchunk > 65535) return LOSA_ERR_UNSUPPORTED;
  char* ws = static_cast<char*>(workspace);
  int* status = reinterpret_cast<int*>(ws + d.off_status);
  int32_t* act_tok = reinterpret_cast<int32_t*>(ws + d.off_act);
  float* sfx = reinterpret_cast<float*>(ws + d.off_sfx);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(ws + d.off_cand);

  sp.qc = q_cur;
  sp.qp = q_prev;
  sp.meta = static_cast<const char*>(page_meta);
  sp.kb = k_blk;
  sp.vb = v_blk;
  sp.o_p = o_p;
  sp.l_p = l_p;
  sp.out = out;
  sp.out_lse = out_lse;
  sp.active_idx = active_idx;
  sp.union_count = union_count;
  sp.act_tok_g = act_tok;
  sp.sfx_g = sfx;
  sp.cand = cand;
  sp.status = status;
  cudaLaunchConfig_t c1 = {};
  c1.gridDim = dim3(d.nchunk, d.S * d.Hkv, 1);
  c1.blockDim = dim3(kThreads, 1, 1);
  c1.dynamicSmemBytes = static_cast<size_t>(sp.lo.total);
  c1.stream = st;

  gp.qc = q_cur;
  gp.K = k_prefix;
  gp.V = v_prefix;
  gp.o_p = o_p;
  gp.l_p = l_p;
  gp.out = out;
  gp.out_lse = out_lse;
  gp.page_idx = page_idx;
  gp.union_count = union_count;
  gp.act_tok_g = act_tok;
  gp.sfx_g = sfx;
  gp.cand = cand;
  gp.status = status;
  cudaLaunchConfig_t c2 = {};
  cudaLaunchAttribute attr[2];
  if (d.A > 0) {
    c2.gridDim = dim3(gp.CL, d.S * d.Hkv, 1);
    c2.blockDim = dim3(kThreads, 1, 1);
    c2.dynamicSmemBytes = static_cast<size_t>(gp.lo.total);
    c2.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = gp.CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;  // overlaps the scan kernel
    c2.attrs = attr;
    c2.numAttrs = 2;
  }
  // one top-k width per compiled kernel: the selection code of the others is
  // never fetched
  const int kp = (d.A > 0 && !d.all_pages) ? sp.kp : 2;
  const cudaLaunchConfig_t* c2p = d.A > 0 ? &c2 : nullptr;
  const cudaError_t e = d.dtype == LOSA_BF16 ? launch_dt<LOSA_BF16>(kp, c1, sp, c2p, gp)
                                             : launch_dt<LOSA_F32>(kp, c1, sp, c2p, gp);
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}

}  // namespace losa
