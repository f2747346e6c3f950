// step_fused.cu -- one LoSA denoising step in three kernel launches.
//
// LoSA paper, methodology: locality pruning (MSE of Q_t vs Q_{t-1}, top-|A|
// per head), reuse of the cached prefix state for stable tokens, QUEST page
// selection for active queries only, union of the selected pages, sparse
// prefix attention, dense intra-block suffix, online-softmax merge, cache
// update.
//
// K1 `losa_scan_kernel` -- a flat grid over the SMs: each CTA owns one chunk
//    of one (sequence, KV head) group's pages.  At launch it bulk-copies (TMA)
//    the group's current and previous queries and the chunk's page metadata
//    into shared memory; the locality score (lanes split a row's channels)
//    and the active set (one warp per head, lane = token) follow as soon as
//    the queries land, then the QUEST bound of the chunk's pages for the
//    group's R active rows -- bf16: tensor cores, U = [q- | q+] . [kmin ;
//    kmax] with mma.sync m16n8k16 (exact products, fp32 accumulation, the
//    A operand held in registers); fp32: CUDA cores, the sum in channel order
//    with one rounding per operation -- and a chunk-local top-k per row into
//    the workspace.  The first CTA of a group also stores the active set.
// K2 `losa_gather_kernel` -- CL CTAs per group, launched with programmatic
//    dependent launch behind K1.  Each CTA stages the block's K/V before K1
//    has finished; then it merges the chunk candidates of every active row
//    into the row's k pages and builds the group's page union (ascending,
//    with a row mask per page); union slot u belongs to CTA u % CL, which
//    copies the page's K and V once for the whole GQA group.  While the
//    copies fly the CTA computes the dense suffix of its share of the block's
//    token rows (stable rows are merged with their untouched cache and
//    finished here).  The pages are then folded into one online-softmax
//    partial per row -- bf16: tensor cores, all rows of an m16 tile at once
//    with a row mask, S = Q K^T and O += P V with P split into bf16 high and
//    remainder parts; fp32: one warp per row on CUDA cores.  The partials go
//    to the workspace (L2).
// K3 `losa_combine_kernel` -- one warp per active row, launched with
//    programmatic dependent launch behind K2: merges the row's non-empty
//    partials, writes the new o_p / L_p and merges them with the row's
//    suffix into the output.
//
// K1's waits on bulk copies are bounded (clock64); a wait that gives up sets
// LOSA_ERR_DEVICE_TIMEOUT in the status word and the CTA stops.  K2 waits on
// its own cp.async groups only; no CTA waits for another.
#include <algorithm>
#include <mutex>

#include "losa_common.cuh"
#include "ptx.cuh"

namespace losa {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxRingBytes = 128 * 1024;
constexpr int kStageBytes = 32 * 1024;
constexpr int kMaxStages = kMaxRingBytes / kStageBytes;
constexpr int kCandCap = 64;                     // per-warp compaction buffer
constexpr int kTopkW = 16;                       // lanes per row in the chunk top-k
constexpr int kThreadsG = 512;                   // gather kernel: one warp per merged row
constexpr int kWarpsG = kThreadsG / 32;
constexpr int kPageWarps = 8;                    // gather kernel: warps sharing an m16 tile's pages
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

// The k-th largest (1 <= k <= W) of the values held by the W lanes of an
// aligned lane group (W a power of two, the same for the whole warp): every
// lane ranks its value against the group's (ties by lane), and the lane of
// rank k-1 holds the answer.  The W shuffles are independent, so they
// overlap instead of forming a chain.
__device__ __forceinline__ unsigned long long group_kth_u64(unsigned long long v, int W, int k) {
  const int lane = threadIdx.x & 31, j = lane & (W - 1), base = lane - j;
  int rk = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i < W) {
      const unsigned long long o = __shfl_sync(0xffffffffu, v, base + i);
      rk += (o > v) || (o == v && i < j);
    }
  }
  const unsigned bal = __ballot_sync(0xffffffffu, rk == k - 1);
  const unsigned grp = W == 32 ? bal : ((bal >> base) & ((1u << W) - 1u));
  return __shfl_sync(0xffffffffu, v, base + __ffs(grp) - 1);
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
    const unsigned long long tau = group_kth_u64(lmax, 32, k);
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

// Top-k (k <= W) of a row of n <= W * NV bound scores in shared memory
// (score i is page p0 + i) by a group of W lanes (aligned inside the warp):
// lane j holds scores j, j + W, ...  The threshold tau is the k-th largest of
// the lanes' maxima: at least k scores reach it, so every score of the top k
// does.  Only the scores >= tau (at most kCandCap) become selection keys;
// they are compacted into buf and rank-sorted into out[0..k) (0 = empty when
// n < k).  Returns false, for every lane of the warp and before writing
// anything, if an active group of the warp had more than kCandCap survivors.
// W and NV are compile-time so that every loop is unrolled without guards
// (one copy per (W, NV) pair, shared by all kernels).
template <int W, int NV>
__device__ __noinline__ bool row_topk(const float* row, int n, int p0, int k,
                                      unsigned long long* buf, unsigned long long* out,
                                      bool active) {
  const int lane = threadIdx.x & 31;
  const int j = lane & (W - 1), base = lane - j;
  const unsigned gmask = W == 32 ? 0xffffffffu : (((1u << (W & 31)) - 1u) << base);
  const unsigned lt = (1u << lane) - 1u;
  float v[NV];
  float lmax = -INFINITY;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    v[t] = j + t * W < n ? row[j + t * W] : -INFINITY;
    lmax = fmaxf(lmax, v[t]);
  }
  // tau: the k-th largest lane maximum (rank by value, ties by lane), the
  // maxima read back from shared memory (broadcast loads, no shuffle chain)
  float* mx = reinterpret_cast<float*>(buf);
  mx[j] = lmax;
  __syncwarp();
  int rk = 0;
#pragma unroll
  for (int i = 0; i < W; ++i) {
    const float o = mx[i];
    rk += (o > lmax) || (o == lmax && i < j);
  }
  const unsigned bal = __ballot_sync(0xffffffffu, rk == k - 1) & gmask;
  const float tau = mx[__ffs(bal) - 1 - base];
  // survivors: one ballot per register slot gives every lane its positions
  unsigned bl[NV];
  int total = 0;
#pragma unroll
  for (int t = 0; t < NV; ++t) {
    bl[t] = __ballot_sync(0xffffffffu, j + t * W < n && v[t] >= tau) & gmask;
    total += __popc(bl[t]);
  }
  if (!__all_sync(0xffffffffu, !active || total <= kCandCap)) return false;
  __syncwarp();  // the maxima are read before buf takes the survivors
  if (active) {
    int pos = 0;
#pragma unroll
    for (int t = 0; t < NV; ++t) {
      if ((bl[t] >> lane) & 1u) buf[pos + __popc(bl[t] & lt)] = sel_key(v[t], p0 + j + t * W);
      pos += __popc(bl[t]);
    }
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

// Byte offset of 16-byte chunk c of row j inside a [rows][kD] tile: bf16 tiles
// XOR-swizzle the chunks by row (conflict-free ldmatrix), fp32 tiles are plain.
template <int DT>
__device__ __forceinline__ int tile_off(int j, int c) {
  return DT == LOSA_BF16 ? j * 256 + ((c ^ (j & 7)) << 4) : j * 512 + c * 16;
}

// fp32 sum of squared differences of two bf16x2 / f32 words, in channel order.
__device__ __forceinline__ float sqd_bf16x2(uint32_t a, uint32_t b, float acc) {
  const float d0 = __fsub_rn(__uint_as_float(a << 16), __uint_as_float(b << 16));
  acc = __fadd_rn(acc, __fmul_rn(d0, d0));
  const float d1 = __fsub_rn(__uint_as_float(a & 0xffff0000u), __uint_as_float(b & 0xffff0000u));
  return __fadd_rn(acc, __fmul_rn(d1, d1));
}
__device__ __forceinline__ float sqd_f32(uint32_t a, uint32_t b, float acc) {
  const float d0 = __fsub_rn(__uint_as_float(a), __uint_as_float(b));
  return __fadd_rn(acc, __fmul_rn(d0, d0));
}

// ---------------------------------------------------------------------------
// K1: scan
// ---------------------------------------------------------------------------
struct ScanLayout {
  int ring, qc, qps, qrows, misc, fbuf, cbuf, mbar, total;
};

struct ScanParams {
  const void* qc;
  const void* qp;
  const char* meta;
  int32_t* act_g;                  // workspace [S*Hkv][R + G*B]: act_tok, then act_slot
  int32_t* active_idx;
  unsigned long long* cand;        // workspace [S*Hkv][nchunk][R][k]
  int* status;
  Dims d;
  int scan;       // this launch scores pages (else: the active set only)
  int rec;        // bytes per metadata record
  int tile;       // pages per ring stage
  int stages;     // ring stages
  int sc_stride;  // floats per score row
  int kp;         // register top-k width (2..16), 0 = warp fallback
  int tpr;        // threads per row for the chunk top-k
  int nv;         // scores per top-k lane (a power of two >= chunk_pages / tpr)
  int mse_t;      // threads per row for the locality score
  ScanLayout lo;
};

// Chunk-local top-k of every active row -> dst_base[r][0..k).  Fast path
// (k <= 16): the threshold filter over a group of W >= k lanes per row, rows
// in passes of kThreads / W; a warp whose groups overflow the filter buffer
// falls back to register sort-and-merge.  k > 16: one warp per row.
template <int DT, int KP, int NV>
__device__ __forceinline__ void chunk_topk(const ScanParams& prm, const float* sc, int R, int k,
                                           int npages, int p0, unsigned long long* dst_base,
                                           unsigned long long* fbuf, unsigned long long* cbuf) {
  const int tid = threadIdx.x;
  if (KP > 0) {
    constexpr int W = kTopkW;
    const int rows_per_pass = kThreads / W;
#pragma unroll 1
    for (int r0 = 0; r0 < R; r0 += rows_per_pass) {
      const int r = r0 + tid / W;
      const bool active = r < R;
      const float* row = sc + (active ? r : 0) * prm.sc_stride;
      unsigned long long* out = dst_base + static_cast<size_t>(active ? r : 0) * k;
      auto key = [&](int i) { return sel_key(row[i], p0 + i); };
      bool done = false;
      if constexpr (NV > 0)
        done = row_topk<W, NV>(row, npages, p0, k, fbuf + (tid / W) * kCandCap, out, active);
      if (!done) {
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

// Bound scores of one 8-page n-tile for the 16 rows of the A fragments:
// acc[0..1] = rows g4, pages 2*t4, 2*t4+1; acc[2..3] = row g4 + 8.  `rec0`
// points to the tile's first record; records are [kmin | kmax] with 16-byte
// chunks swizzled by the page index (which is congruent to the record index
// mod 8 inside a ring stage).
__device__ __forceinline__ void bound_ntile(const uint32_t (&a)[16][4], const char* rec0,
                                            float (&acc)[4]) {
  const int lane = threadIdx.x & 31;
  const int pg = lane & 7;
  acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 16; ks += 2) {
    uint32_t b0, b1, b2, b3;
    const int ch = ks * 2 + (lane >> 3);
    ldsm_x4(su32(rec0 + pg * 512 + ((ch ^ pg) << 4)), b0, b1, b2, b3);
    mma_bf16(acc, a[ks], b0, b1);
    mma_bf16(acc, a[ks + 1], b2, b3);
  }
}

template <int DT, int KP, int NV>
__global__ void __launch_bounds__(kThreads, 1) losa_scan_kernel(const ScanParams prm) {
  extern __shared__ __align__(1024) char smem[];
  const Dims& d = prm.d;
  const ScanLayout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x;
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int GB = G * B;
  constexpr int rowb = DT == LOSA_BF16 ? kD * 2 : kD * 4;

  // launched behind the previous kernel of the stream (programmatic
  // dependent launch): every thread waits for it to complete before reading
  // any input (the sequence's length included) or touching anything it may
  // write; only then may the gather kernel be scheduled, since that kernel
  // stages the block's K/V (an input of this call) before its own wait
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  char* ring = smem + lo.ring;
  const char* qcs = smem + lo.qc;
  const char* qps = smem + lo.qps;
  float* sc = reinterpret_cast<float*>(smem + lo.qps);  // scores, after the locality pass
  char* qrows = smem + lo.qrows;
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  unsigned long long* fbuf = reinterpret_cast<unsigned long long*>(smem + lo.fbuf);
  unsigned long long* cbuf = reinterpret_cast<unsigned long long*>(smem + lo.cbuf);
  uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + lo.mbar);
  int32_t* s_fail = misc;
  float* s_mse = reinterpret_cast<float*>(misc + 4);
  int32_t* act_tok = misc + 4 + kMaxRowsPerGroup;
  int32_t* act_row = act_tok + kMaxRowsPerGroup;

  const int p0 = chunk * d.chunk_pages;
  // this chunk's pages of the sequence
  const int npages =
      prm.scan ? max(0, min((seq_len(d, s) + kPS - 1) / kPS, p0 + d.chunk_pages) - p0) : 0;
  const int ntiles = (npages + prm.tile - 1) / prm.tile;
  const char* meta_g = prm.meta + static_cast<size_t>(sg) * d.Pc * prm.rec;
  const uint32_t qbytes = static_cast<uint32_t>(GB * rowb);

  if (tid == 0) {
    for (int i = 0; i < kMaxStages + 1; ++i) mbar_init(&mbar[i], 1);
    fence_mbar_init();
    *s_fail = 0;
    if (chunk == 0 && g == 0 && seq_len_bad(d, s)) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
    const size_t qoff = (static_cast<size_t>(s) * d.Hq + g * G) * B * rowb;
    mbar_expect_tx(&mbar[kMaxStages], 2 * qbytes);
    bulk_g2s(smem + lo.qc, static_cast<const char*>(prm.qc) + qoff, qbytes, &mbar[kMaxStages]);
    bulk_g2s(smem + lo.qps, static_cast<const char*>(prm.qp) + qoff, qbytes, &mbar[kMaxStages]);
#pragma unroll 1
    for (int t = 0; t < min(ntiles, prm.stages); ++t) {
      const int np = min(prm.tile, npages - t * prm.tile);
      const uint32_t bytes = static_cast<uint32_t>(np * prm.rec);
      mbar_expect_tx(&mbar[t], bytes);
      bulk_g2s(ring + t * kStageBytes, meta_g + static_cast<size_t>(p0 + t * prm.tile) * prm.rec,
               bytes, &mbar[t]);
    }
  }
  __syncthreads();
  if (!mbar_wait(&mbar[kMaxStages], 0)) *s_fail = 1;
  __syncthreads();
  if (*s_fail) {
    if (tid == 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
    return;
  }

  // ---- locality score: mse_t lanes per row, each keeping four running
  // sums over its channels (fp32, one rounding per operation), then a
  // shuffle tree
  {
    const int T = prm.mse_t;
    const int row = tid / T, part = tid % T;
    float acc = 0.f;
    if (row < GB) {  // four running sums (one per 32-bit word of a chunk), added at the end
      constexpr int cpr = rowb / 16;
      const uint4* x = reinterpret_cast<const uint4*>(qcs + row * rowb);
      const uint4* y = reinterpret_cast<const uint4*>(qps + row * rowb);
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 4
      for (int c = part; c < cpr; c += T) {
        const uint4 a = x[c], b = y[c];
        if (DT == LOSA_BF16) {
          a0 = sqd_bf16x2(a.x, b.x, a0);
          a1 = sqd_bf16x2(a.y, b.y, a1);
          a2 = sqd_bf16x2(a.z, b.z, a2);
          a3 = sqd_bf16x2(a.w, b.w, a3);
        } else {
          a0 = sqd_f32(a.x, b.x, a0);
          a1 = sqd_f32(a.y, b.y, a1);
          a2 = sqd_f32(a.z, b.z, a2);
          a3 = sqd_f32(a.w, b.w, a3);
        }
      }
      acc = (a0 + a1) + (a2 + a3);
    }
#pragma unroll 1
    for (int o = 1; o < T; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (row < GB && part == 0) s_mse[row] = acc * (1.0f / kD);  // exact: kD is a power of two
  }
  __syncthreads();

  // ---- active set: one warp per head, lane = token; rank by (mse desc,
  // token asc), slot = active tokens before it
  {
    int32_t* act_g = prm.act_g + static_cast<size_t>(sg) * (R + GB);
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
      const int slot = __popc(bal & ((1u << lane) - 1u));
      if (act) {
        act_tok[h * A + slot] = lane;
        act_row[h * A + slot] = h * B + lane;  // the row's query in the staged group
      }
      if (chunk == 0) {
        if (lane < B) act_g[R + h * B + lane] = act ? slot : -1;
        if (act) {
          act_g[h * A + slot] = lane;
          if (prm.active_idx)
            prm.active_idx[(static_cast<size_t>(s) * d.Hq + g * G + h) * A + slot] = lane;
        }
      }
    }
  }
  __syncthreads();
  if (npages == 0) return;  // past the sequence's end: the gather kernel reads no list of it

  // ---- active rows' queries for the bound: bf16 -> [R16][256] = [q- | q+]
  // in swizzled 16-byte chunks (ldmatrix); fp32 -> [R][128]
  const int R16 = (R + 15) / 16 * 16;
  if (DT == LOSA_BF16) {
#pragma unroll 1
    for (int e = tid; e < R16 * 32; e += kThreads) {
      const int r = e / 32, c = e % 32;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (r < R) {
        const uint4 w4 = *reinterpret_cast<const uint4*>(qcs + act_row[r] * rowb + (c & 15) * 16);
        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
        uint32_t o[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t lo16 = w[u] & 0xffffu, hi16 = w[u] >> 16;
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
      reinterpret_cast<uint32_t*>(qrows)[r * kD + c] =
          reinterpret_cast<const uint32_t*>(qcs + act_row[r] * rowb)[c];
    }
  }
  __syncthreads();  // the previous queries' staging area becomes the score area

  // ---- bound scores of the chunk
  if (DT == LOSA_BF16) {
    const int ntm = R16 / 16;         // 1..8
    const int wpm = kWarps / ntm;     // warps per m16 tile
    const int mt = warp / wpm, sub = warp % wpm;
    const bool sw = mt < ntm;
    const int g4 = lane >> 2, t4 = lane & 3;
    uint32_t a[16][4];
    if (sw) {
      const int mi = lane >> 3, row = mt * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks) {
        const int ch = ks * 2 + (mi >> 1);
        ldsm_x4(su32(qrows + row * 512 + ((ch ^ (row & 7)) << 4)), a[ks][0], a[ks][1], a[ks][2],
                a[ks][3]);
      }
    }
    const int r0 = mt * 16 + g4;
    auto put = [&](const float (&acc)[4], int pc) {  // pc: chunk page of the lane's pair
      if (r0 < R) {
        sc[r0 * prm.sc_stride + pc] = acc[0];
        sc[r0 * prm.sc_stride + pc + 1] = acc[1];
      }
      if (r0 + 8 < R) {
        sc[(r0 + 8) * prm.sc_stride + pc] = acc[2];
        sc[(r0 + 8) * prm.sc_stride + pc + 1] = acc[3];
      }
    };
    if (ntiles <= prm.stages) {
      // every stage was issued at launch: each warp runs through its n-tiles,
      // two at a time, waiting only for the stage that holds them
      const int nnt = (npages + 7) / 8;
      const int ntpt = prm.tile / 8;  // n-tiles per stage
#pragma unroll 1
      for (int nt = sub; sw && nt < nnt; nt += 2 * wpm) {
        const int nu = nt + wpm < nnt ? nt + wpm : nt;
        const int t0 = nt / ntpt, t1 = nu / ntpt;
        if (!mbar_wait(&mbar[t0], 0) || !mbar_wait(&mbar[t1], 0)) {
          *s_fail = 1;
          break;
        }
        float acc0[4], acc1[4];
        bound_ntile(a, ring + t0 * kStageBytes + (nt - t0 * ntpt) * 8 * 512, acc0);
        bound_ntile(a, ring + t1 * kStageBytes + (nu - t1 * ntpt) * 8 * 512, acc1);
        put(acc0, nt * 8 + 2 * t4);
        if (nu != nt) put(acc1, nu * 8 + 2 * t4);
      }
      __syncthreads();
    } else {
#pragma unroll 1
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % prm.stages;
        const uint32_t parity = (t / prm.stages) & 1;
        if (!mbar_wait(&mbar[st], parity)) *s_fail = 1;
        __syncthreads();
        if (*s_fail) break;
        const int np = min(prm.tile, npages - t * prm.tile);
        const int ntn = (np + 7) / 8;
#pragma unroll 1
        for (int nt = sub; sw && nt < ntn; nt += wpm) {
          float acc[4];
          bound_ntile(a, ring + st * kStageBytes + nt * 8 * 512, acc);
          put(acc, t * prm.tile + nt * 8 + 2 * t4);
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
      __syncthreads();
    }
  } else {
#pragma unroll 1
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % prm.stages;
      const uint32_t parity = (t / prm.stages) & 1;
      if (!mbar_wait(&mbar[st], parity)) *s_fail = 1;
      __syncthreads();
      if (*s_fail) break;
      const char* tile = ring + st * kStageBytes;
      const int np = min(prm.tile, npages - t * prm.tile);
      const int pl0 = t * prm.tile;
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
      __syncthreads();
      if (tid == 0 && t + prm.stages < ntiles) {
        const int tn = t + prm.stages;
        const int npn = min(prm.tile, npages - tn * prm.tile);
        const uint32_t bytes = static_cast<uint32_t>(npn * prm.rec);
        mbar_expect_tx(&mbar[st], bytes);
        bulk_g2s(ring + st * kStageBytes, meta_g + static_cast<size_t>(p0 + tn * prm.tile) * prm.rec,
                 bytes, &mbar[st]);
      }
    }
    __syncthreads();
  }
  if (*s_fail) {
    if (tid == 0) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_TIMEOUT);
    return;
  }

  // ---- chunk-local top-k per row -> workspace
  unsigned long long* dst = prm.cand + (static_cast<size_t>(sg) * gridDim.x + chunk) * R * k;
  chunk_topk<DT, KP, NV>(prm, sc, R, k, npages, p0, dst, fbuf, cbuf);
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

// Fold one page (K, V: [16][256 B] bf16, chunks swizzled by key) into the
// state of the 16 query rows at q16 ([16][256 B], swizzled).  Row i of the
// tile takes part iff bit i of `rows` is set; keys >= ntok are masked (their
// V rows must be finite: the loaders zero-fill them).
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
      ldsm_x4(su32(Kp + key * 256 + ((ch ^ (key & 7)) << 4)), b0, b1, b2, b3);
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
    ldsm_x4_trans(su32(Vp + key * 256 + ((ch ^ (key & 7)) << 4)), b0, b1, b2, b3);
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

// Partial of the tile's rows i < nrows -> base[i] = (m, l, -, -, o[128]).
__device__ __forceinline__ void tile_store(const TileAcc& t, float* base, int nrows) {
  const int lane = threadIdx.x & 31, g4 = lane >> 2, t4 = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = g4 + 8 * h;
    if (i >= nrows) continue;
    float* pr = base + i * kPartStride;
    if (t4 == 0) {
      pr[0] = t.m[h];
      pr[1] = t.l[h];
    }
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<float2*>(pr + 4 + n * 8 + 2 * t4) = make_float2(t.o[n][2 * h], t.o[n][2 * h + 1]);
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
// K2: select, union, gather, suffix, combine
// ---------------------------------------------------------------------------
struct GatherLayout {
  int region;   // gathered pages; afterwards the per-warp partials
  int kbv;      // the block's K then V (bpad rows each)
  int qa;       // active rows' queries (bf16: [R16][256 B] swizzled; fp32: [R][512 B])
  int qs;       // this CTA's suffix rows' queries (same formats)
  int ocache;   // cached o_p rows of this CTA's stable suffix rows
  int lcache;   // their cached L_p
  int sel_all, bitmap, wbase, lpages, masks, part, misc, ps, mbuf;
  int total;
};

struct GatherParams {
  const void* qc;
  const void* K;
  const void* V;
  const void* kb;
  const void* vb;
  float* o_p;
  float* l_p;
  float* out;
  float* out_lse;
  int32_t* page_idx;
  int32_t* union_count;
  void* qref;       // drift-safe locality: active rows' q_cur written here (may be null)
  const int32_t* act_g;
  const unsigned long long* cand;
  float* part_g;    // workspace [S*Hkv][CL][R][kPartStride]: every CTA's row partials
  float* sfx_g;     // workspace [S*Hkv][R][kPartStride]: active rows' suffix (L_s, -, -, -, o_s)
  int* status;
  Dims d;
  int CL;        // CTAs per group
  int max_lp;    // max union pages per CTA
  int ngp;       // pages in flight per CTA
  int n_oa;      // max active rows owned per CTA
  int n_os;      // max stable suffix rows per CTA
  int wpart;     // bf16: warps split pages and keep per-warp partials
  GatherLayout lo;
};

// The k best chunk candidates of row r (keys, descending) -> out[0..k).
// Fast path: lane c holds chunk c's sorted list (lists past 32 folded in by
// bitonic merges), then a k-way merge by warp max-reductions over the list
// heads.  Fallback (k > 16): k rounds of warp argmax over all candidates.
// base: the group's lists [nchunk][R][k] (written by the scan kernel: read
// through L2, not L1), of which the first nc cover the sequence's pages
template <int KP>
__device__ __forceinline__ void merge_row(const GatherParams& prm, int r, int nc,
                                          const unsigned long long* base,
                                          unsigned long long* out, unsigned long long* fb,
                                          unsigned long long* hb) {
  const Dims& d = prm.d;
  const int lane = threadIdx.x & 31, k = d.k, R = d.R;
  if (KP > 0) {
    constexpr int KQ = KP > 0 ? KP : 1;
    unsigned long long x[KQ];
    {
      const unsigned long long* lst = base + (static_cast<size_t>(lane) * R + r) * k;
      if (KQ >= 2 && k == KQ && lane < nc) {  // 16-byte loads (k even: 16-byte aligned lists)
#pragma unroll
        for (int i = 0; i < KQ / 2; ++i) {
          const ulonglong2 v = __ldcg(reinterpret_cast<const ulonglong2*>(lst) + i);
          x[2 * i] = v.x;
          x[(2 * i + 1) % KQ] = v.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < KQ; ++i) x[i] = (lane < nc && i < k) ? __ldcg(lst + i) : 0ull;
      }
    }
#pragma unroll 1
    for (int c = lane + 32; c < nc; c += 32) {  // more than 32 chunks: fold lists
      unsigned long long y[KQ];
      const unsigned long long* lst = base + (static_cast<size_t>(c) * R + r) * k;
#pragma unroll
      for (int i = 0; i < KQ; ++i) y[i] = i < k ? __ldcg(lst + i) : 0ull;
      merge_top<KQ>(x, y);
    }
    // k-way merge of the sorted lists (one per lane, descending): each round
    // a warp maximum over the list heads (high then low key half; keys are
    // unique) is the next key, and the list that held it pops its head
#pragma unroll 1
    for (int it = 0; it < k; ++it) {
      const uint32_t hhi = static_cast<uint32_t>(x[0] >> 32), hlo = static_cast<uint32_t>(x[0]);
      const uint32_t mhi = __reduce_max_sync(0xffffffffu, hhi);
      const uint32_t mlo = __reduce_max_sync(0xffffffffu, hhi == mhi ? hlo : 0u);
      if (lane == 0) out[it] = (static_cast<unsigned long long>(mhi) << 32) | mlo;
      if (x[0] != 0ull && hhi == mhi && hlo == mlo) {
#pragma unroll
        for (int i = 0; i + 1 < KQ; ++i) x[i] = x[i + 1];
        x[KQ - 1] = 0ull;
      }
    }
    __syncwarp();
  } else {
    warp_topk([&](int i) { return __ldcg(base + (static_cast<size_t>(i / k) * R + r) * k + i % k); },
              nc * k, k, out, fb);
    __syncwarp();
  }
}

template <int DT, int KP>
__global__ void __launch_bounds__(kThreadsG, 1) losa_gather_kernel(const GatherParams prm) {
  extern __shared__ __align__(1024) char smem[];
  const Dims& d = prm.d;
  const GatherLayout& lo = prm.lo;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g4 = lane >> 2, t4 = lane & 3;
  const int rank = blockIdx.x;  // this CTA's place among the group's CL CTAs
  constexpr int CL = kGatherCtas;
  static_assert((CL & (CL - 1)) == 0 && CL <= 32, "CTAs per group: a power of two, at most a warp");
  const int sg = blockIdx.y;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const int G = d.G, B = d.B, A = d.A, R = d.R, k = d.k;
  const int GB = G * B;
  constexpr int rowb = DT == LOSA_BF16 ? kD * 2 : kD * 4;
  constexpr int cpr = rowb / 16;  // 16-byte chunks per row
  constexpr int pbytes = kPS * rowb;
  const int bpad = (B + kPS - 1) / kPS * kPS;
  const int nwords = (d.P + 31) / 32;
  const size_t grow0 = (static_cast<size_t>(s) * d.Hq + g * G) * B;  // the group's first row

  char* region = smem + lo.region;
  char* kbv = smem + lo.kbv;
  char* qa = smem + lo.qa;
  char* qs = smem + lo.qs;
  float* ocache = reinterpret_cast<float*>(smem + lo.ocache);
  float* lcache = reinterpret_cast<float*>(smem + lo.lcache);
  int32_t* sel_all = reinterpret_cast<int32_t*>(smem + lo.sel_all);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + lo.bitmap);
  int32_t* wbase = reinterpret_cast<int32_t*>(smem + lo.wbase);
  int32_t* lpages = reinterpret_cast<int32_t*>(smem + lo.lpages);
  uint32_t* masks = reinterpret_cast<uint32_t*>(smem + lo.masks);
  float* part = reinterpret_cast<float*>(smem + lo.part);  // [R][kPartStride] (fp32 path)
  float* part_cta = prm.part_g + (static_cast<size_t>(sg) * CL + rank) * R * kPartStride;
  int32_t* misc = reinterpret_cast<int32_t*>(smem + lo.misc);
  float* Ps = reinterpret_cast<float*>(smem + lo.ps);
  unsigned long long* mbuf = reinterpret_cast<unsigned long long*>(smem + lo.mbuf);
  int32_t* s_nlp = misc + 1;
  int32_t* s_len = misc + 2;           // the sequence's prefix length (kept out of registers)
  int32_t* s_wt = misc + 4;            // stable tokens per 32-token warp slice
  int32_t* s_wsum = misc + 8;          // union words' popcounts per warp of the union half
  int32_t* act_tok = misc + 16;        // [R], then act_slot [GB]
  int32_t* act_slot = act_tok + R;
  int32_t* sfx_tok = act_slot + GB;    // [n_oa + n_os]: token row of each suffix row
  float* psw = Ps + warp * 16;

  const int n_oa = R > rank ? (R - rank + CL - 1) / CL : 0;
  const int n_os = GB - R > rank ? (GB - R - rank + CL - 1) / CL : 0;
  const int ns = n_oa + n_os;
  const bool sel = !d.all_pages;
  // after the selection the CTA splits in two halves of kThreads threads:
  // warps [0, 8) build the page union and issue the gather copies, warps
  // [8, 16) stage the suffix rows and compute the suffix
  const bool uhalf = tid < kThreads;
  const int htid = uhalf ? tid : tid - kThreads;
  // the combine kernel may be scheduled now (its CTAs are small); it waits
  // for this grid's completion before it reads anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

#pragma unroll 1
  for (int e = tid; e < R * kPartStride; e += kThreadsG)  // empty partials
    part[e] = (e % kPartStride) == 0 ? -INFINITY : 0.f;
  if (sel) {
#pragma unroll 1
    for (int w = tid; w < nwords; w += kThreadsG) bitmap[w] = 0u;
#pragma unroll 1
    for (int e = tid; e < prm.max_lp * d.MW; e += kThreadsG) masks[e] = 0u;
  }
  // ---- the block's K and V (suffix half, cp.async group 0; rows >= B zero)
  if (!uhalf) {
    const char* kbg = static_cast<const char*>(prm.kb) + static_cast<size_t>(sg) * B * rowb;
    const char* vbg = static_cast<const char*>(prm.vb) + static_cast<size_t>(sg) * B * rowb;
    const int per = bpad * cpr;
#pragma unroll 1
    for (int e = htid; e < 2 * per; e += kThreads) {
      const int h = e >= per ? 1 : 0, rem = e - h * per, j = rem / cpr, c = rem - j * cpr;
      const bool ok = j < B;
      const char* src = (h ? vbg : kbg) + static_cast<size_t>(ok ? j : 0) * rowb + c * 16;
      cp_async16(su32(kbv + h * bpad * rowb + tile_off<DT>(j, c)), src, ok ? 16u : 0u);
    }
    cp_async_commit();
  }
  __syncthreads();

  // everything below reads what the scan kernel wrote
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const unsigned long long* cand_sg =
      prm.cand + static_cast<size_t>(sg) * d.nchunk * R * k;
  if (tid == 0) *s_len = seq_len(d, s);  // read after the selection's barrier
  {
    const int32_t* actg = prm.act_g + static_cast<size_t>(sg) * (R + GB);
#pragma unroll 1
    for (int e = tid; e < R + GB; e += kThreadsG) act_tok[e] = __ldcg(actg + e);
  }

  // ---- every row's k pages, ascending, into sel_all and the union bitmap
  // (each CTA of the group merges all rows; the CTA with r % CL == rank
  // reports row r)
  if (sel) {
    // the scan chunks that hold the sequence's pages
    const int ncs = ((seq_len(d, s) + kPS - 1) / kPS + d.chunk_pages - 1) / d.chunk_pages;
#pragma unroll 1
    for (int r = warp; r < R; r += kWarpsG) {
      unsigned long long* best = mbuf + (kWarpsG + warp) * kCandCap;
      merge_row<KP>(prm, r, ncs, cand_sg, best, mbuf + warp * kCandCap,
                    mbuf + 2 * kWarpsG * kCandCap + warp * 32);
      int32_t* dst = sel_all + r * k;
      const bool report = prm.page_idx && r % CL == rank;
#pragma unroll 1
      for (int j = lane; j < k; j += 32) {
        // an empty key (a sequence of fewer than k pages) sorts after every
        // real one, keeps its slot and reports page -1
        const bool real = best[j] != 0ull;
        const int pj = real ? key_index(best[j]) : -1;
        int rk = j;
        if (real) {
          rk = 0;
#pragma unroll 4
          for (int u = 0; u < k; ++u)  // (empty keys map to index 0xffffffff: never below)
            rk += static_cast<uint32_t>(key_index(best[u])) < static_cast<uint32_t>(pj);
        }
        dst[rk] = pj;
        if (pj >= 0 && pj < d.P) atomicOr(&bitmap[pj >> 5], 1u << (pj & 31));
        else if (real) atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
        if (report) {
          const int hl = r / A, a = r % A;
          prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + a) * k + rk] = pj;
        }
      }
      __syncwarp();
    }
  } else if (prm.page_idx) {
    const int Pseq = (seq_len(d, s) + kPS - 1) / kPS;  // every page of the sequence, then -1
#pragma unroll 1
    for (int r = rank; r < R; r += CL) {
      const int hl = r / A, a = r % A;
#pragma unroll 1
      for (int j = tid; j < k; j += kThreadsG)
        prm.page_idx[((static_cast<size_t>(s) * d.Hq + g * G + hl) * A + a) * k + j] =
            j < Pseq ? j : -1;
    }
  }
  __syncthreads();

  // gather copies (cp.async, union half): this CTA's union pages b0 ..
  // b0 + ngp into the page slots; rows past the prefix end are zero
  auto issue_batch = [&](int b0, int nlp, int t0, int nthr) {
    const int nb = min(prm.ngp, nlp - b0);
    constexpr int per = kPS * cpr;  // chunks of one page's K (or V)
#pragma unroll 1
    for (int i = 0; i < nb; ++i) {
      const int p = lpages[b0 + i];
      const size_t off = (static_cast<size_t>(sg) * d.Lc + static_cast<size_t>(p) * kPS) * rowb;
      const char* kp = static_cast<const char*>(prm.K) + off;
      const char* vp = static_cast<const char*>(prm.V) + off;
      char* dk = region + 2 * i * pbytes;
      const int ntok = min(kPS, *s_len - p * kPS);
#pragma unroll 1
      for (int e = t0; e < per; e += nthr) {
        const int j = e / cpr, c = e - j * cpr;
        const bool ok = j < ntok;
        const int so = (ok ? j : 0) * rowb + c * 16;
        cp_async16(su32(dk + tile_off<DT>(j, c)), kp + so, ok ? 16u : 0u);
        cp_async16(su32(dk + pbytes + tile_off<DT>(j, c)), vp + so, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };

  if (uhalf) {
    // ---- union of the group's pages and this CTA's share (slots u % CL)
    if (d.all_pages) {
      const int U = R > 0 ? (*s_len + kPS - 1) / kPS : 0;
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
      // exclusive prefix of the words' popcounts: each thread a run of words,
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
      if (lane == 31) s_wsum[warp] = incl;
      bar_sync(1, kThreads);
      int off = 0, U = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const int c = s_wsum[w];
        off += w < warp ? c : 0;
        U += c;
      }
      int run = off + incl - sum;
#pragma unroll 1
      for (int w = w0; w < w1; ++w) {
        wbase[w] = run;
        run += __popc(bitmap[w]);
      }
      const int nlp = U > rank ? (U - rank + CL - 1) / CL : 0;
      if (tid == 0) {
        *s_nlp = nlp;
        if (rank == 0 && prm.union_count) prm.union_count[sg] = U;
      }
      bar_sync(1, kThreads);
      // one pass over every (row, page): this CTA's union slots u % CL ==
      // rank get their page and the row's mask bit
#pragma unroll 1
      for (int e = tid; e < R * k; e += kThreads) {
        const int p = sel_all[e];
        if (p < 0 || p >= d.P) continue;
        const int w = p >> 5;
        const int u = wbase[w] + __popc(bitmap[w] & ((1u << (p & 31)) - 1u));
        const int r = e / k;
        if (u % CL != rank) continue;
        if (u / CL < prm.max_lp) {
          lpages[u / CL] = p;
          atomicOr(&masks[(u / CL) * d.MW + (r >> 5)], 1u << (r & 31));
        } else {
          atomicCAS(prm.status, 0, LOSA_ERR_DEVICE_BOUNDS);
        }
      }
    }
    bar_sync(1, kThreads);
    if (d.attend_union && sel) {
      // every active row attends to the whole union: every row's bit on each
      // of this CTA's pages
      const int nlp = min(*s_nlp, prm.max_lp);
#pragma unroll 1
      for (int e = tid; e < nlp * d.MW; e += kThreads) {
        const int nb = min(32, R - 32 * (e % d.MW));
        masks[e] = nb >= 32 ? 0xffffffffu : ((1u << nb) - 1u);
      }
    }
    issue_batch(0, min(*s_nlp, prm.max_lp), tid, kThreads);
    cp_async_wait<0>();  // this half's copies: the gathered pages
  } else {
    // ---- this CTA's suffix rows: its active rows r = rank + CL*j first, then
    // every CL-th stable token row
    {
      const int hw = htid >> 5;
      bool st = false;
      int pre = 0;
      if (hw < 4) {  // G*B <= 128 token rows
        st = htid < GB && act_slot[htid] < 0;
        const unsigned bal = __ballot_sync(0xffffffffu, st);
        pre = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) s_wt[hw] = __popc(bal);
      }
#pragma unroll 1
      for (int j = htid; j < n_oa; j += kThreads) {
        const int r = rank + CL * j;
        sfx_tok[j] = (r / A) * B + act_tok[r];
      }
      bar_sync(2, kThreads);
      if (st) {
        for (int w = 0; w < hw; ++w) pre += s_wt[w];
        if (pre % CL == rank) sfx_tok[n_oa + pre / CL] = htid;
      }
    }
    bar_sync(2, kThreads);
    if (prm.qref) {  // drift-safe locality: this CTA's active rows' reference := q_cur
      const char* qg = static_cast<const char*>(prm.qc) + grow0 * rowb;
      char* qr = static_cast<char*>(prm.qref) + grow0 * rowb;
#pragma unroll 1
      for (int e = htid; e < n_oa * cpr; e += kThreads) {
        const int j = e / cpr, c = e - j * cpr;
        const size_t o = static_cast<size_t>(sfx_tok[j]) * rowb + c * 16;
        *reinterpret_cast<uint4*>(qr + o) = *reinterpret_cast<const uint4*>(qg + o);
      }
    }
    // ---- cp.async group 1: queries of the suffix rows and of the active
    // rows, cached state of the stable suffix rows
    {
      const char* qg = static_cast<const char*>(prm.qc) + grow0 * rowb;
      const int nsr = DT == LOSA_BF16 ? (ns + 15) / 16 * 16 : ns;
#pragma unroll 1
      for (int e = htid; e < nsr * cpr; e += kThreads) {
        const int n = e / cpr, c = e - n * cpr;
        const bool ok = n < ns;
        cp_async16(su32(qs + tile_off<DT>(n, c)),
                   qg + static_cast<size_t>(ok ? sfx_tok[n] : 0) * rowb + c * 16, ok ? 16u : 0u);
      }
      const int nar = DT == LOSA_BF16 ? (R + 15) / 16 * 16 : R;
#pragma unroll 1
      for (int e = htid; e < nar * cpr; e += kThreads) {
        const int r = e / cpr, c = e - r * cpr;
        const bool ok = r < R;
        const int tok = ok ? (r / A) * B + act_tok[r] : 0;
        cp_async16(su32(qa + tile_off<DT>(r, c)), qg + static_cast<size_t>(tok) * rowb + c * 16,
                   ok ? 16u : 0u);
      }
#pragma unroll 1
      for (int e = htid; e < n_os * (kD / 4); e += kThreads) {
        const int n = e / (kD / 4), c = e - n * (kD / 4);
        const size_t grow = grow0 + sfx_tok[n_oa + n];
        cp_async16(su32(ocache + n * kD + 4 * c), prm.o_p + grow * kD + 4 * c, 16u);
      }
#pragma unroll 1
      for (int n = htid; n < n_os; n += kThreads)
        cp_async4(su32(lcache + n), prm.l_p + grow0 + sfx_tok[n_oa + n]);
      cp_async_commit();
    }
    cp_async_wait<0>();  // this half's copies: block K/V, queries, cached state
    bar_sync(2, kThreads);

    // ---- dense suffix of this CTA's rows: stable rows merge with their
    // cached state and are finished; active rows leave (L_s, o_s) for the
    // combine
    const int hw = htid >> 5;
    if (DT == LOSA_BF16) {
      const int nmt = (ns + 15) / 16;
#pragma unroll 1
      for (int mt = hw; mt < nmt; mt += kWarps) {
        TileAcc t;
        tile_init(t);
#pragma unroll 1
        for (int j0 = 0; j0 < B; j0 += kPS)
          tile_attend(t, qs + mt * 16 * 256, kbv + j0 * 256, kbv + (bpad + j0) * 256, 0xffffu,
                      min(kPS, B - j0), d.scale_log2);
        tile_finish(t);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = mt * 16 + g4 + 8 * h;
          if (n >= ns) continue;
          const float inv = __frcp_rn(t.l[h]);
          const float Ls = (t.m[h] + __log2f(t.l[h])) * kLn2;
          if (n < n_oa) {
            float* dst = prm.sfx_g + (static_cast<size_t>(sg) * R + rank + CL * n) * kPartStride;
            if (t4 == 0) dst[0] = Ls;
#pragma unroll
            for (int c = 0; c < 16; ++c)
              *reinterpret_cast<float2*>(dst + 4 + c * 8 + 2 * t4) =
                  make_float2(t.o[c][2 * h] * inv, t.o[c][2 * h + 1] * inv);
          } else {
            const int m = n - n_oa;
            const size_t grow = grow0 + sfx_tok[n];
            float wa, wb, L;
            lse_weights(lcache[m], Ls, wa, wb, L);
            const float* op = ocache + m * kD;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const int ch = c * 8 + 2 * t4;
              const float2 o = *reinterpret_cast<const float2*>(op + ch);
              *reinterpret_cast<float2*>(prm.out + grow * kD + ch) =
                  make_float2(wa * o.x + wb * (t.o[c][2 * h] * inv),
                              wa * o.y + wb * (t.o[c][2 * h + 1] * inv));
            }
            if (prm.out_lse && t4 == 0) prm.out_lse[grow] = L;
          }
        }
      }
    } else {
#pragma unroll 1
      for (int n = hw; n < ns; n += kWarps) {
        const float4 q = row4<DT>(qs, n, lane);
        float m = -INFINITY, l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
        for (int j0 = 0; j0 < B; j0 += kPS)
          attend_page<DT>(q, kbv + j0 * rowb, kbv + (bpad + j0) * rowb, min(kPS, B - j0),
                          d.scale_log2, m, l, acc, psw);
        const float inv = __frcp_rn(l);
        const float4 os = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        const float Ls = (m + __log2f(l)) * kLn2;
        if (n < n_oa) {
          float* dst = prm.sfx_g + (static_cast<size_t>(sg) * R + rank + CL * n) * kPartStride;
          if (lane == 0) dst[0] = Ls;
          *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = os;
        } else {
          const int mm = n - n_oa;
          const size_t grow = grow0 + sfx_tok[n];
          float wa, wb, L;
          lse_weights(lcache[mm], Ls, wa, wb, L);
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
  const int nlp = min(*s_nlp, prm.max_lp);

  // ---- the union pages -> one partial per row (part)
  if (DT == LOSA_BF16) {
    const int ntm = (R + 15) / 16;
    const int wpm = ntm > 0 ? max(1, kPageWarps / ntm) : kWarpsG;  // page warps per m16 tile
    const int mt = warp / wpm, sub = warp % wpm;
    const bool aw = mt < ntm;
    TileAcc t;
    tile_init(t);
#pragma unroll 1
    for (int b0 = 0; b0 < nlp; b0 += prm.ngp) {
      const int nb = min(prm.ngp, nlp - b0);
#pragma unroll 1
      for (int i = sub; aw && i < nb; i += wpm) {
        const uint32_t bits = (masks[(b0 + i) * d.MW + (mt >> 1)] >> ((mt & 1) * 16)) & 0xffffu;
        if (!bits) continue;
        const int p = lpages[b0 + i];
        tile_attend(t, qa + mt * 16 * 256, region + 2 * i * pbytes, region + (2 * i + 1) * pbytes,
                    bits, min(kPS, *s_len - p * kPS), d.scale_log2);
      }
      if (b0 + prm.ngp < nlp) {  // next batch into the same slots
        __syncthreads();
        issue_batch(b0 + prm.ngp, nlp, tid, kThreadsG);
        cp_async_wait<0>();
        __syncthreads();
      }
    }
    tile_finish(t);
    if (wpm == 1) {  // one warp per m16 tile: its state is the CTA's partial
      if (aw) tile_store(t, part_cta + mt * 16 * kPartStride, min(16, R - mt * 16));
    } else {
      float* wp = reinterpret_cast<float*>(region);
      __syncthreads();  // every page consumed: the region takes the warps' partials
      if (aw) tile_store(t, wp + warp * 16 * kPartStride, 16);
      __syncthreads();
#pragma unroll 1
      for (int r = warp; r < R; r += kWarpsG) {
        const int m16 = r >> 4, i = r & 15;
        float mw[kPageWarps], lw[kPageWarps];
        float4 aw4[kPageWarps];
#pragma unroll
        for (int w = 0; w < kPageWarps; ++w) {
          mw[w] = -INFINITY;
          if (w < wpm) {
            const float* pr = wp + ((m16 * wpm + w) * 16 + i) * kPartStride;
            mw[w] = pr[0];
            lw[w] = pr[1];
            aw4[w] = *reinterpret_cast<const float4*>(pr + 4 + 4 * lane);
          }
        }
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kPageWarps; ++w) M = fmaxf(M, mw[w]);
        float* dst = part_cta + r * kPartStride;
        if (M == -INFINITY) {  // none of this CTA's pages serve row r
          if (lane == 0) dst[0] = -INFINITY;
          continue;
        }
        float l = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kPageWarps; ++w) {
          if (mw[w] == -INFINITY) continue;
          const float wgt = exp2f(mw[w] - M);
          l += wgt * lw[w];
          acc.x += wgt * aw4[w].x;
          acc.y += wgt * aw4[w].y;
          acc.z += wgt * aw4[w].z;
          acc.w += wgt * aw4[w].w;
        }
        if (lane == 0) {
          dst[0] = M;
          dst[1] = l;
        }
        *reinterpret_cast<float4*>(dst + 4 + 4 * lane) = acc;
      }
    }
  } else {
#pragma unroll 1
    for (int b0 = 0; b0 < nlp; b0 += prm.ngp) {
      const int nb = min(prm.ngp, nlp - b0);
#pragma unroll 1
      for (int r = warp; r < R; r += kWarpsG) {
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
          const int p = lpages[b0 + i];
          attend_page<DT>(q, region + 2 * i * pbytes, region + (2 * i + 1) * pbytes,
                          min(kPS, *s_len - p * kPS), d.scale_log2, m, l, acc, psw);
        }
        __syncwarp();
        if (lane == 0) {
          pr[0] = m;
          pr[1] = l;
        }
        *reinterpret_cast<float4*>(pr + 4 + 4 * lane) = acc;
      }
      if (b0 + prm.ngp < nlp) {
        __syncthreads();
        issue_batch(b0 + prm.ngp, nlp, tid, kThreadsG);
        cp_async_wait<0>();
        __syncthreads();
      }
    }
  }
  __syncthreads();

  // ---- this CTA's row partials to the workspace (bf16: already there); the
  // combine kernel merges them once every CTA of the grid has finished
  if (DT != LOSA_BF16) {
    float4* dstp = reinterpret_cast<float4*>(part_cta);
    const float4* srcp = reinterpret_cast<const float4*>(part);
#pragma unroll 1
    for (int e = tid; e < R * kPartStride / 4; e += kThreadsG) dstp[e] = srcp[e];
  }
}

// ---------------------------------------------------------------------------
// K3: combine.  One warp per active row, launched behind the gather kernel by
// programmatic dependent launch: lane c reads CTA c's partial maximum and
// sum, the non-empty partials' vectors are loaded together (a CTA that owns
// none of the row's pages left m = -inf), merged in ascending CTA order
// (deterministic); the new o_p / L_p are written back and merged with the
// row's suffix into the output.
// ---------------------------------------------------------------------------
struct CombineParams {
  const int32_t* act_g;
  const float* part_g;
  const float* sfx_g;
  float* o_p;
  float* l_p;
  float* out;
  float* out_lse;
  Dims d;
};

constexpr int kCombineWarps = 4;

__global__ void __launch_bounds__(kCombineWarps * 32) losa_combine_kernel(const CombineParams prm) {
  const Dims& d = prm.d;
  constexpr int CL = kGatherCtas;
  const int lane = threadIdx.x & 31;
  const int sg = blockIdx.y, r = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int R = d.R, A = d.A, B = d.B, GB = d.G * d.B;
  // everything below reads what the gather kernel (and before it the scan
  // kernel) wrote
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the next kernel of the stream (the next step's scan kernel) may be
  // scheduled now, not earlier: its CTAs would sit on SMs the gather kernel
  // still needs; it waits for this grid's completion before it touches
  // anything this grid reads or writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (r >= R) return;
  const int s = sg / d.Hkv, g = sg % d.Hkv;
  const size_t grow0 = (static_cast<size_t>(s) * d.Hq + g * d.G) * B;
  const int tok = __ldcg(prm.act_g + static_cast<size_t>(sg) * (R + GB) + r);
  const size_t cstride = static_cast<size_t>(R) * kPartStride;  // between CTAs' partials
  const float* pg = prm.part_g + (static_cast<size_t>(sg) * CL * R + r) * kPartStride;
  const float* sx = prm.sfx_g + (static_cast<size_t>(sg) * R + r) * kPartStride;
  const float mj = lane < CL ? __ldcg(pg + lane * cstride) : -INFINITY;
  const float lj = lane < CL ? __ldcg(pg + lane * cstride + 1) : 0.f;
  const float4 os = __ldcg(reinterpret_cast<const float4*>(sx + 4) + lane);
  const float Ls = __ldcg(sx);
  const uint32_t nz = __ballot_sync(0xffffffffu, mj != -INFINITY);
  float4 ac[CL];
#pragma unroll
  for (int j = 0; j < CL; ++j)
    if ((nz >> j) & 1u) ac[j] = __ldcg(reinterpret_cast<const float4*>(pg + j * cstride + 4) + lane);
  float M = mj;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float wj = mj == -INFINITY ? 0.f : exp2f(mj - M);
  float lsum = wj * lj;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < CL; ++j) {
    const float w = __shfl_sync(0xffffffffu, wj, j);
    if ((nz >> j) & 1u) {
      acc.x += w * ac[j].x;
      acc.y += w * ac[j].y;
      acc.z += w * ac[j].z;
      acc.w += w * ac[j].w;
    }
  }
  const float inv = __frcp_rn(lsum);
  const float4 op = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  const float Lp = (M + __log2f(lsum)) * kLn2;
  const size_t grow = grow0 + (r / A) * B + tok;
  *reinterpret_cast<float4*>(prm.o_p + grow * kD + 4 * lane) = op;
  if (lane == 0) prm.l_p[grow] = Lp;
  float wa, wb, L;
  lse_weights(Lp, Ls, wa, wb, L);
  *reinterpret_cast<float4*>(prm.out + grow * kD + 4 * lane) =
      make_float4(wa * op.x + wb * os.x, wa * op.y + wb * os.y, wa * op.z + wb * os.z,
                  wa * op.w + wb * os.w);
  if (prm.out_lse && lane == 0) prm.out_lse[grow] = L;
}

// ---------------------------------------------------------------------------
// host side: launch geometry, shared-memory layouts, attributes
// ---------------------------------------------------------------------------
int topk_width(int k) {
  if (k <= 2) return 2;
  if (k <= 4) return 4;
  if (k <= 8) return 8;
  if (k <= 16) return 16;
  return 0;  // warp fallback
}

struct Taker {
  int off = 0;
  int operator()(long long bytes, int align) {
    off = align_up(off, align);
    const int o = off;
    off += static_cast<int>(std::min<long long>(bytes, 1 << 30));
    return o;
  }
};

bool plan_scan(const Dims& d, ScanParams* prm, int max_dyn) {
  prm->d = d;
  prm->scan = d.A > 0 && !d.all_pages;
  prm->rec = 2 * kD * d.esz;
  prm->tile = kStageBytes / prm->rec;  // 64 (bf16) or 32 (fp32) pages per stage
  prm->sc_stride = align_up(d.chunk_pages, 4) + 4;
  prm->kp = topk_width(d.k);
  const int GB = d.G * d.B;
  // a row's top-k group: at least k lanes, and enough lanes to cover the
  // CTA's rows in few passes
  prm->tpr = kTopkW;  // k <= 16 whenever the specialised top-k runs
  prm->mse_t = std::min(16, pow2_floor(std::max(1, kThreads / std::max(GB, 1))));
  prm->nv = 8;
  while (prm->nv * prm->tpr < d.chunk_pages) prm->nv *= 2;
  if (prm->scan && prm->kp > 0 && prm->tpr < d.k) return false;
  if (prm->scan && prm->kp == 0 && d.k > kCandCap) return false;
  const int R16 = (d.R + 15) / 16 * 16;
  const long long qbytes = 1LL * GB * kD * d.esz;
  for (int ring = prm->scan ? kMaxRingBytes : 0; ring >= 0; ring -= 32 * 1024) {
    if (prm->scan && ring < 32 * 1024) break;
    ScanLayout& lo = prm->lo;
    Taker take;
    lo.ring = take(ring, 1024);
    lo.qc = take(qbytes, 128);
    // the previous queries, then (after the locality pass) the scores
    lo.qps = take(std::max(qbytes, prm->scan ? 4LL * d.R * prm->sc_stride : 0LL), 128);
    lo.qrows = take(prm->scan ? (d.esz == 2 ? R16 : d.R) * 512LL : 0, 128);
    lo.misc = take((4 + 3 * kMaxRowsPerGroup) * 4, 16);
    lo.fbuf = take(prm->scan && prm->kp > 0 ? 8LL * (kThreads / prm->tpr) * kCandCap : 0, 16);
    lo.cbuf = take(prm->scan && prm->kp == 0 ? 2 * kWarps * kCandCap * 8 : 0, 16);
    lo.mbar = take((kMaxStages + 1) * 8, 8);
    lo.total = take.off;
    prm->stages = ring / kStageBytes;
    if (lo.total <= max_dyn) return true;
    if (!prm->scan) break;
  }
  return false;
}

bool plan_gather(const Dims& d, GatherParams* prm, int max_dyn, int CL) {
  prm->d = d;
  prm->CL = CL;
  prm->max_lp = (d.Umax + CL - 1) / CL;
  if (!d.all_pages && d.A > 0 && topk_width(d.k) == 0 && d.k > kCandCap) return false;
  const int GB = d.G * d.B;
  prm->n_oa = (d.R + CL - 1) / CL;
  prm->n_os = (GB - d.R + CL - 1) / CL;
  const int ns = prm->n_oa + prm->n_os;
  const bool bf = d.esz == 2;
  const int ntm = (d.R + 15) / 16;
  prm->wpart = bf && ntm > 0 && kPageWarps / ntm > 1;
  const int rowb = kD * d.esz;
  const int nwords = (d.P + 31) / 32;
  const int pbytes = kPS * rowb;
  const int bpad = (d.B + kPS - 1) / kPS * kPS;
  const bool sel = !d.all_pages && d.A > 0;
  // the region holds, in turn: the gathered pages, the page warps' partials
  auto layout = [&](int ngp) {
    GatherLayout& lo = prm->lo;
    Taker take;
    lo.region = take(std::max(2LL * ngp * pbytes,
                              prm->wpart ? 4LL * kPageWarps * 16 * kPartStride : 0LL),
                     1024);
    lo.kbv = take(2LL * bpad * rowb, 128);
    lo.qa = take(1LL * (bf ? ntm * 16 : d.R) * rowb, 128);
    lo.qs = take(1LL * (bf ? (ns + 15) / 16 * 16 : ns) * rowb, 128);
    lo.ocache = take(4LL * prm->n_os * kD, 16);
    lo.lcache = take(4LL * prm->n_os, 16);
    lo.sel_all = take(sel ? 4LL * d.R * d.k : 0, 16);
    lo.bitmap = take(nwords * 4, 16);
    lo.wbase = take(nwords * 4, 16);
    lo.lpages = take(prm->max_lp * 4, 16);
    lo.masks = take(4LL * prm->max_lp * d.MW, 16);
    lo.part = take(4LL * d.R * kPartStride, 16);
    lo.misc = take((16 + d.R + GB + ns) * 4, 16);
    lo.ps = take(kWarpsG * 16 * 4, 16);
    lo.mbuf = take(sel ? (2 * kCandCap + 32) * kWarpsG * 8 : 0, 16);
    lo.total = take.off;
    prm->ngp = ngp;
    return lo.total;
  };
  // the largest batch of pages in flight that fits
  for (int ngp = std::min(kMaxGatherPages, std::max(1, prm->max_lp)); ngp >= 1; ngp /= 2)
    if (layout(ngp) <= max_dyn) return true;
  return false;
}

std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices] = {};
int g_attr_dyn[kMaxDevices] = {};

template <int DT, int KP>
cudaError_t set_attrs_one(int optin, int* dyn) {
  const void* fns[6] = {reinterpret_cast<const void*>(losa_gather_kernel<DT, KP>),
                        reinterpret_cast<const void*>(losa_scan_kernel<DT, KP, 0>),
                        reinterpret_cast<const void*>(losa_scan_kernel<DT, KP, KP ? 8 : 0>),
                        reinterpret_cast<const void*>(losa_scan_kernel<DT, KP, KP ? 16 : 0>),
                        reinterpret_cast<const void*>(losa_scan_kernel<DT, KP, KP ? 32 : 0>),
                        reinterpret_cast<const void*>(losa_scan_kernel<DT, KP, KP ? 64 : 0>)};
  for (int i = 0; i < 6; ++i) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, fns[i]);
    if (e != cudaSuccess) return e;
    const int mine = optin - static_cast<int>(fa.sharedSizeBytes);
    e = cudaFuncSetAttribute(fns[i], cudaFuncAttributeMaxDynamicSharedMemorySize, mine);
    if (e != cudaSuccess) return e;
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

int ensure_attributes(int* max_dyn) {
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
    g_attr_done[dev] = true;
  }
  *max_dyn = g_attr_dyn[dev];
  return LOSA_OK;
}

// One scan kernel per (top-k width, scores per lane): each carries the one
// row top-k it runs, which keeps its code small (instruction fetch is a
// measurable part of a step); NV = 0 is the general fallback.
struct StepLaunch {
  cudaLaunchConfig_t c1, c2, c3;
  ScanParams sp;
  GatherParams gp;
  CombineParams cp;
};

template <int DT, int KP, int NV>
cudaError_t launch_step_nv(const StepLaunch& L) {
  cudaError_t e = cudaLaunchKernelEx(&L.c1, losa_scan_kernel<DT, KP, NV>, L.sp);
  if (e != cudaSuccess) return e;
  e = cudaLaunchKernelEx(&L.c2, losa_gather_kernel<DT, KP>, L.gp);
  if (e != cudaSuccess || L.c3.gridDim.x == 0) return e;  // no active row: nothing to combine
  return cudaLaunchKernelEx(&L.c3, losa_combine_kernel, L.cp);
}

template <int DT, int KP>
cudaError_t launch_step_kp(const StepLaunch& L) {
  if constexpr (KP > 0) {
    switch (L.sp.nv) {
      case 8: return launch_step_nv<DT, KP, 8>(L);
      case 16: return launch_step_nv<DT, KP, 16>(L);
      case 32: return launch_step_nv<DT, KP, 32>(L);
      case 64: return launch_step_nv<DT, KP, 64>(L);
      default: break;
    }
  }
  return launch_step_nv<DT, KP, 0>(L);
}

template <int DT>
cudaError_t launch_dt(int kp, const StepLaunch& L) {
  switch (kp) {
    case 2: return launch_step_kp<DT, 2>(L);
    case 4: return launch_step_kp<DT, 4>(L);
    case 8: return launch_step_kp<DT, 8>(L);
    case 16: return launch_step_kp<DT, 16>(L);
    default: return launch_step_kp<DT, 0>(L);
  }
}

}  // namespace

bool fused_step_fits(const Dims& d, int max_dyn) {
  ScanParams sp;
  GatherParams gp;
  return plan_scan(d, &sp, max_dyn) && plan_gather(d, &gp, max_dyn, kGatherCtas);
}

int launch_fused_step(const Dims& d, const void* q_cur, const void* q_prev, const void* k_prefix,
                      const void* v_prefix, const void* page_meta, const void* k_blk,
                      const void* v_blk, float* o_p, float* l_p, float* out, float* out_lse,
                      int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                      void* workspace, cudaStream_t st, void* q_ref_out) {
  int max_dyn = 0;
  int rc = ensure_attributes(&max_dyn);
  if (rc != LOSA_OK) return rc;
  StepLaunch L = {};
  ScanParams& sp = L.sp;
  GatherParams& gp = L.gp;
  if (!plan_scan(d, &sp, max_dyn)) return LOSA_ERR_UNSUPPORTED;
  if (!plan_gather(d, &gp, max_dyn, kGatherCtas)) return LOSA_ERR_UNSUPPORTED;
  if (d.S * d.Hkv > 65535 || d.nchunk > 65535) return LOSA_ERR_UNSUPPORTED;
  char* ws = static_cast<char*>(workspace);
  int* status = reinterpret_cast<int*>(ws + d.off_status);
  int32_t* act = reinterpret_cast<int32_t*>(ws + d.off_act);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(ws + d.off_cand);
  float* part_g = reinterpret_cast<float*>(ws + d.off_gpart);
  float* sfx_g = reinterpret_cast<float*>(ws + d.off_gsfx);

  sp.qc = q_cur;
  sp.qp = q_prev;
  sp.meta = static_cast<const char*>(page_meta);
  sp.act_g = act;
  sp.active_idx = active_idx;
  sp.cand = cand;
  sp.status = status;
  cudaLaunchConfig_t& c1 = L.c1;
  cudaLaunchAttribute attr1[1];
  c1.gridDim = dim3(sp.scan ? d.nchunk : 1, d.S * d.Hkv, 1);
  c1.blockDim = dim3(kThreads, 1, 1);
  c1.dynamicSmemBytes = static_cast<size_t>(sp.lo.total);
  c1.stream = st;
  attr1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr1[0].val.programmaticStreamSerializationAllowed = 1;  // overlaps the previous kernel's tail
  c1.attrs = attr1;
  c1.numAttrs = 1;

  gp.qc = q_cur;
  gp.K = k_prefix;
  gp.V = v_prefix;
  gp.kb = k_blk;
  gp.vb = v_blk;
  gp.o_p = o_p;
  gp.l_p = l_p;
  gp.out = out;
  gp.out_lse = out_lse;
  gp.page_idx = page_idx;
  gp.qref = q_ref_out;
  gp.union_count = union_count;
  gp.act_g = act;
  gp.cand = cand;
  gp.part_g = part_g;
  gp.sfx_g = sfx_g;
  gp.status = status;
  cudaLaunchConfig_t& c2 = L.c2;
  cudaLaunchAttribute attr[1];
  c2.gridDim = dim3(gp.CL, d.S * d.Hkv, 1);
  c2.blockDim = dim3(kThreadsG, 1, 1);
  c2.dynamicSmemBytes = static_cast<size_t>(gp.lo.total);
  c2.stream = st;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;  // overlaps the scan kernel
  c2.attrs = attr;
  c2.numAttrs = 1;

  CombineParams& cp = L.cp;
  cp.act_g = act;
  cp.part_g = part_g;
  cp.sfx_g = sfx_g;
  cp.o_p = o_p;
  cp.l_p = l_p;
  cp.out = out;
  cp.out_lse = out_lse;
  cp.d = d;
  cudaLaunchConfig_t& c3 = L.c3;
  cudaLaunchAttribute attr3[1];
  c3.gridDim = dim3((d.R + kCombineWarps - 1) / kCombineWarps, d.S * d.Hkv, 1);
  c3.blockDim = dim3(kCombineWarps * 32, 1, 1);
  c3.dynamicSmemBytes = 0;
  c3.stream = st;
  attr3[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr3[0].val.programmaticStreamSerializationAllowed = 1;  // overlaps the gather kernel
  c3.attrs = attr3;
  c3.numAttrs = 1;
  // one top-k width per compiled kernel: the selection code of the others is
  // never fetched
  const int kp = sp.scan ? sp.kp : 2;
  const cudaError_t e = d.dtype == LOSA_BF16 ? launch_dt<LOSA_BF16>(kp, L)
                                             : launch_dt<LOSA_F32>(kp, L);
  return e == cudaSuccess ? LOSA_OK : record_cuda_error(e);
}

}  // namespace losa
