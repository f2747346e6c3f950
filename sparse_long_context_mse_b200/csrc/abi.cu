// abi.cu -- host side of the C ABI: shape validation, workspace layout,
// status reporting.  No kernel lives here.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>

#include "losa_common.cuh"

namespace losa {

namespace {
thread_local std::string g_last_error;

// The workspace is sized for the B200's SM count so that sizes do not depend
// on which device happens to be current (and can be queried without one).
constexpr int kSizingSms = 148;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
}  // namespace

int record_cuda_error(cudaError_t e) {
  g_last_error = std::string(cudaGetErrorName(e)) + ": " + cudaGetErrorString(e);
  return LOSA_ERR_CUDA;
}

int make_tmap(CUtensorMap* map, const void* base, unsigned long long nrows, unsigned box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return LOSA_ERR_CUDA;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kD), nrows};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kD) * 2};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LOSA_OK : LOSA_ERR_CUDA;
}

int make_page_tmap(CUtensorMap* map, const void* base, unsigned long long nrows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!encode) return LOSA_ERR_CUDA;
  const cuuint64_t dims[3] = {64u, nrows, 2u};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2, 128u};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(kPS), 2u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LOSA_OK : LOSA_ERR_CUDA;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kSizingSms;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return kSizingSms;
  return n;
}

int make_dims(const losa_shape* sh, int which, Dims* d) {
  if (!sh || !d) return LOSA_ERR_INVALID_ARG;
  std::memset(d, 0, sizeof(*d));
  if (sh->num_seqs < 1 || sh->n_q_heads < 1 || sh->n_kv_heads < 1 || sh->prefix_len < 1 ||
      sh->block_size < 1 || sh->page_size < 1 || sh->head_dim < 1 || sh->n_active < 0 ||
      sh->token_budget < 0)
    return LOSA_ERR_INVALID_ARG;
  if (sh->n_q_heads % sh->n_kv_heads != 0) return LOSA_ERR_INVALID_ARG;
  if (sh->n_active > sh->block_size) return LOSA_ERR_INVALID_ARG;
  if (!(std::isfinite(sh->scale)) || sh->scale < 0.f) return LOSA_ERR_INVALID_ARG;
  if (sh->head_dim != kD || sh->page_size != kPS) return LOSA_ERR_UNSUPPORTED;
  if (sh->dtype != LOSA_F32 && sh->dtype != LOSA_BF16) return LOSA_ERR_UNSUPPORTED;
  if (sh->flags & ~LOSA_STEP_ATTEND_UNION) return LOSA_ERR_INVALID_ARG;
  if (sh->prefix_capacity != 0 && sh->prefix_capacity < sh->prefix_len) return LOSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(sh->prefix_lens) & 3u) return LOSA_ERR_INVALID_ARG;
  const int G = sh->n_q_heads / sh->n_kv_heads;
  if (sh->block_size > kMaxB || G * sh->block_size > kMaxRowsPerGroup) return LOSA_ERR_UNSUPPORTED;
  const long long P = (static_cast<long long>(sh->prefix_len) + kPS - 1) / kPS;
  const long long kk = std::min<long long>(sh->token_budget / kPS, P);
  if (sh->n_active > 0 && kk < 1) return LOSA_ERR_INVALID_ARG;
  if (kk > kMaxK && kk != P) return LOSA_ERR_UNSUPPORTED;

  d->S = sh->num_seqs;
  d->Hq = sh->n_q_heads;
  d->Hkv = sh->n_kv_heads;
  d->G = G;
  d->L = sh->prefix_len;
  d->P = static_cast<int>(P);
  d->Lc = sh->prefix_capacity > 0 ? sh->prefix_capacity : sh->prefix_len;
  d->Pc = (d->Lc + kPS - 1) / kPS;
  d->B = sh->block_size;
  d->A = sh->n_active;
  d->k = static_cast<int>(kk);
  d->R = G * sh->n_active;
  d->MW = (d->R + 31) / 32;
  d->dtype = sh->dtype;
  d->esz = sh->dtype == LOSA_BF16 ? 2 : 4;
  d->all_pages = (d->k == d->P);
  d->attend_union = (sh->flags & LOSA_STEP_ATTEND_UNION) != 0;
  d->lens = sh->prefix_lens;
  d->scale = sh->scale > 0.f ? sh->scale : 1.0f / std::sqrt(static_cast<float>(sh->head_dim));
  d->scale_log2 = d->scale * kLog2e;
  d->Umax = static_cast<int>(std::min<long long>(P, static_cast<long long>(d->R) * d->k));

  const size_t SG = static_cast<size_t>(d->S) * d->Hkv;
  size_t off = 0;
  d->off_status = off;
  off += 256;
  if (which == LOSA_WS_DENSE) {
    // bf16 (tensor cores, one 211-227 KB CTA per SM): one wave of whole
    // 128-key tiles; fp32: two CTAs' worth of splits per SM
    const bool tc = sh->dtype == LOSA_BF16;
    int nsplit = tc ? static_cast<int>(kSizingSms / SG)
                    : static_cast<int>((2 * kSizingSms + SG - 1) / SG);
    if (nsplit < 1) nsplit = 1;
    if (nsplit > d->P) nsplit = d->P;
    d->split_pages = (d->P + nsplit - 1) / nsplit;
    if (tc) d->split_pages = (d->split_pages + 7) / 8 * 8;
    d->nsplit = (d->P + d->split_pages - 1) / d->split_pages;
    d->off_part = off;
    off += align256(SG * d->nsplit * static_cast<size_t>(G * d->B) * kPartStride * sizeof(float));
    d->total = off;
    return LOSA_OK;
  }
  if (which != LOSA_WS_STEP) return LOSA_ERR_INVALID_ARG;
  // step: one cluster per group keeps its whole state in shared memory; the
  // workspace holds only the status word
  d->total = off;
  // the fused step keeps each group's selection state in shared memory
  if (!fused_step_fits(*d, kB200MaxDynSmem)) return LOSA_ERR_UNSUPPORTED;
  return LOSA_OK;
}

}  // namespace losa

extern "C" {

size_t losa_page_meta_size(const losa_shape* shape) {
  losa::Dims d;
  if (losa::make_dims(shape, LOSA_WS_DENSE, &d) != LOSA_OK) return 0;
  return losa::meta_norm_offset(d) +
         static_cast<size_t>(d.S) * d.Hkv * losa::meta_norm_stride(d) * 2 * sizeof(float);
}

size_t losa_workspace_size(const losa_shape* shape, int which) {
  losa::Dims d;
  if (losa::make_dims(shape, which, &d) != LOSA_OK) return 0;
  return d.total;
}

int losa_read_device_status(void* workspace, void* stream) {
  if (!workspace) return LOSA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int status = 0;
  cudaError_t e = cudaMemcpyAsync(&status, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return losa::record_cuda_error(e);
  return status;
}

const char* losa_status_string(int status) {
  switch (status) {
    case LOSA_OK: return "ok";
    case LOSA_ERR_INVALID_ARG: return "invalid argument";
    case LOSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LOSA_ERR_CUDA: return "CUDA error";
    case LOSA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case LOSA_ERR_DEVICE_BOUNDS: return "device-side bounds check failed";
    default: return "unknown status";
  }
}

const char* losa_last_error(void) { return losa::g_last_error.c_str(); }

}  // extern "C"
