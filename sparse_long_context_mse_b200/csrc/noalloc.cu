// noalloc.cu -- losa_step with library-owned scratch, for callers that cannot
// allocate device memory.
//
// losa_step takes its scratch ("workspace") from the caller.  Some callers
// have no way to provide it: a plugin running inside a host framework whose
// caching allocator already owns the GPU's memory (a raw cudaMalloc there
// fails or fragments the framework's pool), or a latency-critical loop that
// must not call cudaMalloc/cudaFree because those can synchronise the whole
// device.  losa_step_noalloc serves them: its scratch is a fixed-size array
// in device global memory that is part of this library's module, created when
// the module is loaded on a GPU and kept until the process exits.
#include <mutex>

#include "losa_common.cuh"

namespace losa {
namespace {

// The scratch every losa_step_noalloc call on a device shares.  In host code
// `g_noalloc_scratch` names a host-side stand-in, not a device address: it
// must never be passed to a kernel; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LOSA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch, per device; filled on the first call made
// while that device is current.
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return record_cuda_error(e);
  if (dev < 0 || dev >= kMaxDevices) return LOSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return record_cuda_error(e);
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return LOSA_OK;
}

}  // namespace
}  // namespace losa

extern "C" int losa_step_noalloc(const losa_shape* shape, const void* q_cur, const void* q_prev,
                                 const void* k_prefix, const void* v_prefix,
                                 const void* page_meta, const void* k_blk, const void* v_blk,
                                 float* o_p, float* l_p, float* out, float* out_lse,
                                 int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                                 void* stream) {
  using namespace losa;
  // size check first: a shape whose scratch does not fit is rejected before
  // anything touches the device
  const size_t need = losa_workspace_size(shape, LOSA_WS_STEP);
  if (need == 0) {
    Dims d;
    const int rc = make_dims(shape, LOSA_WS_STEP, &d);
    return rc != LOSA_OK ? rc : LOSA_ERR_INVALID_ARG;
  }
  if (need > static_cast<size_t>(LOSA_NOALLOC_SCRATCH_BYTES)) return LOSA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != LOSA_OK) return rc;
  // losa_step needs nothing in its workspace to start at zero, so the
  // previous call's leftovers are harmless as long as the calls ended with
  // LOSA_OK (losa_noalloc_read_status tells)
  return losa_step(shape, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p, l_p,
                   out, out_lse, active_idx, page_idx, union_count, scratch,
                   static_cast<size_t>(LOSA_NOALLOC_SCRATCH_BYTES), stream);
}

extern "C" int losa_noalloc_read_status(void* stream) {
  using namespace losa;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != LOSA_OK) return rc;
  // the status word sits at the start of a step workspace, and so at the
  // start of the scratch array
  return losa_read_device_status(scratch, stream);
}
