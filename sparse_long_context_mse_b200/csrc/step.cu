// step.cu -- C entry points of one LoSA denoising step (plain and drift-safe):
// host validation, then the two step kernels of step_fused.cu.
#include "losa_common.cuh"

namespace {

int step_common(const losa_shape* shape, const void* q_cur, const void* q_prev, void* q_ref_out,
                const void* k_prefix, const void* v_prefix, const void* page_meta,
                const void* k_blk, const void* v_blk, float* o_p, float* l_p, float* out,
                float* out_lse, int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                void* workspace, size_t ws_bytes, void* stream) {
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
  if (q_ref_out) {  // the reference is rewritten: it may alias nothing else
    const size_t lb = rows * sizeof(float);
    if (overlaps(q_ref_out, qb, q_cur, qb) || overlaps(q_ref_out, qb, o_p, ob) ||
        overlaps(q_ref_out, qb, l_p, lb) || overlaps(q_ref_out, qb, out, ob) ||
        (out_lse && overlaps(q_ref_out, qb, out_lse, lb)))
      return LOSA_ERR_INVALID_ARG;
  }
  if (d.S * d.Hkv > 65535) return LOSA_ERR_UNSUPPORTED;
  return launch_fused_step(d, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p,
                           l_p, out, out_lse, active_idx, page_idx, union_count, workspace,
                           static_cast<cudaStream_t>(stream), q_ref_out);
}

}  // namespace

extern "C" int losa_step(const losa_shape* shape, const void* q_cur, const void* q_prev,
                         const void* k_prefix, const void* v_prefix, const void* page_meta,
                         const void* k_blk, const void* v_blk, float* o_p, float* l_p,
                         float* out, float* out_lse, int32_t* active_idx, int32_t* page_idx,
                         int32_t* union_count, void* workspace, size_t ws_bytes, void* stream) {
  return step_common(shape, q_cur, q_prev, nullptr, k_prefix, v_prefix, page_meta, k_blk, v_blk,
                     o_p, l_p, out, out_lse, active_idx, page_idx, union_count, workspace,
                     ws_bytes, stream);
}

extern "C" int losa_step_ref(const losa_shape* shape, const void* q_cur, void* q_ref,
                             const void* k_prefix, const void* v_prefix, const void* page_meta,
                             const void* k_blk, const void* v_blk, float* o_p, float* l_p,
                             float* out, float* out_lse, int32_t* active_idx, int32_t* page_idx,
                             int32_t* union_count, void* workspace, size_t ws_bytes,
                             void* stream) {
  if (!q_ref) return LOSA_ERR_INVALID_ARG;
  return step_common(shape, q_cur, q_ref, q_ref, k_prefix, v_prefix, page_meta, k_blk, v_blk,
                     o_p, l_p, out, out_lse, active_idx, page_idx, union_count, workspace,
                     ws_bytes, stream);
}
