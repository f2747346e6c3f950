// step.cu -- C entry points of one LoSA denoising step (plain and drift-safe):
// host validation, then the step kernels of step_fused.cu.
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
  // no written buffer may overlap another buffer of the call (q_ref is
  // q_prev, read and then rewritten, in the drift-safe variant)
  const size_t rows = static_cast<size_t>(d.S) * d.Hq * d.B;
  const size_t SG = static_cast<size_t>(d.S) * d.Hkv;
  const size_t ob = rows * kD * sizeof(float), lb = rows * sizeof(float);
  const size_t qb = rows * kD * d.esz, kvb = SG * d.Lc * kD * d.esz, kbb = SG * d.B * kD * d.esz;
  const size_t mb = SG * d.Pc * 2 * kD * d.esz;
  const size_t ab = static_cast<size_t>(d.S) * d.Hq * d.A * sizeof(int32_t);
  const Region reg[] = {{q_cur, qb, false},       {q_prev, qb, q_ref_out != nullptr},
                        {k_prefix, kvb, false},   {v_prefix, kvb, false},
                        {page_meta, mb, false},   {k_blk, kbb, false},
                        {v_blk, kbb, false},      {o_p, ob, true},
                        {l_p, lb, true},          {out, ob, true},
                        {out_lse, lb, true},      {active_idx, ab, true},
                        {page_idx, ab * d.k, true}, {union_count, SG * sizeof(int32_t), true},
                        {workspace, d.total, true}};
  if (any_write_alias(reg, static_cast<int>(sizeof(reg) / sizeof(reg[0]))))
    return LOSA_ERR_INVALID_ARG;
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
