/*
 * losa.h -- C ABI of the LoSA per-denoising-step attention library for
 * NVIDIA B200 (sm_100a).
 *
 * LoSA ("LoSA: Locality Aware Sparse Attention for Block-Wise Diffusion
 * Language Models") speeds up the prefix attention of block-wise diffusion
 * LMs.  Between two denoising steps only a few block tokens change much
 * (paper, "locality of representation changes"), so each step
 *
 *   1. scores every block token by the MSE between its current and previous
 *      query and keeps the top-|A| per query head as "active";
 *   2. picks, for each active query only, the top-k prefix pages by the QUEST
 *      bound sum_i max(q_i*kmax_i, q_i*kmin_i) over per-page key min/max,
 *      k = budget / page_size;
 *   3. loads the union of those pages once per GQA group and recomputes the
 *      prefix output o_p and log-normaliser L_p of the active tokens over
 *      their own pages; stable tokens reuse last step's o_p, L_p untouched;
 *   4. attends every block token densely to the block's own keys (o_s, L_s);
 *   5. merges prefix and suffix with the online-softmax (log-sum-exp) merge.
 *
 * The first denoising step of a block is a dense pass over the whole prefix
 * that fills the cache for every block token (paper, limitations: the
 * cold-start dense step), and the page min/max metadata is built once per
 * prefix.
 *
 * Conventions for every entry point
 * ---------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *   in the row-major layouts given below (innermost index last), 16-byte
 *   aligned.  The library never allocates or frees memory and keeps no state
 *   between calls; the workspace is caller-owned scratch (losa_step_noalloc
 *   alone uses a fixed array owned by the library instead).
 * - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *   legacy default stream).  Host-side validation happens before any launch;
 *   a call that returns an error has launched nothing, except LOSA_ERR_CUDA
 *   after a failed launch.
 * - Stream order holds for every input, including one written by the
 *   kernel right before the call: the step's kernels are chained by
 *   programmatic dependent launch, and none reads an argument before the
 *   work queued ahead of the call has completed.
 * - Element types: LOSA_BF16 (bfloat16) or LOSA_F32 (float) for Q, K, V and
 *   the page metadata; the cached prefix state, the outputs and all
 *   accumulation are fp32.
 * - Sizes:  S sequences, Hq query heads, Hkv KV heads (G = Hq / Hkv query
 *   heads share KV head g = h / G), d = head_dim, L = prefix_len,
 *   ps = page_size, P = ceil(L / ps) pages (the last may be partial),
 *   B = block_size, A = n_active, k = min(token_budget / ps, P).
 * - Prefix buffers have a capacity Lc = prefix_capacity (>= L; 0 means L):
 *   prefix K/V are [S][Hkv][Lc][d] (tokens L..Lc-1 of each (s, g) are
 *   unused), and the page metadata has Pc = ceil(Lc / ps) records per
 *   (s, g).  losa_append_block grows L inside that capacity.
 * - Variable-length batches: with losa_shape.prefix_lens set, sequence s has
 *   its own prefix length L_s (P_s = ceil(L_s / ps) pages); prefix_len is
 *   then the largest length and sizes the buffers, the workspaces and k.
 *   Every sequence gets what a one-sequence call with prefix_len = L_s
 *   gives (up to rounding order), except that its rows of page_idx are
 *   padded with -1 past min(k, P_s) entries; tokens L_s..Lc-1 of its prefix
 *   buffers are never used, whatever they hold.  The array is read on the
 *   device in stream order (it may be written by the kernel right before the
 *   call, and a captured graph reads its current contents).  An entry
 *   outside [1, L] is clamped into it; losa_dense_prefix and the step calls
 *   also report it as LOSA_ERR_DEVICE_BOUNDS through losa_read_device_status.
 */
#ifndef LOSA_H_
#define LOSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ----------------------------------------------------- */
#define LOSA_OK                 0
#define LOSA_ERR_INVALID_ARG    1  /* null/misaligned pointer, inconsistent sizes      */
#define LOSA_ERR_UNSUPPORTED    2  /* valid but outside what the kernels implement     */
#define LOSA_ERR_CUDA           3  /* a CUDA launch failed (message: losa_last_error)  */
#define LOSA_ERR_DEVICE_TIMEOUT 4  /* a bounded device-side wait gave up               */
#define LOSA_ERR_DEVICE_BOUNDS  5  /* a device-side index check failed (access skipped)*/

/* ---- element types ---------------------------------------------------- */
#define LOSA_F32  0
#define LOSA_BF16 1

/* ---- workspace kinds -------------------------------------------------- */
#define LOSA_WS_DENSE 0
#define LOSA_WS_STEP  1

/* Problem shape shared by every call.  Limits checked by the library:
 * head_dim == 128, page_size == 16 (LOSA_ERR_UNSUPPORTED otherwise);
 * 1 <= block_size <= 32; G * block_size <= 128; 0 <= n_active <= block_size;
 * n_active > 0 needs k >= 1; k <= 64 unless k == P (every page selected). */
typedef struct {
    int32_t num_seqs;      /* S                                           */
    int32_t n_q_heads;     /* Hq                                          */
    int32_t n_kv_heads;    /* Hkv, Hq % Hkv == 0                          */
    int32_t head_dim;      /* d                                           */
    int32_t prefix_len;    /* L >= 1                                      */
    int32_t page_size;     /* ps                                          */
    int32_t block_size;    /* B                                           */
    int32_t n_active;      /* |A| per query head                          */
    int32_t token_budget;  /* prefix tokens each active query may attend  */
    float   scale;         /* softmax scale; 0 selects 1/sqrt(d)          */
    int32_t dtype;         /* LOSA_F32 or LOSA_BF16                       */
    int32_t flags;         /* 0, or LOSA_STEP_ATTEND_UNION (below)        */
    int32_t prefix_capacity; /* Lc >= L tokens per (s, g) in the prefix
                                buffers; 0 selects L                       */
    const int32_t* prefix_lens; /* NULL, or a DEVICE array [S] (4-byte
                                aligned) of per-sequence prefix lengths
                                1 <= L_s <= L: a variable-length batch   */
} losa_shape;

/* ---- step variants (losa_shape.flags) ----------------------------------
 * LOSA_STEP_ATTEND_UNION: each active row attends to every page of its GQA
 *   group's union -- the pages the step loads once per (sequence, KV head),
 *   paper, methodology: sparse computation for active tokens -- instead of
 *   only its own top-k pages.  Selection (active_idx, page_idx) and the union
 *   are unchanged; o_p/L_p of active rows cover more prefix tokens for the
 *   same HBM traffic.  Only losa_step / losa_step_ref / losa_step_noalloc
 *   read the flag; any other bit is LOSA_ERR_INVALID_ARG. */
#define LOSA_STEP_ATTEND_UNION 1

/* Bytes of page metadata for `shape` (the size of `page_meta` below): the
 * records, then the page-norm rows. */
size_t losa_page_meta_size(const losa_shape* shape);

/* Bytes of workspace needed by losa_dense_prefix (which = LOSA_WS_DENSE) or
 * losa_step (LOSA_WS_STEP).  0 for an invalid shape. */
size_t losa_workspace_size(const losa_shape* shape, int which);

/*
 * Page metadata build (once per prefix): for every page and channel, the min
 * and max of the keys of the page's valid tokens -- what the QUEST bound
 * needs (paper, methodology: QUEST-style page selection over KV pages).
 *
 *   k_prefix   [S][Hkv][Lc][d]  keys, element type `dtype` (tokens < L read)
 *   page_meta  out, losa_page_meta_size() bytes, element type `dtype`:
 *              for page p of (s, g), a record of 2*d elements -- kmin[0..d)
 *              then kmax[0..d) -- at record index (s*Hkv + g)*Pc + p.  Inside
 *              a record the 16-byte chunks are stored XOR-swizzled: logical
 *              chunk c sits at chunk position c ^ (p & 7).  (This keeps the
 *              scoring kernel's shared-memory reads free of bank conflicts.)
 *              After the S*Hkv*Pc records: for every (s, g) a row of
 *              Pn = ceil(Pc / 8) * 8 float pairs, pair p = (||kmin||_2,
 *              ||kmax||_2) of page p, computed in fp32 with every operation
 *              rounded up (upper bounds of the exact norms; the step uses them
 *              to bound the rounding error of its tensor-core page scores).
 *              The row padding past a sequence's pages is never written.
 * Min/max introduce no rounding: the values are exact copies of key values.
 * With prefix_lens, sequence s gets records for its own P_s pages (the last
 * over its tokens < L_s only); its records from P_s on are not written.
 */
int losa_build_page_meta(const losa_shape* shape, const void* k_prefix, void* page_meta,
                         void* stream);

/*
 * Prefix growth: commit a finished block to the prefix.  When a block's last
 * denoising step is done its tokens become prefix tokens for the blocks
 * after it (paper, block-wise generation: each block is generated
 * conditioned on the committed prefix).  This copies the block's keys and
 * values into prefix positions L .. L+B-1 of every (s, g) and rebuilds the
 * min/max records of the pages those positions touch (the old last page, if
 * it was partial, and the new ones), exactly as losa_build_page_meta would
 * on the grown prefix.  Afterwards the caller uses prefix_len = L + B.
 *
 *   shape      the shape BEFORE the append (prefix_len = L); requires
 *              L + B <= prefix capacity (LOSA_ERR_INVALID_ARG otherwise).
 *              With prefix_lens, sequence s appends at its own L_s (and the
 *              caller then adds B to every entry and to prefix_len).
 *   k_blk,
 *   v_blk      [S][Hkv][B][d]   the committed block's keys/values
 *   k_prefix,
 *   v_prefix   in/out [S][Hkv][Lc][d]
 *   page_meta  in/out, built for the prefix of length L
 * Other pages' records and prefix tokens < L are not written.
 */
int losa_append_block(const losa_shape* shape, const void* k_blk, const void* v_blk,
                      void* k_prefix, void* v_prefix, void* page_meta, void* stream);

/*
 * Cold-start dense pass (first denoising step of a block; paper,
 * limitations): every block token attends to the whole prefix, which fills
 * the cached prefix state of every row; then dense suffix attention over the
 * block and the log-sum-exp merge give the step output.
 *
 *   q          [S][Hq][B][d]    queries of this step
 *   k_prefix,
 *   v_prefix   [S][Hkv][Lc][d]
 *   k_blk,
 *   v_blk      [S][Hkv][B][d]   the block's own keys/values
 *   o_p        out [S][Hq][B][d] fp32  prefix output, all rows
 *   l_p        out [S][Hq][B]    fp32  prefix log-normaliser (natural log)
 *   out        out [S][Hq][B][d] fp32  attention over prefix + block
 *   out_lse    out [S][Hq][B]    fp32  its log-normaliser; may be NULL
 *   workspace  >= losa_workspace_size(shape, LOSA_WS_DENSE) bytes, 256-byte
 *              aligned; contents on entry are irrelevant.
 */
int losa_dense_prefix(const losa_shape* shape, const void* q, const void* k_prefix,
                      const void* v_prefix, const void* k_blk, const void* v_blk, float* o_p,
                      float* l_p, float* out, float* out_lse, void* workspace, size_t ws_bytes,
                      void* stream);

/*
 * One LoSA denoising step (steps 2..T of a block; paper, methodology).
 *
 *   q_cur      [S][Hq][B][d]    this step's queries
 *   q_prev     [S][Hq][B][d]    the previous step's queries (caller rotates)
 *   k_prefix,
 *   v_prefix   [S][Hkv][Lc][d]
 *   page_meta  from losa_build_page_meta on the same k_prefix
 *   k_blk,
 *   v_blk      [S][Hkv][B][d]
 *   o_p, l_p   in/out cached prefix state [S][Hq][B][d], [S][Hq][B] fp32:
 *              rows of active tokens are overwritten with their sparse
 *              prefix result; rows of stable tokens are not written at all.
 *   out        out [S][Hq][B][d] fp32; must not alias any input
 *   out_lse    out [S][Hq][B] fp32; may be NULL
 *   active_idx optional out [S][Hq][A] int32: active tokens, ascending
 *   page_idx   optional out [S][Hq][A][k] int32: each active row's pages,
 *              ascending (then -1 past a short sequence's P_s pages)
 *   union_count optional out [S][Hkv] int32: distinct pages loaded per
 *              (sequence, KV head) -- the union over its G*A active rows
 *   workspace  >= losa_workspace_size(shape, LOSA_WS_STEP) bytes, 256-byte
 *              aligned; contents on entry are irrelevant.
 * Selection rules: the active set is the top-A tokens by MSE (fp32, channels
 * summed in order), ties to the lower token index; pages are the top-k by the
 * bound (ties to the lower page index, -0 == +0).  n_active == 0 is legal
 * (every row reuses its cache); n_active == B with k == P equals dense
 * attention.
 */
int losa_step(const losa_shape* shape, const void* q_cur, const void* q_prev,
              const void* k_prefix, const void* v_prefix, const void* page_meta,
              const void* k_blk, const void* v_blk, float* o_p, float* l_p, float* out,
              float* out_lse, int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
              void* workspace, size_t ws_bytes, void* stream);

/*
 * Drift-safe locality (a variant of losa_step).  The pages score a token's
 * locality between denoising steps t-1 and t (methodology: locality
 * pruning).  A stable token, though, keeps the prefix state computed from
 * the query it had when it was last recomputed, and a slow drift in one
 * direction never shows between two adjacent steps.  This entry point scores
 * every token against that reference query instead:
 *
 *   q_ref  in/out [S][Hq][B][d], element type `dtype`: on entry, for each
 *          row, the query its cached o_p/L_p were computed from (after the
 *          cold-start dense pass: that pass's q).  The locality score is the
 *          MSE of q_cur against q_ref.  On return the active rows hold
 *          q_cur (their cache was recomputed from it); the other rows are
 *          unchanged.  Must not overlap q_cur or any output.
 *
 * Every other argument, result and error is losa_step's (q_prev is replaced
 * by q_ref).  The rewrite of q_ref happens after every read of it in this
 * call, on `stream`.
 */
int losa_step_ref(const losa_shape* shape, const void* q_cur, void* q_ref,
                  const void* k_prefix, const void* v_prefix, const void* page_meta,
                  const void* k_blk, const void* v_blk, float* o_p, float* l_p, float* out,
                  float* out_lse, int32_t* active_idx, int32_t* page_idx, int32_t* union_count,
                  void* workspace, size_t ws_bytes, void* stream);

/* Size of the scratch array behind losa_step_noalloc: 8 MiB per GPU. */
#define LOSA_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)

/*
 * losa_step for callers that cannot allocate device memory.  The paper has
 * no counterpart to this entry point; it exists for callers such as a plugin
 * inside a host framework whose caching allocator already owns the GPU's
 * memory (where a raw cudaMalloc fails or fragments that pool), or a
 * latency-critical loop that must not call cudaMalloc/cudaFree because they
 * can synchronise the device.
 *
 * Same arguments and results as losa_step, minus `workspace`/`ws_bytes`: the
 * scratch is a LOSA_NOALLOC_SCRATCH_BYTES array in device global memory that
 * belongs to this library.  Every GPU that loads the library holds that
 * array until the process exits.  This function itself allocates nothing
 * (no cudaMalloc, no cudaFree, no allocating library routine).
 *  - Shapes whose losa_workspace_size(shape, LOSA_WS_STEP) exceeds
 *    LOSA_NOALLOC_SCRATCH_BYTES are rejected with LOSA_ERR_UNSUPPORTED before
 *    anything is launched.
 *  - The first call on a device looks up the array's device address (once
 *    per device, with that device current); make that first call before any
 *    stream capture on that device.
 *  - All calls on a device share the one array, which keeps whatever the
 *    last call left in it.  losa_step needs nothing there to start at zero,
 *    so those leftovers are harmless while every call ends with LOSA_OK;
 *    read the device-side status with losa_noalloc_read_status.
 *    Calls that can overlap on the GPU -- on different streams without an
 *    ordering between them -- race on the array and give wrong results;
 *    order them on one stream or with events.
 *  - The array's address is looked up once per device and kept; after a
 *    cudaDeviceReset on that device the library's module (and the array)
 *    is gone, and later calls in the same process are invalid.
 */
int losa_step_noalloc(const losa_shape* shape, const void* q_cur, const void* q_prev,
                      const void* k_prefix, const void* v_prefix, const void* page_meta,
                      const void* k_blk, const void* v_blk, float* o_p, float* l_p, float* out,
                      float* out_lse, int32_t* active_idx, int32_t* page_idx,
                      int32_t* union_count, void* stream);

/* losa_read_device_status for the scratch array of losa_step_noalloc on the
 * current device: synchronises `stream`, returns the status the noalloc
 * calls recorded there (LOSA_OK, LOSA_ERR_DEVICE_TIMEOUT or
 * LOSA_ERR_DEVICE_BOUNDS) and clears it.  Allocates nothing.  The paper has
 * no counterpart to this entry point either. */
int losa_noalloc_read_status(void* stream);

/* Synchronises `stream`, then returns the device-side status recorded in the
 * workspace by the last call that used it (LOSA_OK, LOSA_ERR_DEVICE_TIMEOUT
 * or LOSA_ERR_DEVICE_BOUNDS) and clears it.  LOSA_ERR_CUDA if the copy
 * fails. */
int losa_read_device_status(void* workspace, void* stream);

/* Static description of a status code. */
const char* losa_status_string(int status);

/* Message of the last LOSA_ERR_CUDA on the calling thread ("" if none). */
const char* losa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LOSA_H_ */
