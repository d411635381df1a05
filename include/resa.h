/*
 * resa.h - C ABI of libresa.so, the B200 (sm_100a) implementation of the
 * attention hot path of Rectified Sparse Attention (ReSA, arXiv 2506.04108).
 *
 * Method (pages describing ReSA; "Rectified Sparse Attention", pith.science
 * review, section "What carries the argument", Eq. 2, Eq. 5, Eq. 6):
 *   - group block sparse attention (GBSA): keys are cut into blocks of b = 16
 *     tokens; each block keeps a per-channel min/max descriptor (Quest); every
 *     GQA group scores all blocks with the pooled Quest bound and all query
 *     heads of the group attend to the same top-n blocks;
 *   - n = max(n_min, ceil(M r)) with M the number of blocks and r the active
 *     block ratio (Eq. 5; the pages' p read as the active ratio), capped at M;
 *   - the block that holds the newest token is always kept (n_local = 1);
 *   - dense rectification: every f decode steps the last f tokens are
 *     re-encoded with dense causal attention, their KV entries replaced and
 *     the block statistics updated.
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *     and 16-byte aligned. The library allocates no memory and keeps no state
 *     between calls apart from a per-device cache of launch attributes.
 *   - Layouts (row-major, innermost last):
 *       k_cache, v_cache  [batch][n_kv_heads][max_len][head_dim]
 *       desc              [batch][n_kv_heads][max_len/16][2][head_dim]
 *                         (row 0 = per-channel min, row 1 = max of the valid
 *                          keys of the block; same dtype as the cache)
 *       q, out            [batch][n_q_heads][head_dim]
 *       k_new, v_new      [batch][n_kv_heads][head_dim]
 *       q_f, out_f        [batch][f][n_q_heads][head_dim]
 *       k_f, v_f          [batch][f][n_kv_heads][head_dim]
 *       lse               [batch][n_q_heads]           float32
 *       sel               [batch][n_kv_heads][n]        int32, ascending
 *   - Query head h reads KV head h / (n_q_heads / n_kv_heads).
 *   - `len` is the number of valid tokens in the cache, counting the token a
 *     decode call appends. All batch rows share one len, except in the
 *     *_varlen calls, where row b has lens[b] tokens (see below).
 *   - q, k, v, desc and out share the dtype in resa_dims.dtype; softmax and
 *     accumulation are float32; softmax_scale must be finite and positive.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call
 *     only enqueues work on it and returns; nothing synchronises.
 *   - `workspace` is caller-provided device scratch of at least
 *     resa_workspace_bytes() bytes, 256-byte aligned. Zero all of it once
 *     before first use: it holds an error word and arrival counters that every
 *     call leaves at zero again. After a call reports an error, zero it again.
 *     Calls that share one workspace must be ordered on one stream.
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid argument returns a negative resa_status and launches nothing.
 *     A failed launch returns RESA_ERR_CUDA. A device-side wait that gives up
 *     sets a flag in the workspace control block, read by
 *     resa_workspace_status().
 */
#ifndef RESA_H_
#define RESA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RESA_API __attribute__((visibility("default")))
#else
#define RESA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RESA_OK = 0,
  RESA_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misalignment, len/f/r out of range */
  RESA_ERR_UNSUPPORTED = -2,  /* head_dim not 64/128, group > 8, block_size != 16,
                                 more than 262144 blocks (4M tokens) to select from */
  RESA_ERR_CAPACITY = -3,     /* len > max_len */
  RESA_ERR_WORKSPACE = -4,    /* workspace smaller than resa_workspace_bytes() */
  RESA_ERR_CUDA = -5,         /* a CUDA runtime/driver call or launch failed */
  RESA_ERR_TIMEOUT = -6,      /* a device-side wait gave up (flag in the workspace) */
  RESA_ERR_BAD_INDEX = -7     /* a block id in `sel`, or an entry of `lens`, was out of
                                 range (flag in the workspace) */
} resa_status;

typedef enum { RESA_F32 = 0, RESA_BF16 = 1 } resa_dtype;

typedef struct {
  int32_t batch;       /* B >= 1 */
  int32_t n_q_heads;   /* H_q, a multiple of n_kv_heads */
  int32_t n_kv_heads;  /* H_kv >= 1; group G = H_q / H_kv must be <= 8 */
  int32_t head_dim;    /* d: 64 or 128 */
  int32_t block_size;  /* b: must be 16 */
  int32_t dtype;       /* resa_dtype of q, k, v, desc, out */
  int64_t max_len;     /* cache capacity in tokens, a positive multiple of 16 */
} resa_dims;

/* Block budget of Eq. 5: M = ceil(len / 16) blocks (the partial block counts),
 * n = min(M, max(n_min, ceil(M * r))) with ceil(M * r) evaluated in double as
 * ceil(M * r - 1e-9). Returns n, or a negative resa_status for len < 1,
 * r not in (0, 1], n_min < 1 or block_size != 16. */
RESA_API int32_t resa_num_selected(int64_t len, int32_t block_size, double r, int32_t n_min);

/* Workspace bytes that suffice for resa_decode_sparse, resa_decode_dense and
 * resa_rectify (with any window 1 <= f' <= f) at any length up to `len`, and
 * for the *_varlen calls with len_bound <= len. f = 0 sizes a workspace for
 * the decode and prefill calls only (a rectification given one returns
 * RESA_ERR_WORKSPACE). Returns 0 for invalid dims, len < 1 or f outside
 * [0, 256]. */
RESA_API size_t resa_workspace_bytes(const resa_dims* dims, int64_t len, int32_t f);

/* Quest block descriptors of the first `len` tokens (per-block, per-channel
 * key minimum and maximum; section "What carries the argument"): for every batch
 * row, KV head and block j < ceil(len/16), desc[..][j][0][c] = min and
 * desc[..][j][1][c] = max of k_cache[..][t][c] over the valid tokens
 * t in [16 j, min(16 j + 16, len)). Blocks at or past ceil(len/16) are not
 * written. */
RESA_API int resa_build_desc(const resa_dims* dims, const void* k_cache, int64_t len, void* desc,
                    void* stream);

/* One GBSA decode step (section "What carries the argument"; Eq. 2, Eq. 5):
 *  1. if k_new != NULL: write k_new/v_new at slot len-1 and merge k_new into
 *     the descriptor of block (len-1)/16 (set it to (k_new, k_new) when the
 *     token opens a new block);
 *  2. per (batch, KV group) and block j < M-1:
 *     s_j = sum_{h in group} sum_c max(q_hc * min_jc, q_hc * max_jc);
 *  3. keep block M-1 plus the n-1 best other blocks (ties to the lower index),
 *     n = resa_num_selected(len, 16, r, n_min); written ascending to `sel`
 *     when sel != NULL;
 *  4. every query head attends (softmax(scale * q.k) v) over the tokens of the
 *     selected blocks that are < len, split across CTAs and merged by
 *     log-sum-exp (Flash-Decoding);
 *  5. out = the result in the cache dtype; lse (if not NULL) = natural-log
 *     log-sum-exp of the scaled logits.
 * k_new and v_new are both NULL or both set. */
RESA_API int resa_decode_sparse(const resa_dims* dims, const void* q, const void* k_new,
                       const void* v_new, void* k_cache, void* v_cache, void* desc,
                       int64_t len, double r, int32_t n_min, float softmax_scale, void* out,
                       float* lse, int32_t* sel, void* workspace, size_t workspace_bytes,
                       void* stream);

/* Steps 1-3 of resa_decode_sparse alone (append, group scores, top-n): writes
 * the ascending block list to `sel` ([batch][n_kv_heads][n], required) with
 * n = resa_num_selected(len, 16, r, n_min). Together with
 * resa_attend_blocks this is exactly resa_decode_sparse. */
RESA_API int resa_select_blocks(const resa_dims* dims, const void* q, const void* k_new,
                                const void* v_new, void* k_cache, void* v_cache, void* desc,
                                int64_t len, double r, int32_t n_min, int32_t* sel,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Steps 4-5 of resa_decode_sparse alone: every query head attends over the
 * tokens (< len) of the n_sel blocks its KV group lists in `sel`
 * ([batch][n_kv_heads][n_sel], distinct block ids below ceil(len/16), in any
 * order; 1 <= n_sel <= ceil(len/16)). An id outside that range is skipped and
 * raises the RESA_ERR_BAD_INDEX flag read by resa_workspace_status(). */
RESA_API int resa_attend_blocks(const resa_dims* dims, const void* q, const void* k_cache,
                                const void* v_cache, int64_t len, const int32_t* sel,
                                int32_t n_sel, float softmax_scale, void* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Dense decode of the same step: step 1 of resa_decode_sparse (desc may be
 * NULL, then descriptors are not updated), then attention over every token
 * < len. This is the r = 1 comparison arm; it skips scoring and selection. */
RESA_API int resa_decode_dense(const resa_dims* dims, const void* q, const void* k_new,
                      const void* v_new, void* k_cache, void* v_cache, void* desc, int64_t len,
                      float softmax_scale, void* out, float* lse, void* workspace,
                      size_t workspace_bytes, void* stream);

/* Dense rectification (section "What carries the argument": after every f
 * decode steps the newest f tokens go through one dense causal pass whose K/V
 * overwrite the ones the sparse steps produced, and the affected block
 * summaries are refreshed; f = 32 by default, "Assumptions & free
 * parameters"):
 *  1. k_cache/v_cache slots [len-f, len) := k_f/v_f;
 *  2. descriptors of blocks (len-f)/16 .. ceil(len/16)-1 recomputed from the
 *     full block contents;
 *  3. out_f[b][i][h] = causal dense attention of q_f[b][i][h], whose position
 *     is len-f+i, over keys 0 .. len-f+i.
 * Requires 1 <= f <= len and f <= 256. */
RESA_API int resa_rectify(const resa_dims* dims, const void* q_f, const void* k_f, const void* v_f,
                 void* k_cache, void* v_cache, void* desc, int64_t len, int32_t f,
                 float softmax_scale, void* out_f, void* workspace, size_t workspace_bytes,
                 void* stream);

/* resa_decode_sparse without a caller-provided workspace. The method has no
 * counterpart for this call; it exists for callers that cannot allocate
 * device memory themselves (a framework's caching allocator owns the GPU, a
 * decode loop captured into CUDA graphs must not allocate, a plugin host only
 * passes input and output pointers).
 *  - Scratch is a fixed 16 MiB array inside libresa.so's device memory, held
 *    by every GPU that loads the library until the process exits. Calls whose
 *    resa_workspace_bytes(dims, len, 0) exceeds 16 MiB return
 *    RESA_ERR_WORKSPACE and launch nothing.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) and caches it; make that first call outside any
 *    stream capture.
 *  - Each call clears the array's arrival counters on `stream`
 *    (cudaMemsetAsync), then runs resa_decode_sparse on it. It allocates
 *    nothing. All calls on a device share the one array: calls that may
 *    overlap on the GPU (different streams, different threads) race and must
 *    be serialised by the caller.
 *  - Device-side errors (a timed-out wait, a bad block id) set the array's
 *    error word, which stays set across later calls until
 *    resa_noalloc_status() reads and clears it.
 *  - After cudaDeviceReset the first call must again come outside any
 *    stream capture (a failed call forgets the cached address).
 * Arguments and results are those of resa_decode_sparse. */
RESA_API int resa_decode_sparse_noalloc(const resa_dims* dims, const void* q, const void* k_new,
                                        const void* v_new, void* k_cache, void* v_cache,
                                        void* desc, int64_t len, double r, int32_t n_min,
                                        float softmax_scale, void* out, float* lse,
                                        int32_t* sel, void* stream);

/* Device error flags of the array resa_decode_sparse_noalloc uses on the
 * current device (no counterpart in the method): synchronises `stream`, then
 * reads and clears them, as resa_workspace_status() does for a caller
 * workspace. Returns RESA_OK, RESA_ERR_TIMEOUT, RESA_ERR_BAD_INDEX or
 * RESA_ERR_CUDA. */
RESA_API int resa_noalloc_status(void* stream);

/* Prefill-side step: dense causal attention of every position of a prompt,
 * with the Quest descriptors of its keys produced by the same pass ("Rectified
 * Sparse Attention", section "What carries the argument": decoding starts from
 * a prefilled cache whose blocks carry min/max descriptors; the causal pass is
 * the one the rectification applies to its last f tokens, here over all of
 * them).
 *  - q, out: [batch][len][n_q_heads][head_dim]; k_cache, v_cache hold the
 *    prompt's keys and values in slots [0, len) (read only);
 *  - out[b][i][h] = softmax_t(scale * q[b][i][h] . k[b][h/G][t], t <= i) . V;
 *  - desc receives the descriptors of blocks 0 .. ceil(len/16)-1, exactly as
 *    resa_build_desc(len) writes them, taken from the key tiles the attention
 *    already holds in shared memory (K is read from HBM once).
 * bf16 and groups of 1, 2, 4 or 8 query heads only (tensor cores; other
 * shapes return RESA_ERR_UNSUPPORTED), as do len * n_q_heads / n_kv_heads >
 * 65535 * 128 rows. The workspace only carries the error word:
 * resa_workspace_bytes(dims, len, 0) suffices. */
RESA_API int resa_prefill(const resa_dims* dims, const void* q, const void* k_cache,
                          const void* v_cache, void* desc, int64_t len, float softmax_scale,
                          void* out, void* workspace, size_t workspace_bytes, void* stream);

/* ---- variable-length batches (continuous batching) ----
 * The pages run ReSA one sequence at a time; batching sequences of different
 * lengths is this library's extension and changes nothing per row: every row
 * computes exactly what the fixed-length call computes at its own length.
 *  - lens: DEVICE int32 array [batch], 4-byte aligned, owned by the caller;
 *    lens[b] is row b's token count (counting a decode call's appended token).
 *  - len_bound >= every lens[b] (for instance the longest row); it sizes the
 *    grids, the workspace (resa_workspace_bytes(dims, len_bound, f)) and the
 *    stride n_cap = resa_num_selected(len_bound, 16, r, n_min) of `sel`.
 *    Host checks apply to len_bound as to len (1 <= len_bound <= max_len).
 *  - An entry outside [1, len_bound] is clamped into it and raises the
 *    RESA_ERR_BAD_INDEX flag read by resa_workspace_status() (no flag for
 *    resa_build_desc_varlen, which has no workspace).
 *  - lens is read on the device only: the calls can be captured in a CUDA
 *    graph once and replayed while the lengths change. */

/* resa_build_desc for every row b over its first lens[b] tokens. */
RESA_API int resa_build_desc_varlen(const resa_dims* dims, const void* k_cache,
                                    const int32_t* lens, int64_t len_bound, void* desc,
                                    void* stream);

/* resa_decode_sparse with row b at length lens[b]: the appended token goes to
 * slot lens[b]-1, row b's KV groups select n_b = resa_num_selected(lens[b],
 * 16, r, n_min) of its ceil(lens[b]/16) blocks. sel (optional) is
 * [batch][n_kv_heads][n_cap]: n_b ascending ids, then -1 up to n_cap.
 * Always runs the three-kernel path. */
RESA_API int resa_decode_sparse_varlen(const resa_dims* dims, const void* q, const void* k_new,
                                       const void* v_new, void* k_cache, void* v_cache,
                                       void* desc, const int32_t* lens, int64_t len_bound,
                                       double r, int32_t n_min, float softmax_scale, void* out,
                                       float* lse, int32_t* sel, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* resa_decode_dense with row b at length lens[b]. */
RESA_API int resa_decode_dense_varlen(const resa_dims* dims, const void* q, const void* k_new,
                                      const void* v_new, void* k_cache, void* v_cache,
                                      void* desc, const int32_t* lens, int64_t len_bound,
                                      float softmax_scale, void* out, float* lse,
                                      void* workspace, size_t workspace_bytes, void* stream);

/* resa_rectify with row b at length lens[b] and its own window w_b, so rows
 * can sit at different rectification phases: w_b = windows[b] (device int32
 * [batch], 4-byte aligned), or f for every row when windows is NULL. Row b
 * uses the first w_b rows of its q_f/k_f/v_f block ([batch][f][..] as in
 * resa_rectify): slots [lens[b]-w_b, lens[b]) are rewritten, the blocks they
 * touch refreshed, and out_f[b][i] (i < w_b) is the causal dense attention of
 * q_f[b][i] at position lens[b]-w_b+i. Rows i >= w_b of out_f are not
 * written. A row with w_b = 0, or with lens[b] < w_b, is left untouched
 * (cache, descriptors and out_f). A window outside [0, f] is clamped into it
 * and raises the RESA_ERR_BAD_INDEX flag. Requires 1 <= f <= len_bound and
 * f <= 256. */
RESA_API int resa_rectify_varlen(const resa_dims* dims, const void* q_f, const void* k_f,
                                 const void* v_f, void* k_cache, void* v_cache, void* desc,
                                 const int32_t* lens, const int32_t* windows, int64_t len_bound,
                                 int32_t f, float softmax_scale, void* out_f, void* workspace,
                                 size_t workspace_bytes, void* stream);

/* Failure-detection check of the device-side bounded wait (no counterpart in
 * the method): one thread waits until the device int32 *flag >= target, as
 * the one-launch decode kernel's group barrier waits on its arrival counter,
 * for at most limit_us microseconds (1 .. 2,000,000). A wait that runs out
 * sets the RESA_ERR_TIMEOUT flag of `workspace` (read by
 * resa_workspace_status()) and the kernel returns: the context stays usable.
 * Passing a flag that nothing sets checks that a stuck wait ends and is
 * reported. flag: 4-byte aligned device pointer; workspace: as for the other
 * calls. Only enqueues work on `stream`. */
RESA_API int resa_wait_check(const int32_t* flag, int32_t target, uint32_t limit_us,
                             void* workspace, void* stream);

/* Synchronises `stream`, then reads and clears the device error flags of the
 * workspace control block. Returns RESA_OK, RESA_ERR_TIMEOUT,
 * RESA_ERR_BAD_INDEX or RESA_ERR_CUDA. */
RESA_API int resa_workspace_status(void* workspace, void* stream);

/* Human-readable name of a resa_status value (static string). */
RESA_API const char* resa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* RESA_H_ */
