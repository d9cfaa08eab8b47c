/*
 * dsa.h -- C ABI of libdsa.so, the B200 (sm_100a) implementation of the
 * DeepSeek Sparse Attention hot path described on the page
 * "2.2.1 · DSA 与索引器: 先召回 token, 再计算 Sparse MLA":
 *
 *   eq. (1)  I[t,s] = sum_j w[t,j] * ReLU(q[t,j] . k[s])        (Lightning Indexer)
 *   eq. (2)  S_t = TopK({I[t,s] : 0 <= s <= t}, min(k, t+1))     (causal selector)
 *   eq. (3)  u_t = Attn(h_t, {c_s : s in S_t})                    (sparse attention)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor arguments are DEVICE pointers to contiguous row-major arrays
 *    owned by the caller.  The library never allocates, frees or synchronises
 *    (except dsa_read_device_status).  Calls are asynchronous on `stream`
 *    (a cudaStream_t passed as void*; NULL = legacy default stream).
 *  - bf16 tensors hold raw bfloat16 bit patterns; FP8 tensors hold E4M3
 *    ("fn", max 448) codes, one byte each, with one positive fp32 scale per
 *    token (the dequantised value is code * scale; §2 keeps the indexer key
 *    cache quantised, with its scales).
 *  - Base pointers of the indexer operands (qI, kI) must be 16-byte aligned
 *    (they are read with TMA); so must w in the decode step and the score
 *    matrix entry point (each token's head weights are staged by a bulk
 *    copy); other tensors need their natural alignment.
 *  - Positions are 0-based.  A query at absolute position t may select keys
 *    0..t (the current token included).  Index outputs have width k: the
 *    min(k, t+1) selected positions first, in unspecified order, then -1.
 *    Equal scores are broken toward the lower position, so the selected set
 *    is unique.  -0.0 and +0.0 are the same score.
 *  - Scratch: calls that need scratch memory take a caller-provided device
 *    workspace of at least the size the matching *_workspace() query returns
 *    (queries depend only on sizes and on the current device's SM count).
 *    Every workspace starts with a 256-byte status header: call
 *    dsa_workspace_init() once after allocating it.  Kernels record the first
 *    device-side failure there (a bounded wait that gave up, an index outside
 *    its row); dsa_read_device_status() returns and clears it.  Kernels never
 *    trap; after such a failure the outputs of that call are unspecified.
 *  - Host-side argument checks return DSA_ERR_INVALID_ARG / _UNSUPPORTED /
 *    _WORKSPACE before anything is launched; a failed launch returns
 *    DSA_ERR_CUDA.  dsa_last_error() gives a message (thread-local).
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* bad size, null or misaligned pointer */
  DSA_ERR_UNSUPPORTED = 2,   /* a size this build has no kernel for */
  DSA_ERR_WORKSPACE = 3,     /* workspace missing or too small */
  DSA_ERR_CUDA = 4,          /* a CUDA call or kernel launch failed */
  DSA_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up */
  DSA_ERR_DEVICE_CHECK = 6   /* device: an input failed a device-side check */
} dsa_status;

typedef enum { DSA_BF16 = 0, DSA_FP8_E4M3 = 1 } dsa_dtype;

/* Library version string. */
const char* dsa_version(void);
/* Message for the last non-OK status returned on this thread ("" if none). */
const char* dsa_last_error(void);
/* Name of a status code. */
const char* dsa_status_string(int status);

/* Time limit of every device-side wait (default 2 s).  Applies to later launches. */
void dsa_set_wait_timeout_ns(uint64_t ns);
uint64_t dsa_get_wait_timeout_ns(void);

/* Zero the 256-byte status header at the start of a workspace (async). */
dsa_status dsa_workspace_init(void* workspace, size_t workspace_bytes, void* stream);
/* Synchronise `stream`, return the device status recorded in `workspace`
 * (DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_CHECK), store its detail word in
 * *detail if non-NULL, and clear it.  The first failure of a launch wins.
 * Detail words: DSA_ERR_TIMEOUT -> the wait that gave up (0x1xxx indexer
 * prefill, 0x2xxx sparse attention, 0x3101 sparse-stage teacher,
 * 0x1xx..0x3xx indexer scan, 0x7e57 self-test);
 * DSA_ERR_DEVICE_CHECK -> 0xA77E an attention, teacher or KL index outside
 * [-1, L),
 * 0x70E1 a top-k row longer than its matrix, 0x5e1ec6..0x5e1ec9 a selection
 * whose candidate count broke its invariant (output slots may then hold
 * any in-range position or -1). */
dsa_status dsa_read_device_status(void* workspace, void* stream, uint32_t* detail);

/* ------------------------------------------------------------------------
 * Prefill: fused Lightning Indexer + causal top-k  (eqs. (1) and (2), §1.1;
 * the fusion of §2: score tiles are filtered as they are produced and merged
 * into each row's top-k, the score matrix is never written).
 *
 * Query rows i = 0..nq-1 of each of B sequences sit at absolute positions
 * t = q_offset + i; keys 0..kv_len-1 are available (kv_len >= q_offset + nq).
 *   qI      [B, nq, HI, dI]  bf16 or e4m3 codes
 *   q_scale [B, nq]          fp32, FP8 only (else NULL): one scale per query token
 *   kI      [B, kv_len, dI]  bf16 or e4m3 codes
 *   k_scale [B, kv_len]      fp32, FP8 only (else NULL)
 *   w       [B, nq, HI]      fp32 head weights (any sign)
 *   idx_out [B, nq, k]       int32 output (see conventions)
 *   score_out [B, nq, k]     fp32 output or NULL: the fp32 score of each
 *                            selected slot, -inf in padding slots.
 * Supported: HI in {4, 8, 16, 32, 64}; dI <= 128 and a multiple of 8 (bf16)
 * or 16 (FP8); k >= 1.  Chunked prefill = several calls with increasing
 * q_offset over the same kI / workspace.
 * Workspace.  dsa_indexer_topk_prefill_workspace() is bounded independently
 * of the history past 16384 keys: each token streams at most 16384 candidate
 * (score, position) pairs (SMs x 12 x 16384 x 8 B, about 0.23 GB on 148
 * SMs), plus a second-pass area of 64 score rows.  A row whose candidates
 * outgrow that buffer (scores with very many near-ties at its cut-off) is
 * finished by the second pass: its score row is recomputed into the
 * workspace, 64 rows at a time, and selected there by the row top-k (the
 * same selection, from the same eq. (1) scores up to fp32 summation order).
 * With kv_len > 16384 the call therefore reads the overflow count back and
 * synchronises `stream` once.  A workspace of at least
 * dsa_indexer_topk_prefill_workspace_full() bytes (candidate buffers sized
 * for the whole history: no overflow, no synchronisation, the size grows
 * with kv_len) selects that mode instead.
 * ---------------------------------------------------------------------- */
size_t dsa_indexer_topk_prefill_workspace(int B, int nq, int kv_len, int HI, int dI, int k, int dtype);
size_t dsa_indexer_topk_prefill_workspace_full(int B, int nq, int kv_len, int HI, int dI, int k, int dtype);
dsa_status dsa_indexer_topk_prefill(int B, int nq, int q_offset, int kv_len, int HI, int dI, int k, int dtype,
                                    const void* qI, const float* q_scale, const void* kI, const float* k_scale,
                                    const float* w, int32_t* idx_out, float* score_out, void* workspace,
                                    size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Sparse attention, prefill  (eq. (3), §1.1): for each query row and head h,
 *   z_s = scale * q[h] . c_s over the selected s (slots holding -1 skipped),
 *   out[h] = softmax_s(z) . c_s[0:Dv],   lse[h] = log sum_s exp(z_s).
 * The same selected rows serve every head of the row (shared key, §1.1).
 *   q      [B, nq, H, Dqk]  bf16      latent [B, kv_len, Dqk] bf16 (row c_s)
 *   idx    [B, nq, k]       int32 positions in [0, kv_len) or -1
 *   out    [B, nq, H, Dv]   bf16      lse [B, nq, H] fp32 or NULL
 * A row with no valid slot gives out = 0, lse = -inf.  An index outside
 * [-1, kv_len) is skipped and recorded as DSA_ERR_DEVICE_CHECK.
 * Supported: Dqk a multiple of 16, <= 576; Dv a multiple of 64, <= min(512, Dqk);
 * k <= 2048.
 * ---------------------------------------------------------------------- */
size_t dsa_sparse_attn_workspace(void);
dsa_status dsa_sparse_attn_prefill(int B, int nq, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                                   const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Dense masked attention, prefill  (§2, the short-prefill paragraph: for
 * short sequences the fixed costs of top-k, index materialisation and the
 * irregular gather exceed the attention they save, and DSA is run as masked
 * MHA instead; the serving side picks the path by length).  Same result as
 * dsa_sparse_attn_prefill on the same selection (eq. (3), §1.1), computed
 * over dense causal key tiles that a block of 8 tokens shares:
 *   row i of sequence b (absolute position t = q_offset + i) attends the
 *   keys s <= t; if idx is given and t + 1 > k it attends only the
 *   positions its row of idx selects (rows with t + 1 <= k select every
 *   position, eq. (2)); with idx NULL it is plain causal attention over the
 *   whole history, whose lse is the dense normaliser of eq. (15).
 *   q [B, nq, 16, 576] bf16   latent [B, kv_len, 576] bf16 (rows 0..kv_len-1)
 *   idx [B, nq, k] int32 (positions in [0, kv_len) or -1) or NULL
 *   out [B, nq, 16, 512] bf16   lse [B, nq, 16] fp32 or NULL
 * Workspace: dsa_attn_dense_prefill_workspace(B, nq, kv_len, idx != NULL)
 * bytes (the status header, plus one selection bit per (row, key) when idx
 * is given).  An index outside [-1, kv_len) is skipped and recorded as
 * DSA_ERR_DEVICE_CHECK (0xA77E).  Supported: H = 16, Dqk = 576, Dv = 512;
 * q, latent and out 16-byte aligned; q_offset + nq <= kv_len.
 * ---------------------------------------------------------------------- */
size_t dsa_attn_dense_prefill_workspace(int B, int nq, int kv_len, int with_selection);
dsa_status dsa_attn_dense_prefill(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                                  const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* Length dispatch of the prefill attention (§2: the serving side picks the
 * path by length; masked dense attention wins for short histories).
 * dsa_prefill_attention_path returns DSA_PATH_DENSE_MASKED when the chunk's
 * longest history (q_offset + nq keys) is at most 6144 and the shape is the
 * dense kernel's (H = 16, Dqk = 576, Dv = 512), else DSA_PATH_GATHER (the
 * threshold is where the two paths' measured times cross on one B200 with
 * k = 2048).  dsa_attn_prefill runs eq. (3) on that path with the arguments
 * of dsa_attn_dense_prefill (idx required); both paths give the same result
 * on the same selection.  Its workspace is dsa_attn_prefill_workspace(...)
 * bytes. */
enum { DSA_PATH_GATHER = 0, DSA_PATH_DENSE_MASKED = 1 };
int dsa_prefill_attention_path(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k);
size_t dsa_attn_prefill_workspace(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k);
dsa_status dsa_attn_prefill(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                            const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Teacher mass coverage of a selection (§3.1, eq. (15)): for each of `rows`
 * query rows and each head h, the dense attention probabilities on the
 * selected positions sum to exp(lse_sparse[r, h] - lse_dense[r, h]) (the lse
 * outputs of the sparse attention over the selection and of the dense causal
 * attention); the teacher of eq. (16) (heads summed, L1-normalised) covers
 * their mean.  lse_sparse, lse_dense [rows, H] fp32 device arrays; outputs
 * (each may be NULL): m_out [rows] the aggregate M_k, per_head_out [rows, H],
 * min_out [rows] the lowest per-head coverage.  Needs no workspace. */
dsa_status dsa_mass_coverage(int rows, int H, const float* lse_sparse, const float* lse_dense, float* m_out,
                             float* per_head_out, float* min_out, void* stream);

/* ------------------------------------------------------------------------
 * Decode step  (§2: one new query per sequence scans every cached indexer
 * key; the latent cache is shared by all query heads, MQA form).
 * Ragged caches: sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 of
 * kI_cache / latent_cache; its length L_b includes the new token, which is
 * the query at local position L_b - 1.  cu_seqlens is a DEVICE int64 array
 * [B+1]; total_len = cu_seqlens[B] and max_len = max L_b are passed from the
 * host so nothing has to be read back.
 *   qI [B, HI, dI], q_scale [B] (FP8) / NULL, w [B, HI],
 *   kI_cache [total_len, dI], k_scale [total_len] (FP8) / NULL,
 *   idx_out [B, k] local positions, score_out [B, k] or NULL.
 * The step's scores (total_len fp32) live in the workspace.
 * ---------------------------------------------------------------------- */
size_t dsa_indexer_topk_decode_workspace(int B, int HI, int dI, int k, int dtype, int64_t total_len, int max_len);
dsa_status dsa_indexer_topk_decode(int B, int HI, int dI, int k, int dtype, const void* qI, const float* q_scale,
                                   const float* w, const void* kI_cache, const float* k_scale,
                                   const int64_t* cu_seqlens, int64_t total_len, int max_len, int32_t* idx_out,
                                   float* score_out, void* workspace, size_t workspace_bytes, void* stream);

/* dsa_indexer_topk_decode_noalloc: the same decode-step selection as
 * dsa_indexer_topk_decode (same arguments, same results), for callers that
 * cannot allocate device memory and so cannot pass a workspace: for example
 * a component inside a host runtime that owns every device allocation and
 * hands it only its input and output buffers, or code called where no
 * allocator is reachable.  The paper has no counterpart; this is a calling
 * convenience of this library.
 *   Scratch: a buffer built into the library (256 B status word + one fp32
 *   score per cached key), a fixed 16 MiB + 256 B that every GPU which loads
 *   the library holds until the process exits.  Nothing is allocated.
 *   Limit: total_len <= 4,194,304 (2^22) cached keys over all B sequences;
 *   larger steps return DSA_ERR_UNSUPPORTED with a message naming the limit.
 *   Set-up: every call looks up the current device's copy of the buffer
 *   with cudaGetSymbolAddress (a host-side step, so a device reset between
 *   calls is harmless); the first call on a device also loads the library's
 *   module there, so make that first call before any stream capture.
 *   Sharing: every call uses the same buffer, which keeps the last call's
 *   contents; the status word is cleared at the start of each call (the
 *   scores are fully rewritten).  Calls whose work overlaps on the GPU (two
 *   streams, two threads) race on the buffer: order them on one stream.
 *   status_out: NULL, or 2 device uint32 that receive this call's device
 *   status word (code, detail; code 0 = success, else a dsa_status value),
 *   copied on the stream after the kernels. */
dsa_status dsa_indexer_topk_decode_noalloc(int B, int HI, int dI, int k, int dtype, const void* qI,
                                           const float* q_scale, const float* w, const void* kI_cache,
                                           const float* k_scale, const int64_t* cu_seqlens, int64_t total_len,
                                           int max_len, int32_t* idx_out, float* score_out, uint32_t* status_out,
                                           void* stream);

/*   q [B, H, Dqk] bf16, latent_cache [total_len, Dqk] bf16, idx [B, k] local
 *   positions or -1, out [B, H, Dv] bf16, lse [B, H] fp32 or NULL. */
dsa_status dsa_sparse_attn_decode(int B, int H, int Dqk, int Dv, int k, float scale, const void* q,
                                  const void* latent_cache, const int64_t* cu_seqlens, int64_t total_len,
                                  const int32_t* idx, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Debug / test entry points.
 * dsa_indexer_scores: the dense causal score matrix of eq. (1),
 *   scores [B, nq, kv_len] fp32, -inf where s > q_offset + i (small n only).
 * dsa_topk_rows: eq. (2) over materialised rows: row r has row_len[r]
 *   valid scores (row_len NULL: all ncols) at scores + r*row_stride; the
 *   first min(k, len) slots get the selected positions (0..len-1), then -1.
 * dsa_selftest_bounded_wait: runs one kernel whose wait can never complete;
 *   the wait gives up after timeout_ns and the workspace status becomes
 *   DSA_ERR_TIMEOUT (exercises the failure path without hanging the GPU).
 * ---------------------------------------------------------------------- */
size_t dsa_small_workspace(void);
dsa_status dsa_indexer_scores(int B, int nq, int q_offset, int kv_len, int HI, int dI, int dtype, const void* qI,
                              const float* q_scale, const void* kI, const float* k_scale, const float* w,
                              float* scores, void* workspace, size_t workspace_bytes, void* stream);
dsa_status dsa_topk_rows(int rows, int ncols, int64_t row_stride, const float* scores, const int32_t* row_len,
                         int k, int32_t* idx_out, float* val_out, void* workspace, size_t workspace_bytes,
                         void* stream);
dsa_status dsa_selftest_bounded_wait(uint64_t timeout_ns, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Selection diagnostic (§3.1, eq. (14)): the set recall of a student
 * selection S against a teacher selection T is R = |T ∩ S| / k.  For each
 * of `rows` rows of two index arrays idx_a (teacher) and idx_b (student),
 * both [rows, k] int32 (positions, -1 = unused; slot order irrelevant):
 *   inter_out[r]   = |valid(A_r) ∩ valid(B_r)|     (int32, [rows])
 *   count_a_out[r] = |valid(A_r)|                  (int32, [rows], or NULL)
 * so R_r = inter_out[r] / count_a_out[r] (= / k when every row holds k).
 * Positions outside [0, max_pos) are not counted.  max_pos <= 2^20.
 * A row's positions must be distinct within each array (true of every
 * selection this library produces).  Needs no workspace.
 * ---------------------------------------------------------------------- */
dsa_status dsa_selection_overlap(int rows, int k, int max_pos, const int32_t* idx_a, const int32_t* idx_b,
                                 int32_t* inter_out, int32_t* count_a_out, void* stream);

/* ------------------------------------------------------------------------
 * Sparse-stage indexer loss (§1.2, eq. (8)), forward and backward.
 * In the sparse training stage the indexer is fitted, for every token t,
 * by KL_t = D_KL(p_{t,S_t} || Softmax(I_{t,S_t})) on the selected set S_t
 * only; both sides are distributions over S_t (the teacher's weights are
 * divided by their retained mass, the remark after eq. (8)), and I are the
 * eq. (1) scores recomputed on S_t.  The indexer's inputs are detached from
 * the main model, so this loss alone trains the indexer (§1.2).
 *
 *   rows (b, i), i < nq, of a chunk; positions index the sequence's keys.
 *   qI      [B, nq, HI, dI] bf16      kI [B, kv_len, dI] bf16
 *   w       [B, nq, HI]     fp32      idx [B, nq, k] int32 positions in
 *                                     [0, kv_len) or -1 (unused slot);
 *                                     the valid ones distinct in a row
 *   teacher [B, nq, k] fp32 weights >= 0 aligned with idx's slots (any
 *           scale: each row is renormalised over its valid slots)
 *   grad_scale   dL/dKL_t of the caller's loss (1 for the plain sum of
 *                eq. (8), 1/rows for a mean)
 * Outputs (all fp32; every one but kl_out may be NULL to skip it):
 *   kl_out          [B, nq]        KL_t (0 for a row with no valid slot or
 *                                  a teacher with no mass on it)
 *   grad_logits_out [B, nq, k]     dL/dI_{t,s} = grad_scale (softmax - p),
 *                                  0 in unused slots
 *   dq_out          [B, nq, HI, dI] dL/dq^I (overwritten)
 *   dw_out          [B, nq, HI]     dL/dw   (overwritten)
 *   dk_out          [B, kv_len, dI] dL/dk^I ADDED to the buffer (several
 *                                  rows select the same key; the caller
 *                                  zeroes it first), in an unspecified
 *                                  order (float atomics)
 * The ReLU of eq. (1) has derivative 0 at 0.  dq and dk are accumulated
 * from bf16-rounded G = g * w * [q.k > 0] products in fp32.
 * Supported: HI 1..64, dI in {32, 64, 128}, k <= 4096.  Pointers 16-byte
 * aligned (dq 8).  Indices outside [-1, kv_len) are skipped and set
 * DSA_ERR_DEVICE_CHECK (detail 0xA77E) in the workspace status.
 * ---------------------------------------------------------------------- */
size_t dsa_indexer_kl_workspace(void);
dsa_status dsa_indexer_kl_sparse(int B, int nq, int kv_len, int HI, int dI, int k, const void* qI, const void* kI,
                                 const float* w, const int32_t* idx, const float* teacher, float grad_scale,
                                 float* kl_out, float* grad_logits_out, float* dq_out, float* dw_out, float* dk_out,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Sparse-stage teacher (§1.2, the remark after eq. (8), and eq. (16)).
 * When the teacher of eq. (8) comes from the current sparse main attention
 * it is already a distribution over S_t: the heads' attention probabilities
 * a_h(s) = exp(scale q_{t,h} . c_s - lse_{t,h}) summed over the heads and
 * L1-normalised along the selected positions (the DSA aggregation).  This
 * recomputes the attention scores of the selected set from the forward's
 * lse; nothing else of the forward is kept.
 *   q [B, nq, H, Dqk] bf16, latent [B, kv_len, Dqk] bf16, idx [B, nq, k]
 *   (as given to dsa_sparse_attn_prefill), lse [B, nq, H] fp32 (its lse
 *   output), scale (its scale).
 *   p_out [B, nq, k] fp32: p_{t,s} per slot, 0 in unused slots; a row
 *   with no valid slot is all 0.
 * Supported: Dqk a multiple of 16 up to 576, k <= 4096, any H.  q and latent
 * 16-byte aligned.  Indices outside [-1, kv_len) are skipped and set
 * DSA_ERR_DEVICE_CHECK (detail 0xA77E).
 * ---------------------------------------------------------------------- */
dsa_status dsa_attn_teacher_prefill(int B, int nq, int kv_len, int H, int Dqk, int k, float scale, const void* q,
                                    const void* latent, const int32_t* idx, const float* lse, float* p_out,
                                    void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
