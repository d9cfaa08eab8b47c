// api.cu -- the C ABI of libdsa.so (declared in include/dsa.h): argument
// checks, workspace layout, TMA tensor maps and kernel launches.  No entry
// point allocates memory or synchronises except dsa_read_device_status.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "dsa.h"
#include "kernels.h"
#include "sm100.cuh"

namespace {

thread_local char g_err[512] = "";
uint64_t g_timeout_ns = 2000000000ull;

dsa_status fail(dsa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

dsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DSA_CHECK(cond, st, ...) \
  do {                           \
    if (!(cond)) return fail(st, __VA_ARGS__); \
  } while (0)

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

constexpr size_t kHeader = 256;
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D K-major operand [rows, cols] of 1- or 2-byte elements, 128-byte
// swizzled boxes of (128 bytes) x box_rows.  Columns beyond `cols` inside a
// box are zero-filled by TMA.
dsa_status make_tmap(CUtensorMap* m, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                     uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  const cuuint32_t box[2] = {(cuuint32_t)(128 / elem_bytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
  return DSA_OK;
}

bool supported_hi(int HI) { return HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64; }

dsa_status check_indexer_dims(int HI, int dI, int dtype) {
  DSA_CHECK(dtype == DSA_BF16 || dtype == DSA_FP8_E4M3, DSA_ERR_INVALID_ARG, "dtype %d is not a dsa_dtype", dtype);
  DSA_CHECK(supported_hi(HI), DSA_ERR_UNSUPPORTED, "HI=%d: supported indexer head counts are 4, 8, 16, 32, 64", HI);
  const int mult = dtype == DSA_BF16 ? 8 : 16;
  DSA_CHECK(dI > 0 && dI <= 128 && dI % mult == 0, DSA_ERR_UNSUPPORTED,
            "dI=%d: must be a multiple of %d in [%d, 128]", dI, mult, mult);
  return DSA_OK;
}

dsa::DeviceStatus* status_of(void* ws) { return reinterpret_cast<dsa::DeviceStatus*>(ws); }

dsa_status check_ws(void* ws, size_t have, size_t need) {
  DSA_CHECK(ws != nullptr && aligned(ws, 256), DSA_ERR_WORKSPACE, "workspace must be non-null and 256-byte aligned");
  DSA_CHECK(have >= need, DSA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
  return DSA_OK;
}

int ksteps_of(int dI, int dtype) { return (dI * (dtype == DSA_BF16 ? 2 : 1) + 31) / 32; }

}  // namespace

// Helpers shared with other translation units of the library (kernels.h).
namespace dsa {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }
int device_sm_count() { return sm_count(); }
uint64_t wait_timeout_ns() { return g_timeout_ns; }
int encode_tensor_map(CUtensorMap* m, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                      uint32_t box_rows) {
  return (int)make_tmap(m, base, elem_bytes, cols, rows, box_rows);
}
}  // namespace dsa

extern "C" {

const char* dsa_version(void) { return "dsa-b200 0.1 (sm_100a)"; }
const char* dsa_last_error(void) { return g_err; }
const char* dsa_status_string(int s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_DEVICE_CHECK: return "DSA_ERR_DEVICE_CHECK";
    default: return "unknown dsa_status";
  }
}

void dsa_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns; }
uint64_t dsa_get_wait_timeout_ns(void) { return g_timeout_ns; }

dsa_status dsa_workspace_init(void* ws, size_t bytes, void* stream) {
  if (dsa_status st = check_ws(ws, bytes, kHeader)) return st;
  cudaError_t e = cudaMemsetAsync(ws, 0, kHeader, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status header)");
  return DSA_OK;
}

dsa_status dsa_read_device_status(void* ws, void* stream, uint32_t* detail) {
  DSA_CHECK(ws != nullptr, DSA_ERR_WORKSPACE, "workspace is null");
  dsa::DeviceStatus h;
  cudaError_t e = cudaMemcpyAsync(&h, ws, 8, cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
  e = cudaMemsetAsync(ws, 0, 8, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status");
  if (detail) *detail = h.detail;
  if (h.code == 0) return DSA_OK;
  if (h.code == DSA_ERR_TIMEOUT) return fail(DSA_ERR_TIMEOUT, "device wait timed out (detail 0x%x)", h.detail);
  return fail((dsa_status)h.code, "device check failed (code %u, detail 0x%x)", h.code, h.detail);
}

size_t dsa_small_workspace(void) { return kHeader; }
size_t dsa_sparse_attn_workspace(void) { return kHeader; }

// ---------------------------------------------------------------- prefill
// Streamed candidates kept per token (4 warp sub-buffers of a quarter each);
// rows whose candidates outgrow them are finished by the second pass, which
// recomputes kRepairRows score rows at a time.
static constexpr int64_t kPrefillCandCap = 16384;
static constexpr int kScanChunkTiles = 8;   // key tiles per work item of the indexer scan
static constexpr int kRepairRows = 64;

static size_t history_cap(int kv_len) { return round_up((size_t)(kv_len > 0 ? kv_len : 1), 128); }

// candidates of the 8 tokens of a block, then one cut-off scratch per epilogue group
static size_t prefill_cand_bytes(size_t cap) {
  return (size_t)sm_count() * (dsa::prefill_block_tokens() + 4) * cap * sizeof(uint2);
}

// The second pass: overflow count (16 B), overflow list [B * nq], then
// kRepairRows score rows of kv_len fp32.
static size_t prefill_repair_bytes(int B, int nq, int kv_len) {
  return 256 + round_up((size_t)B * (size_t)(nq > 0 ? nq : 0) * 4, 256) +
         (size_t)kRepairRows * (size_t)(kv_len > 0 ? kv_len : 1) * 4;
}

size_t dsa_indexer_topk_prefill_workspace_full(int B, int nq, int kv_len, int HI, int dI, int k, int dtype) {
  (void)B; (void)nq; (void)HI; (void)dI; (void)k; (void)dtype;
  return kHeader + prefill_cand_bytes(history_cap(kv_len));
}

size_t dsa_indexer_topk_prefill_workspace(int B, int nq, int kv_len, int HI, int dI, int k, int dtype) {
  const size_t full = dsa_indexer_topk_prefill_workspace_full(B, nq, kv_len, HI, dI, k, dtype);
  if ((int64_t)history_cap(kv_len) <= kPrefillCandCap) return full;
  return std::min(full, kHeader + prefill_cand_bytes((size_t)kPrefillCandCap) + prefill_repair_bytes(B, nq, kv_len));
}

dsa_status dsa_indexer_topk_prefill(int B, int nq, int q_offset, int kv_len, int HI, int dI, int k, int dtype,
                                    const void* qI, const float* q_scale, const void* kI, const float* k_scale,
                                    const float* w, int32_t* idx_out, float* score_out, void* workspace,
                                    size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_indexer_dims(HI, dI, dtype)) return st;
  DSA_CHECK(B >= 1 && nq >= 0 && q_offset >= 0 && k >= 1, DSA_ERR_INVALID_ARG,
            "need B >= 1, nq >= 0, q_offset >= 0, k >= 1 (got %d, %d, %d, %d)", B, nq, q_offset, k);
  DSA_CHECK((int64_t)q_offset + nq <= kv_len, DSA_ERR_INVALID_ARG, "q_offset + nq (%d) exceeds kv_len (%d)",
            q_offset + nq, kv_len);
  DSA_CHECK((int64_t)B * nq * HI < INT32_MAX && (int64_t)B * kv_len < INT32_MAX, DSA_ERR_UNSUPPORTED,
            "tensor rows exceed 2^31");
  DSA_CHECK(qI && kI && w && idx_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(qI, 16) && aligned(kI, 16) && aligned(w, 4) && aligned(idx_out, 4), DSA_ERR_INVALID_ARG,
            "qI and kI must be 16-byte aligned");
  const bool fp8 = dtype == DSA_FP8_E4M3;
  DSA_CHECK(!fp8 || (q_scale && k_scale), DSA_ERR_INVALID_ARG, "FP8 needs q_scale and k_scale");
  const size_t need = dsa_indexer_topk_prefill_workspace(B, nq, kv_len, HI, dI, k, dtype);
  if (dsa_status st = check_ws(workspace, workspace_bytes, need)) return st;
  if (nq == 0) return DSA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = fp8 ? 1 : 2;
  const int QB = dsa::prefill_block_tokens();
  // capped candidate buffers unless the workspace holds the full-history ones
  const bool capped = workspace_bytes < dsa_indexer_topk_prefill_workspace_full(B, nq, kv_len, HI, dI, k, dtype);

  dsa::PrefillArgs a{};
  a.B = B;
  a.nq = nq;
  a.q_offset = q_offset;
  a.kv_len = kv_len;
  a.k = k;
  a.ksteps = ksteps_of(dI, dtype);
  a.nblk = (nq + QB - 1) / QB;
  a.first_blk = 0;
  if (score_out == nullptr) {
    // Leading blocks whose every row has t + 1 <= k select all of 0..t.
    while (a.first_blk < a.nblk &&
           (int64_t)q_offset + std::min(a.first_blk * QB + QB - 1, nq - 1) + 1 <= k)
      ++a.first_blk;
  }
  a.w = w;
  a.q_scale = fp8 ? q_scale : nullptr;
  a.k_scale = fp8 ? k_scale : nullptr;
  a.idx_out = idx_out;
  a.score_out = score_out;
  a.cand = reinterpret_cast<uint2*>(static_cast<char*>(workspace) + kHeader);
  a.cand_cap = capped ? kPrefillCandCap : (int64_t)history_cap(kv_len);
  a.bnd = a.cand + (int64_t)sm_count() * dsa::prefill_block_tokens() * a.cand_cap;
  char* repair = static_cast<char*>(workspace) + kHeader + prefill_cand_bytes((size_t)a.cand_cap);
  a.ovf_count = capped ? reinterpret_cast<uint32_t*>(repair) : nullptr;
  a.ovf_list = capped ? reinterpret_cast<int32_t*>(repair + 256) : nullptr;
  a.status = status_of(workspace);
  a.timeout_ns = g_timeout_ns;

  if (a.first_blk > 0) {
    cudaError_t e = dsa::launch_fill_trivial_rows(B, nq, q_offset, std::min(a.first_blk * QB, nq), k, idx_out, s);
    if (e != cudaSuccess) return cuda_fail(e, "fill_trivial_rows launch");
  }
  if (a.first_blk == a.nblk) return DSA_OK;

  CUtensorMap tq, tk;
  if (dsa_status st = make_tmap(&tq, qI, eb, (uint64_t)dI, (uint64_t)B * nq * HI, 4 * HI)) return st;
  if (dsa_status st = make_tmap(&tk, kI, eb, (uint64_t)dI, (uint64_t)B * kv_len, 128)) return st;
  const int kblocks = (dI * eb + 127) / 128;
  const int items = B * (a.nblk - a.first_blk);
  const int grid = std::min(sm_count(), items);
  if (capped) {
    cudaError_t e = cudaMemsetAsync(a.ovf_count, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail(e, "overflow count reset");
  }
  cudaError_t e = dsa::launch_indexer_topk_prefill(HI, fp8, kblocks, tq, tk, a, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_topk_prefill launch");
  if (!capped) return DSA_OK;

  // Second pass for the rows whose candidates outgrew their buffers: their
  // score rows are recomputed (indexer scan over the row list) and selected
  // with the row top-k, kRepairRows at a time.
  uint32_t n_ovf = 0;
  e = cudaMemcpyAsync(&n_ovf, a.ovf_count, sizeof(n_ovf), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "overflow count read-back");
  if (n_ovf > (uint32_t)B * (uint32_t)nq) return fail(DSA_ERR_DEVICE_CHECK, "overflow count %u above %d rows", n_ovf, B * nq);
  if (n_ovf == 0) return DSA_OK;
  float* rscores = reinterpret_cast<float*>(repair + 256 + round_up((size_t)B * nq * 4, 256));
  for (uint32_t r0 = 0; r0 < n_ovf; r0 += kRepairRows) {
    const int nr = (int)std::min<uint32_t>(kRepairRows, n_ovf - r0);
    dsa::ScanArgs sa{};
    sa.mode = 0;
    sa.rows = nr;
    sa.nq = nq;
    sa.q_offset = q_offset;
    sa.kv_len = kv_len;
    sa.ksteps = a.ksteps;
    sa.chunk_tiles = kScanChunkTiles;
    sa.max_chunks = std::max(1, ((kv_len + 127) / 128 + kScanChunkTiles - 1) / kScanChunkTiles);
    sa.balanced = 0;
    sa.w = w;
    sa.q_scale = a.q_scale;
    sa.k_scale = a.k_scale;
    sa.out = rscores;
    sa.row_list = a.ovf_list + r0;
    sa.status = a.status;
    sa.timeout_ns = g_timeout_ns;
    CUtensorMap tq1;
    const int box_rows = HI < 16 ? 16 : HI;
    if (dsa_status st = make_tmap(&tq1, qI, eb, (uint64_t)dI, (uint64_t)B * nq * HI, box_rows)) return st;
    e = dsa::launch_indexer_scan(HI, fp8, kblocks, tq1, tk, sa, std::min(sm_count(), nr * sa.max_chunks), s);
    if (e != cudaSuccess) return cuda_fail(e, "indexer_scan (second pass) launch");
    dsa::TopkRowsArgs t{};
    t.rows = nr;
    t.k = k;
    t.scores = rscores;
    t.row_stride = kv_len;
    t.ncols = kv_len;
    t.row_list = sa.row_list;
    t.nq = nq;
    t.q_offset = q_offset;
    t.idx_out = idx_out;
    t.val_out = score_out;
    t.status = a.status;
    e = dsa::launch_topk_rows(t, s);
    if (e != cudaSuccess) return cuda_fail(e, "topk_rows (second pass) launch");
  }
  return DSA_OK;
}

// ---------------------------------------------------------------- attention
static dsa_status check_attn(int H, int Dqk, int Dv, int k, const void* q, const void* lat, const int32_t* idx,
                             const void* out, const float* lse) {
  DSA_CHECK(H >= 1 && k >= 1, DSA_ERR_INVALID_ARG, "need H >= 1 and k >= 1");
  DSA_CHECK(k <= 2048, DSA_ERR_UNSUPPORTED, "k=%d: sparse attention supports k <= 2048", k);
  DSA_CHECK(Dqk % 16 == 0 && Dqk >= 16 && Dqk <= 576, DSA_ERR_UNSUPPORTED,
            "Dqk=%d: must be a multiple of 16 in [16, 576]", Dqk);
  DSA_CHECK(Dv % 64 == 0 && Dv >= 64 && Dv <= 512 && Dv <= Dqk, DSA_ERR_UNSUPPORTED,
            "Dv=%d: must be a multiple of 64 in [64, 512] and <= Dqk", Dv);
  DSA_CHECK(q && lat && idx && out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(q, 16) && aligned(lat, 16) && aligned(idx, 4) && aligned(out, 4) && aligned(lse, 4),
            DSA_ERR_INVALID_ARG, "q and latent must be 16-byte aligned");
  return DSA_OK;
}

static dsa_status run_attn(dsa::AttnArgs& a, const void* q, const void* latent, int64_t latent_rows,
                           cudaStream_t s) {
  a.nh = 16;
  a.cb = (a.Dqk + 63) / 64;
  a.ksteps = a.Dqk / 16;
  a.dv_tiles = a.Dv / 64;
  a.timeout_ns = g_timeout_ns;
  DSA_CHECK((int64_t)a.rows * a.H < INT32_MAX && latent_rows < INT32_MAX, DSA_ERR_UNSUPPORTED,
            "tensor rows exceed 2^31");
  (void)q;
  (void)latent;
  const int64_t items = (int64_t)a.rows * ((a.H + a.nh - 1) / a.nh);
  const int grid = (int)std::min<int64_t>(sm_count(), items);
  cudaError_t e = dsa::launch_sparse_attn(a, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "sparse_attn launch");
  return DSA_OK;
}

dsa_status dsa_sparse_attn_prefill(int B, int nq, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                                   const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_attn(H, Dqk, Dv, k, q, latent, idx, out, lse)) return st;
  DSA_CHECK(B >= 1 && nq >= 0 && kv_len >= 1, DSA_ERR_INVALID_ARG, "need B >= 1, nq >= 0, kv_len >= 1");
  DSA_CHECK(std::isfinite(scale), DSA_ERR_INVALID_ARG, "scale must be finite");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  if (nq == 0) return DSA_OK;
  dsa::AttnArgs a{};
  a.rows = B * nq;
  a.H = H;
  a.Dqk = Dqk;
  a.Dv = Dv;
  a.k = k;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q = static_cast<const uint16_t*>(q);
  a.latent = static_cast<const uint16_t*>(latent);
  a.idx = idx;
  a.mode = 0;
  a.nq = nq;
  a.kv_len = kv_len;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.status = status_of(workspace);
  return run_attn(a, q, latent, (int64_t)B * kv_len, (cudaStream_t)stream);
}

dsa_status dsa_sparse_attn_decode(int B, int H, int Dqk, int Dv, int k, float scale, const void* q,
                                  const void* latent_cache, const int64_t* cu_seqlens, int64_t total_len,
                                  const int32_t* idx, void* out, float* lse, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_attn(H, Dqk, Dv, k, q, latent_cache, idx, out, lse)) return st;
  DSA_CHECK(B >= 0 && cu_seqlens && total_len >= 1, DSA_ERR_INVALID_ARG, "need B >= 0, cu_seqlens, total_len >= 1");
  DSA_CHECK(std::isfinite(scale), DSA_ERR_INVALID_ARG, "scale must be finite");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  if (B == 0) return DSA_OK;
  dsa::AttnArgs a{};
  a.rows = B;
  a.H = H;
  a.Dqk = Dqk;
  a.Dv = Dv;
  a.k = k;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q = static_cast<const uint16_t*>(q);
  a.latent = static_cast<const uint16_t*>(latent_cache);
  a.idx = idx;
  a.mode = 1;
  a.cu_seqlens = cu_seqlens;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.status = status_of(workspace);
  if (H == 128 && Dqk == 576 && Dv == 512 && aligned(out, 16)) {
    // the MQA shape of the decode step: all 128 heads on the tensor-core M
    DSA_CHECK(total_len < INT32_MAX && (int64_t)B * 2 <= INT32_MAX, DSA_ERR_UNSUPPORTED, "tensor rows exceed 2^31");
    a.timeout_ns = g_timeout_ns;
    cudaError_t e = dsa::launch_latent_attn_decode(a, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "latent_attn_decode launch");
    return DSA_OK;
  }
  return run_attn(a, q, latent_cache, total_len, (cudaStream_t)stream);
}

// ---------------------------------------------------------------- dense masked attention
size_t dsa_attn_dense_prefill_workspace(int B, int nq, int kv_len, int with_selection) {
  if (!with_selection || B <= 0 || nq <= 0 || kv_len <= 0) return kHeader;
  return kHeader + round_up((size_t)B * nq * (size_t)((kv_len + 63) / 64) * sizeof(uint64_t), 256);
}

dsa_status dsa_attn_dense_prefill(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                                  const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  DSA_CHECK(H == 16 && Dqk == 576 && Dv == 512, DSA_ERR_UNSUPPORTED,
            "dense attention supports H=16, Dqk=576, Dv=512 (got H=%d Dqk=%d Dv=%d)", H, Dqk, Dv);
  DSA_CHECK(B >= 1 && nq >= 0 && q_offset >= 0 && kv_len >= 1 && (int64_t)q_offset + nq <= kv_len,
            DSA_ERR_INVALID_ARG, "need B >= 1, nq >= 0, q_offset >= 0, q_offset + nq <= kv_len");
  DSA_CHECK(idx == nullptr || k >= 1, DSA_ERR_INVALID_ARG, "k must be >= 1 with an index tensor");
  DSA_CHECK(std::isfinite(scale), DSA_ERR_INVALID_ARG, "scale must be finite");
  DSA_CHECK((int64_t)B * kv_len < INT32_MAX && (int64_t)B * nq * H < INT32_MAX, DSA_ERR_UNSUPPORTED,
            "tensor rows exceed 2^31");
  DSA_CHECK(q && latent && out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(q, 16) && aligned(latent, 16) && aligned(out, 16) && aligned(idx, 4) && aligned(lse, 4),
            DSA_ERR_INVALID_ARG, "q, latent and out must be 16-byte aligned");
  const size_t need = dsa_attn_dense_prefill_workspace(B, nq, kv_len, idx != nullptr);
  if (dsa_status st = check_ws(workspace, workspace_bytes, need)) return st;
  if (nq == 0) return DSA_OK;
  dsa::DenseAttnArgs a{};
  a.B = B;
  a.nq = nq;
  a.q_offset = q_offset;
  a.kv_len = kv_len;
  a.k = idx ? k : 0;
  a.nblk = (nq + 7) / 8;
  a.kv_tiles = (kv_len + 63) / 64;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.q = static_cast<const uint16_t*>(q);
  // rows with t + 1 <= k select their whole history: a chunk made only of
  // such rows needs no selection bits
  const bool need_bits = idx != nullptr && (int64_t)q_offset + nq > k;
  a.sel_bits = need_bits ? reinterpret_cast<const uint64_t*>(static_cast<char*>(workspace) + kHeader) : nullptr;
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.status = status_of(workspace);
  a.timeout_ns = g_timeout_ns;
  DSA_CHECK((int64_t)B * a.nblk * 2 < INT32_MAX, DSA_ERR_UNSUPPORTED, "too many token blocks");
  CUtensorMap tm;
  if (dsa_status st = make_tmap(&tm, latent, 2, 576, (uint64_t)B * kv_len, 64)) return st;
  cudaError_t e = dsa::launch_latent_attn_dense(tm, a, idx, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "latent_attn_dense launch");
  return DSA_OK;
}

// Length dispatch of the prefill attention (§2: short prefill runs DSA as
// masked dense attention, long prefill gathers the selected rows).  Measured
// on one B200 with k = 2048, 16 heads, 576/512 latent rows, one sequence:
// the dense path takes 0.77 / 1.16 / 1.65 / 2.20 / 2.82 ms for histories of
// 4096 / 5120 / 6144 / 7168 / 8192 keys, the gathering path 1.04 / 1.36 /
// 1.69 / 2.02 / 2.34 ms.
static constexpr int kDenseMaxHistory = 6144;

int dsa_prefill_attention_path(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k) {
  (void)B;
  (void)kv_len;
  (void)k;
  const bool shape = H == 16 && Dqk == 576 && Dv == 512;
  return (shape && nq > 0 && (int64_t)q_offset + nq <= kDenseMaxHistory) ? DSA_PATH_DENSE_MASKED
                                                                         : DSA_PATH_GATHER;
}

size_t dsa_attn_prefill_workspace(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k) {
  if (dsa_prefill_attention_path(B, nq, q_offset, kv_len, H, Dqk, Dv, k) == DSA_PATH_DENSE_MASKED)
    return dsa_attn_dense_prefill_workspace(B, nq, kv_len, 1);
  return dsa_sparse_attn_workspace();
}

dsa_status dsa_attn_prefill(int B, int nq, int q_offset, int kv_len, int H, int Dqk, int Dv, int k, float scale,
                            const void* q, const void* latent, const int32_t* idx, void* out, float* lse,
                            void* workspace, size_t workspace_bytes, void* stream) {
  DSA_CHECK(idx != nullptr, DSA_ERR_INVALID_ARG, "idx is required");
  if (dsa_prefill_attention_path(B, nq, q_offset, kv_len, H, Dqk, Dv, k) == DSA_PATH_DENSE_MASKED)
    return dsa_attn_dense_prefill(B, nq, q_offset, kv_len, H, Dqk, Dv, k, scale, q, latent, idx, out, lse, workspace,
                                  workspace_bytes, stream);
  return dsa_sparse_attn_prefill(B, nq, kv_len, H, Dqk, Dv, k, scale, q, latent, idx, out, lse, workspace,
                                 workspace_bytes, stream);
}

dsa_status dsa_mass_coverage(int rows, int H, const float* lse_sparse, const float* lse_dense, float* m_out,
                             float* per_head_out, float* min_out, void* stream) {
  DSA_CHECK(rows >= 0 && H >= 1, DSA_ERR_INVALID_ARG, "need rows >= 0 and H >= 1");
  DSA_CHECK(lse_sparse && lse_dense, DSA_ERR_INVALID_ARG, "null tensor pointer");
  cudaError_t e = dsa::launch_mass_coverage(rows, H, lse_sparse, lse_dense, m_out, per_head_out, min_out,
                                            (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "mass_coverage launch");
  return DSA_OK;
}

// ---------------------------------------------------------------- decode indexer

size_t dsa_indexer_topk_decode_workspace(int B, int HI, int dI, int k, int dtype, int64_t total_len, int max_len) {
  (void)B; (void)HI; (void)dI; (void)k; (void)dtype; (void)max_len;
  return kHeader + round_up((size_t)(total_len > 0 ? total_len : 1) * sizeof(float), 256);
}

dsa_status dsa_indexer_topk_decode(int B, int HI, int dI, int k, int dtype, const void* qI, const float* q_scale,
                                   const float* w, const void* kI_cache, const float* k_scale,
                                   const int64_t* cu_seqlens, int64_t total_len, int max_len, int32_t* idx_out,
                                   float* score_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_indexer_dims(HI, dI, dtype)) return st;
  DSA_CHECK(B >= 0 && k >= 1 && total_len >= 0 && max_len >= 0, DSA_ERR_INVALID_ARG,
            "need B >= 0, k >= 1, total_len >= 0, max_len >= 0");
  DSA_CHECK(total_len < INT32_MAX && (int64_t)B * HI < INT32_MAX, DSA_ERR_UNSUPPORTED, "cache rows exceed 2^31");
  DSA_CHECK(qI && w && kI_cache && cu_seqlens && idx_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(qI, 16) && aligned(kI_cache, 16) && aligned(w, 16), DSA_ERR_INVALID_ARG,
            "qI, kI_cache and w must be 16-byte aligned");
  const bool fp8 = dtype == DSA_FP8_E4M3;
  DSA_CHECK(!fp8 || (q_scale && k_scale), DSA_ERR_INVALID_ARG, "FP8 needs q_scale and k_scale");
  const size_t need = dsa_indexer_topk_decode_workspace(B, HI, dI, k, dtype, total_len, max_len);
  if (dsa_status st = check_ws(workspace, workspace_bytes, need)) return st;
  if (B == 0) return DSA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  const int eb = fp8 ? 1 : 2;
  float* scores = reinterpret_cast<float*>(static_cast<char*>(workspace) + kHeader);

  dsa::ScanArgs a{};
  a.mode = 1;
  a.rows = B;
  a.cu_seqlens = cu_seqlens;
  a.ksteps = ksteps_of(dI, dtype);
  a.chunk_tiles = kScanChunkTiles;
  const int tiles = (max_len + 127) / 128;
  a.max_chunks = std::max(1, (tiles + kScanChunkTiles - 1) / kScanChunkTiles);
  a.balanced = B <= dsa::kScanMaxBalancedRows ? 1 : 0;
  a.w = w;
  a.q_scale = fp8 ? q_scale : nullptr;
  a.k_scale = fp8 ? k_scale : nullptr;
  a.out = scores;
  a.status = status_of(workspace);
  a.timeout_ns = g_timeout_ns;
  if (total_len > 0 && max_len > 0) {
    CUtensorMap tq, tk;
    const int box_rows = HI < 16 ? 16 : HI;
    if (dsa_status st = make_tmap(&tq, qI, eb, (uint64_t)dI, (uint64_t)B * HI, box_rows)) return st;
    if (dsa_status st = make_tmap(&tk, kI_cache, eb, (uint64_t)dI, (uint64_t)total_len, 128)) return st;
    const int kblocks = (dI * eb + 127) / 128;
    const int items = B * a.max_chunks;
    const int grid = std::min(sm_count(), items);
    cudaError_t e = dsa::launch_indexer_scan(HI, fp8, kblocks, tq, tk, a, grid, s);
    if (e != cudaSuccess) return cuda_fail(e, "indexer_scan (decode) launch");
  }
  dsa::TopkRowsArgs t{};
  t.rows = B;
  t.k = k;
  t.scores = scores;
  t.cu_seqlens = cu_seqlens;
  t.idx_out = idx_out;
  t.val_out = score_out;
  t.status = status_of(workspace);
  cudaError_t e = dsa::launch_topk_rows(t, s);
  if (e != cudaSuccess) return cuda_fail(e, "topk_rows (decode) launch");
  return DSA_OK;
}

// ---------------------------------------------------------------- debug entry points
dsa_status dsa_indexer_scores(int B, int nq, int q_offset, int kv_len, int HI, int dI, int dtype, const void* qI,
                              const float* q_scale, const void* kI, const float* k_scale, const float* w,
                              float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_indexer_dims(HI, dI, dtype)) return st;
  DSA_CHECK(B >= 1 && nq >= 0 && q_offset >= 0 && (int64_t)q_offset + nq <= kv_len, DSA_ERR_INVALID_ARG,
            "need B >= 1, nq >= 0, q_offset >= 0, q_offset + nq <= kv_len");
  DSA_CHECK((int64_t)B * nq * HI < INT32_MAX && (int64_t)B * kv_len < INT32_MAX, DSA_ERR_UNSUPPORTED,
            "tensor rows exceed 2^31");
  DSA_CHECK(qI && kI && w && scores, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(qI, 16) && aligned(kI, 16) && aligned(w, 16), DSA_ERR_INVALID_ARG,
            "qI, kI and w must be 16-byte aligned");
  const bool fp8 = dtype == DSA_FP8_E4M3;
  DSA_CHECK(!fp8 || (q_scale && k_scale), DSA_ERR_INVALID_ARG, "FP8 needs q_scale and k_scale");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  if (nq == 0) return DSA_OK;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = dsa::launch_fill_f32(scores, (int64_t)B * nq * kv_len, -INFINITY, s);
  if (e != cudaSuccess) return cuda_fail(e, "fill launch");
  const int eb = fp8 ? 1 : 2;
  dsa::ScanArgs a{};
  a.mode = 0;
  a.rows = B * nq;
  a.nq = nq;
  a.q_offset = q_offset;
  a.kv_len = kv_len;
  a.ksteps = ksteps_of(dI, dtype);
  a.chunk_tiles = kScanChunkTiles;
  const int tiles = (q_offset + nq + 127) / 128;
  a.max_chunks = std::max(1, (tiles + kScanChunkTiles - 1) / kScanChunkTiles);
  a.balanced = 0;   // dense prefill rows: every row has max_chunks item slots
  a.w = w;
  a.q_scale = fp8 ? q_scale : nullptr;
  a.k_scale = fp8 ? k_scale : nullptr;
  a.out = scores;
  a.status = status_of(workspace);
  a.timeout_ns = g_timeout_ns;
  CUtensorMap tq, tk;
  const int box_rows = HI < 16 ? 16 : HI;
  if (dsa_status st = make_tmap(&tq, qI, eb, (uint64_t)dI, (uint64_t)B * nq * HI, box_rows)) return st;
  if (dsa_status st = make_tmap(&tk, kI, eb, (uint64_t)dI, (uint64_t)B * kv_len, 128)) return st;
  const int kblocks = (dI * eb + 127) / 128;
  const int items = a.rows * a.max_chunks;
  const int grid = std::min(sm_count(), items);
  e = dsa::launch_indexer_scan(HI, fp8, kblocks, tq, tk, a, grid, s);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_scan launch");
  return DSA_OK;
}

dsa_status dsa_topk_rows(int rows, int ncols, int64_t row_stride, const float* scores, const int32_t* row_len, int k,
                         int32_t* idx_out, float* val_out, void* workspace, size_t workspace_bytes, void* stream) {
  DSA_CHECK(rows >= 0 && ncols >= 0 && k >= 1 && row_stride >= ncols, DSA_ERR_INVALID_ARG,
            "need rows >= 0, ncols >= 0, k >= 1, row_stride >= ncols");
  DSA_CHECK(scores && idx_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  dsa::TopkRowsArgs t{};
  t.rows = rows;
  t.k = k;
  t.scores = scores;
  t.row_stride = row_stride;
  t.row_len = row_len;
  t.ncols = ncols;
  t.idx_out = idx_out;
  t.val_out = val_out;
  t.status = status_of(workspace);
  cudaError_t e = dsa::launch_topk_rows(t, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "topk_rows launch");
  return DSA_OK;
}

dsa_status dsa_selftest_bounded_wait(uint64_t timeout_ns, void* workspace, size_t workspace_bytes, void* stream) {
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  DSA_CHECK(timeout_ns <= 10000000000ull, DSA_ERR_INVALID_ARG, "timeout above 10 s");
  cudaError_t e = dsa::launch_wait_selftest(status_of(workspace), timeout_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "wait selftest launch");
  return DSA_OK;
}

// ---------------------------------------------------------------- diagnostics
dsa_status dsa_selection_overlap(int rows, int k, int max_pos, const int32_t* idx_a, const int32_t* idx_b,
                                 int32_t* inter_out, int32_t* count_a_out, void* stream) {
  DSA_CHECK(rows >= 0 && k >= 1 && max_pos >= 1, DSA_ERR_INVALID_ARG, "need rows >= 0, k >= 1, max_pos >= 1");
  DSA_CHECK(max_pos <= (1 << 20), DSA_ERR_UNSUPPORTED, "max_pos above 2^20 (the row bitmap lives in shared memory)");
  DSA_CHECK(idx_a && idx_b && inter_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  if (rows == 0) return DSA_OK;
  const int grid = std::min(rows, 4 * sm_count());
  cudaError_t e = dsa::launch_selection_overlap(rows, k, max_pos, idx_a, idx_b, inter_out, count_a_out, grid,
                                                (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "selection_overlap launch");
  return DSA_OK;
}

// ---------------------------------------------------------------- training: indexer KL (eq. 8)
size_t dsa_indexer_kl_workspace(void) { return kHeader; }

dsa_status dsa_indexer_kl_sparse(int B, int nq, int kv_len, int HI, int dI, int k, const void* qI, const void* kI,
                                 const float* w, const int32_t* idx, const float* teacher, float grad_scale,
                                 float* kl_out, float* grad_logits_out, float* dq_out, float* dw_out, float* dk_out,
                                 void* workspace, size_t workspace_bytes, void* stream) {
  DSA_CHECK(B >= 1 && nq >= 0 && kv_len >= 1 && k >= 1, DSA_ERR_INVALID_ARG,
            "need B >= 1, nq >= 0, kv_len >= 1, k >= 1");
  DSA_CHECK(HI >= 1 && HI <= 64, DSA_ERR_UNSUPPORTED, "HI=%d: the KL kernel supports 1..64 indexer heads", HI);
  DSA_CHECK(dI == 32 || dI == 64 || dI == 128, DSA_ERR_UNSUPPORTED, "dI=%d: supported are 32, 64, 128", dI);
  DSA_CHECK(k <= dsa::kMaxKLTopk, DSA_ERR_UNSUPPORTED, "k=%d above %d (the row's scores live in shared memory)", k,
            dsa::kMaxKLTopk);
  DSA_CHECK((int64_t)B * nq <= INT32_MAX, DSA_ERR_UNSUPPORTED, "too many rows");
  DSA_CHECK(qI && kI && w && idx && teacher && kl_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(qI, 16) && aligned(kI, 16), DSA_ERR_INVALID_ARG, "qI and kI must be 16-byte aligned");
  DSA_CHECK((!dq_out || aligned(dq_out, 8)) && (!dk_out || aligned(dk_out, 16)), DSA_ERR_INVALID_ARG,
            "dq must be 8-byte and dk 16-byte aligned");
  DSA_CHECK(std::isfinite(grad_scale), DSA_ERR_INVALID_ARG, "grad_scale must be finite");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  if (nq == 0) return DSA_OK;
  dsa::KLArgs a{};
  a.rows = B * nq;
  a.nq = nq;
  a.kv_len = kv_len;
  a.HI = HI;
  a.k = k;
  a.grad_scale = grad_scale;
  a.q = static_cast<const uint16_t*>(qI);
  a.kI = static_cast<const uint16_t*>(kI);
  a.w = w;
  a.idx = idx;
  a.teacher = teacher;
  a.kl = kl_out;
  a.grad_logits = grad_logits_out;
  a.dq = dq_out;
  a.dw = dw_out;
  a.dk = dk_out;
  a.status = status_of(workspace);
  cudaError_t e = dsa::launch_indexer_kl(dI, a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "indexer_kl launch");
  return DSA_OK;
}

dsa_status dsa_attn_teacher_prefill(int B, int nq, int kv_len, int H, int Dqk, int k, float scale, const void* q,
                                    const void* latent, const int32_t* idx, const float* lse, float* p_out,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  DSA_CHECK(B >= 1 && nq >= 0 && kv_len >= 1 && k >= 1 && H >= 1, DSA_ERR_INVALID_ARG,
            "need B >= 1, nq >= 0, kv_len >= 1, k >= 1, H >= 1");
  DSA_CHECK(Dqk >= 16 && Dqk <= 576 && Dqk % 16 == 0, DSA_ERR_UNSUPPORTED,
            "Dqk=%d: supported are multiples of 16 up to 576", Dqk);
  DSA_CHECK(k <= dsa::kMaxTeacherTopk, DSA_ERR_UNSUPPORTED, "k=%d above %d", k, dsa::kMaxTeacherTopk);
  DSA_CHECK((int64_t)B * nq <= INT32_MAX, DSA_ERR_UNSUPPORTED, "too many rows");
  DSA_CHECK(q && latent && idx && lse && p_out, DSA_ERR_INVALID_ARG, "null tensor pointer");
  DSA_CHECK(aligned(q, 16) && aligned(latent, 16), DSA_ERR_INVALID_ARG, "q and latent must be 16-byte aligned");
  DSA_CHECK(std::isfinite(scale), DSA_ERR_INVALID_ARG, "scale must be finite");
  if (dsa_status st = check_ws(workspace, workspace_bytes, kHeader)) return st;
  if (nq == 0) return DSA_OK;
  dsa::TeacherArgs a{};
  a.rows = B * nq;
  a.nq = nq;
  a.kv_len = kv_len;
  a.H = H;
  a.Dqk = Dqk;
  a.k = k;
  a.scale = scale;
  a.q = static_cast<const uint16_t*>(q);
  a.latent = static_cast<const uint16_t*>(latent);
  a.idx = idx;
  a.lse = lse;
  a.p_out = p_out;
  a.status = status_of(workspace);
  a.timeout_ns = dsa::wait_timeout_ns();
  cudaError_t e = dsa::launch_attn_teacher(a, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "attn_teacher launch");
  return DSA_OK;
}

}  // extern "C"
