// noalloc.cu -- the decode step's indexer + top-k for callers that cannot
// allocate device memory.
//
// dsa_indexer_topk_decode needs a caller-provided workspace to hold the
// step's scores.  Some callers have no way to provide one: code that runs
// where cudaMalloc is not available or not allowed (a host runtime that owns
// every device allocation and hands a component only its input and output
// buffers, a plug-in called from a context whose allocator it cannot reach).
// For them this file adds one entry point whose scratch is a buffer built
// into the library: a file-scope __device__ array, which every GPU that loads
// the library holds until the process exits.  Nothing here allocates.
#include <cstdio>

#include "dsa.h"
#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int64_t kMaxKeys = int64_t(1) << 22;   // cached keys per call, all sequences together
constexpr size_t kHeaderBytes = 256;             // device status word, then the scores
constexpr size_t kScratchBytes = kHeaderBytes + size_t(kMaxKeys) * sizeof(float);   // 16 MiB + 256 B
constexpr int kChunkTiles = 8;

// In host code this name is only a stand-in for the device array: its device
// address comes from cudaGetSymbolAddress, looked up on every call (below).
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

dsa_status fail(dsa_status st, const char* msg) {
  dsa::set_last_error(msg);
  return st;
}

dsa_status launch_fail(cudaError_t e, const char* what) {
  char msg[256];
  snprintf(msg, sizeof(msg), "dsa_indexer_topk_decode_noalloc: %s: %s", what, cudaGetErrorString(e));
  return fail(DSA_ERR_CUDA, msg);
}

// Device address of the built-in scratch on the current device.  It is looked
// up on every call rather than cached: after a context teardown
// (cudaDeviceReset) the module is loaded again and the array may sit at
// another address, so a cached pointer would go stale.  The lookup is a host
// call; the first one on a device also loads this library's module there.
dsa_status scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) {
    char msg[256];
    snprintf(msg, sizeof(msg), "dsa_indexer_topk_decode_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    return fail(DSA_ERR_CUDA, msg);
  }
  *out = p;
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_indexer_topk_decode_noalloc(int B, int HI, int dI, int k, int dtype, const void* qI,
                                                      const float* q_scale, const float* w, const void* kI_cache,
                                                      const float* k_scale, const int64_t* cu_seqlens,
                                                      int64_t total_len, int max_len, int32_t* idx_out,
                                                      float* score_out, uint32_t* status_out, void* stream) {
  if (dtype != DSA_BF16 && dtype != DSA_FP8_E4M3) return fail(DSA_ERR_INVALID_ARG, "dtype is not a dsa_dtype");
  if (!(HI == 4 || HI == 8 || HI == 16 || HI == 32 || HI == 64))
    return fail(DSA_ERR_UNSUPPORTED, "HI: supported indexer head counts are 4, 8, 16, 32, 64");
  const int mult = dtype == DSA_BF16 ? 8 : 16;
  if (dI <= 0 || dI > 128 || dI % mult != 0) return fail(DSA_ERR_UNSUPPORTED, "dI: must be a multiple of 8 (bf16) or 16 (FP8), <= 128");
  if (B < 0 || k < 1 || total_len < 0 || max_len < 0)
    return fail(DSA_ERR_INVALID_ARG, "need B >= 0, k >= 1, total_len >= 0, max_len >= 0");
  if ((int64_t)B * HI >= INT32_MAX) return fail(DSA_ERR_UNSUPPORTED, "B * HI exceeds 2^31 rows");
  if (total_len > kMaxKeys) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "dsa_indexer_topk_decode_noalloc: total_len %lld exceeds the built-in scratch limit of %lld keys; "
             "use dsa_indexer_topk_decode with a workspace",
             (long long)total_len, (long long)kMaxKeys);
    return fail(DSA_ERR_UNSUPPORTED, msg);
  }
  if (!qI || !w || !kI_cache || !cu_seqlens || !idx_out) return fail(DSA_ERR_INVALID_ARG, "null tensor pointer");
  if ((reinterpret_cast<uintptr_t>(qI) | reinterpret_cast<uintptr_t>(kI_cache)) & 15u)
    return fail(DSA_ERR_INVALID_ARG, "qI and kI_cache must be 16-byte aligned");
  const bool fp8 = dtype == DSA_FP8_E4M3;
  if (fp8 && (!q_scale || !k_scale)) return fail(DSA_ERR_INVALID_ARG, "FP8 needs q_scale and k_scale");
  if (B == 0) return DSA_OK;

  void* scratch = nullptr;
  if (dsa_status st = scratch_address(&scratch)) return st;
  cudaStream_t s = (cudaStream_t)stream;
  dsa::DeviceStatus* status = static_cast<dsa::DeviceStatus*>(scratch);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(scratch) + kHeaderBytes);
  // The status word starts at zero on every call; the scores need no clearing
  // (the scan writes every cached position before the select reads it).
  cudaError_t e = cudaMemsetAsync(scratch, 0, kHeaderBytes, s);
  if (e != cudaSuccess) return launch_fail(e, "cudaMemsetAsync(status word)");

  const int eb = fp8 ? 1 : 2;
  dsa::ScanArgs a{};
  a.mode = 1;
  a.rows = B;
  a.cu_seqlens = cu_seqlens;
  a.ksteps = (dI * eb + 31) / 32;
  a.chunk_tiles = kChunkTiles;
  const int tiles = (max_len + 127) / 128;
  a.max_chunks = (tiles + kChunkTiles - 1) / kChunkTiles > 0 ? (tiles + kChunkTiles - 1) / kChunkTiles : 1;
  a.balanced = B <= dsa::kScanMaxBalancedRows ? 1 : 0;
  a.w = w;
  a.q_scale = fp8 ? q_scale : nullptr;
  a.k_scale = fp8 ? k_scale : nullptr;
  a.out = scores;
  a.status = status;
  a.timeout_ns = dsa::wait_timeout_ns();
  if (total_len > 0 && max_len > 0) {
    CUtensorMap tq, tk;
    const int box_rows = HI < 16 ? 16 : HI;
    if (int st = dsa::encode_tensor_map(&tq, qI, eb, (uint64_t)dI, (uint64_t)B * HI, box_rows)) return (dsa_status)st;
    if (int st = dsa::encode_tensor_map(&tk, kI_cache, eb, (uint64_t)dI, (uint64_t)total_len, 128))
      return (dsa_status)st;
    const int items = B * a.max_chunks;
    const int grid = dsa::device_sm_count() < items ? dsa::device_sm_count() : items;
    e = dsa::launch_indexer_scan(HI, fp8, (dI * eb + 127) / 128, tq, tk, a, grid, s);
    if (e != cudaSuccess) return launch_fail(e, "indexer_scan");
  }
  dsa::TopkRowsArgs t{};
  t.rows = B;
  t.k = k;
  t.scores = scores;
  t.cu_seqlens = cu_seqlens;
  t.idx_out = idx_out;
  t.val_out = score_out;
  t.status = status;
  e = dsa::launch_topk_rows(t, s);
  if (e != cudaSuccess) return launch_fail(e, "topk_rows");
  if (status_out) {
    e = cudaMemcpyAsync(status_out, scratch, 2 * sizeof(uint32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return launch_fail(e, "cudaMemcpyAsync(status_out)");
  }
  return DSA_OK;
}
