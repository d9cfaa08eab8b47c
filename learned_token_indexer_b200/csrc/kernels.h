// kernels.h -- internal interface between the C ABI (api.cu) and the kernels.
#pragma once
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

namespace dsa {

struct DeviceStatus;

// A kernel's one-time host set-up (its shared-memory attribute, checks of its
// compiled register count): `setup` runs on the first launch from a call site
// on each device and its result is reused, keeping host calls off the launch
// path.  Thread-safe.
template <typename F>
cudaError_t setup_once_per_device(F&& setup) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static bool done[kMaxDev] = {};
  static cudaError_t result[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return setup();
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    result[dev] = setup();
    done[dev] = true;
  }
  return result[dev];
}

// Dense score rows (indexer_scan.cu).
constexpr int kScanMaxBalancedRows = 4096;
struct ScanArgs {
  int mode;                    // 0: prefill rows (b, i); 1: ragged decode rows
  int rows;                    // prefill B*nq; decode B
  int nq, q_offset, kv_len;    // prefill geometry
  const int64_t* cu_seqlens;   // decode: [rows + 1]
  int ksteps;                  // 32-byte MMA K steps holding data
  int chunk_tiles;             // key tiles per work item
  int max_chunks;              // work items per row (upper bound)
  int balanced;                // decode: number only non-empty chunks (rows <= kScanMaxBalancedRows)
  const float* w;              // [rows, HI]
  const float* q_scale;        // [rows] (FP8) or null
  const float* k_scale;        // [key rows] (FP8) or null
  float* out;                  // prefill [rows, kv_len]; decode [sum L]
  const int32_t* row_list;     // prefill only, or null: scan row r is query row row_list[r] (b * nq + i)
  DeviceStatus* status;
  uint64_t timeout_ns;
};

// Fused prefill indexer + top-k (indexer_topk_prefill.cu).
struct PrefillArgs {
  int B, nq, q_offset, kv_len, k;
  int ksteps;
  int nblk;                    // 8-token blocks per sequence
  int first_blk;               // blocks below this one need no scoring
  const float* w;              // [B, nq, HI]
  const float* q_scale;        // [B, nq] (FP8) or null
  const float* k_scale;        // [B, kv_len] (FP8) or null
  int32_t* idx_out;            // [B, nq, k]
  float* score_out;            // [B, nq, k] or null
  uint2* cand;                 // [grid * 8, cand_cap] candidate (key, pos) buffers
  int64_t cand_cap;
  uint2* bnd;                  // [grid * 4, cand_cap] cut-off bin entries of the row being selected
  // Candidate overflow (cand_cap below the history): a row whose accepted
  // entries outgrow its buffer is not selected here; its index b * nq + i is
  // appended to ovf_list (count in *ovf_count) for a second pass.
  uint32_t* ovf_count;
  int32_t* ovf_list;
  DeviceStatus* status;
  uint64_t timeout_ns;
};

// Row-wise top-k over materialised scores (topk.cu).
struct TopkRowsArgs {
  int rows, k;
  const float* scores;
  int64_t row_stride;          // used when cu_seqlens == null
  const int32_t* row_len;      // [rows] or null (then every row has ncols)
  int ncols;
  const int64_t* cu_seqlens;   // ragged rows: row r = scores[cu[r] .. cu[r+1])
  int32_t* idx_out;            // [rows, k]
  float* val_out;              // [rows, k] or null
  // Prefill rows given by list (row_stride layout): score row r belongs to
  // query row q = row_list[r] = b * nq + i, has length q_offset + i + 1 and
  // writes idx_out / val_out row q.
  const int32_t* row_list;
  int nq, q_offset;
  DeviceStatus* status;
};

// Sparse attention over selected latent rows (sparse_attn.cu).
struct AttnArgs {
  int rows;                    // query rows (prefill B*nq, decode B)
  int H, Dqk, Dv, k;
  int nh;                      // heads per CTA (MMA N)
  int cb;                      // 64-column blocks per latent row
  int ksteps;                  // 16-column K steps of the logits MMA (Dqk / 16)
  int dv_tiles;                // 64-wide value tiles (Dv / 64)
  uint64_t timeout_ns;
  float scale_log2;            // softmax scale * log2(e)
  float scale;
  const uint16_t* q;           // [rows, H, Dqk] bf16
  const uint16_t* latent;      // prefill [B, kv_len, Dqk]; decode [sum L, Dqk]
  const int32_t* idx;          // [rows, k]
  int mode;                    // 0 prefill (row r -> b = r / nq), 1 decode (cu_seqlens)
  int nq, kv_len;
  const int64_t* cu_seqlens;
  uint16_t* out;               // [rows, H, Dv] bf16
  float* lse;                  // [rows, H] or null
  DeviceStatus* status;
};

// Attention over dense causal key tiles, masked to the selection
// (latent_attn_dense.cu): 16 heads, latent rows 576 / value 512.
struct DenseAttnArgs {
  int B, nq, q_offset, kv_len, k;
  int nblk;                    // 8-token blocks per sequence
  int kv_tiles;                // 64-key tiles of a sequence's history (words per selection row)
  float scale_log2;
  const uint16_t* q;           // [B, nq, 16, 576] bf16
  const uint64_t* sel_bits;    // [B, nq, kv_tiles] or null (every causal key)
  uint16_t* out;               // [B, nq, 16, 512] bf16
  float* lse;                  // [B, nq, 16] or null
  DeviceStatus* status;
  uint64_t timeout_ns;
};

// Sparse-stage indexer KL on the selected set, forward and backward (indexer_kl.cu).
constexpr int kMaxKLTopk = 4096;
struct KLArgs {
  int rows, nq, kv_len, HI, k;
  float grad_scale;            // dL/dKL_t for every row
  const uint16_t* q;           // [rows, HI, dI] bf16
  const uint16_t* kI;          // [B, kv_len, dI] bf16
  const float* w;              // [rows, HI]
  const int32_t* idx;          // [rows, k]
  const float* teacher;        // [rows, k]
  float* kl;                   // [rows]
  float* grad_logits;          // [rows, k] or null
  float* dq;                   // [rows, HI, dI] or null
  float* dw;                   // [rows, HI] or null
  float* dk;                   // [B, kv_len, dI] (accumulated) or null
  DeviceStatus* status;
};

// Sparse-stage teacher: head-summed, L1-normalised attention probabilities on
// the selected set, from the forward's lse (attn_teacher.cu).
constexpr int kMaxTeacherTopk = 4096;
struct TeacherArgs {
  int rows, nq, kv_len, H, Dqk, k;
  float scale;
  const uint16_t* q;           // [rows, H, Dqk] bf16
  const uint16_t* latent;      // [B, kv_len, Dqk] bf16
  const int32_t* idx;          // [rows, k]
  const float* lse;            // [rows, H]
  float* p_out;                // [rows, k]
  DeviceStatus* status;
  uint64_t timeout_ns;
};

cudaError_t launch_indexer_scan(int HI, bool fp8, int kblocks, const CUtensorMap& tq, const CUtensorMap& tk,
                                const ScanArgs& a, int grid, cudaStream_t stream);
cudaError_t launch_indexer_topk_prefill(int HI, bool fp8, int kblocks, const CUtensorMap& tq,
                                        const CUtensorMap& tk, const PrefillArgs& a, int grid, cudaStream_t stream);
int prefill_block_tokens();
cudaError_t launch_topk_rows(const TopkRowsArgs& a, cudaStream_t stream);
cudaError_t launch_fill_trivial_rows(int B, int nq, int q_offset, int rows_per_seq, int k, int32_t* idx,
                                     cudaStream_t stream);
cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t stream);
cudaError_t launch_sparse_attn(const AttnArgs& a, int grid, cudaStream_t stream);
// Decode attention with 128 heads on the tcgen05 M (latent_attn_decode.cu):
// H = 128, Dqk = 576, Dv = 512; one 2-CTA cluster per sequence (a.rows).
cudaError_t launch_latent_attn_decode(const AttnArgs& a, cudaStream_t stream);
size_t latent_attn_decode_smem();
cudaError_t launch_latent_attn_dense(const CUtensorMap& tmap_lat, const DenseAttnArgs& a, const int32_t* idx,
                                     cudaStream_t stream);
size_t latent_attn_dense_smem();
cudaError_t launch_mass_coverage(int rows, int H, const float* lse_sparse, const float* lse_dense, float* m_out,
                                 float* per_head_out, float* min_out, cudaStream_t stream);
size_t indexer_kl_smem_bytes(int dI, int k);
size_t attn_teacher_smem_bytes(int k);
cudaError_t launch_attn_teacher(const TeacherArgs& a, cudaStream_t stream);
cudaError_t launch_indexer_kl(int dI, const KLArgs& a, cudaStream_t stream);
cudaError_t launch_wait_selftest(DeviceStatus* status, uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_selection_overlap(int rows, int k, int max_pos, const int32_t* idx_a, const int32_t* idx_b,
                                     int32_t* inter, int32_t* count_a, int grid, cudaStream_t stream);

// Host helpers implemented in api.cu.
void set_last_error(const char* msg);                 // message returned by dsa_last_error()
int device_sm_count();                                // SMs of the current device
uint64_t wait_timeout_ns();                           // bound of every device-side wait
int encode_tensor_map(CUtensorMap* m, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                      uint32_t box_rows);             // a dsa_status value

}  // namespace dsa
