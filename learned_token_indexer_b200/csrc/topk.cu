// topk.cu -- standalone top-k over materialised score rows with per-row
// lengths (eq. (2) of page "2.2.1 · DSA 与索引器"; the page's §2 lists a
// separate radix top-k that handles variable-length rows via seq_lens), plus
// small helper kernels.
//
// One CTA (1024 threads) per row; 2048-bin digit histograms in shared memory.
// The first refinement pass histograms the top 11 bits of every score's
// order-preserving key; later passes only count entries still inside the
// cut-off interval.  Used by the decode step (64 rows of 4096..65536 scores)
// and by the debug path.
#include "kernels.h"
#include "select.cuh"

namespace dsa {

namespace {
constexpr int kRowThreads = 1024;
constexpr int kRowBins = 2048;
}  // namespace

__global__ void __launch_bounds__(kRowThreads, 1) topk_rows_kernel(const TopkRowsArgs a) {
  __shared__ uint32_t hist[kRowBins];
  __shared__ SelectShared<kRowThreads> sh;
  const int row = blockIdx.x;
  const uint32_t tid = threadIdx.x;
  const float* src;
  int len;
  if (a.cu_seqlens) {
    const int64_t lo = a.cu_seqlens[row];
    src = a.scores + lo;
    len = (int)(a.cu_seqlens[row + 1] - lo);
  } else {
    src = a.scores + (int64_t)row * a.row_stride;
    len = a.row_len ? a.row_len[row] : a.ncols;
    if (len > a.ncols) {   // a row cannot be longer than the matrix
      if (threadIdx.x == 0) report_status(a.status, kStatusDeviceCheck, 0x70E1u);
      len = a.ncols;
    }
  }
  if (len < 0) len = 0;
  const int kk = len < a.k ? len : a.k;
  int32_t* idx_row = a.idx_out + (int64_t)row * a.k;
  float* val_row = a.val_out ? a.val_out + (int64_t)row * a.k : nullptr;
  auto get = [src](int i, uint32_t& key, uint32_t& pos) {
    key = float_to_key(src[i]);
    pos = (uint32_t)i;
  };
  SelectResult r;
  r.lo = 0xFFFFFFFFu;
  r.hi = 0xFFFFFFFFu;
  r.key_all_in = 1;
  r.pos_hi = 0;
  if (kk > 0 && kk < len)
    r = group_refine<kRowThreads, kRowBins>(get, len, 0u, 0xFFFFFFFFu, (uint32_t)kk, (uint32_t)(len - 1), hist, sh,
                                             tid, 0, a.status);
  else if (kk == len && len > 0)
    r.lo = 0u;   // every entry is selected
  group_emit<kRowThreads>(get, kk > 0 ? len : 0, r, kk, a.k, idx_row, val_row, sh, tid, 0, a.status);
}

cudaError_t launch_topk_rows(const TopkRowsArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  topk_rows_kernel<<<a.rows, kRowThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

// Rows whose history fits in the budget (t + 1 <= k) select every position:
// S_t = {0, ..., t}, the rest of the row is -1 (eq. (2), short history).
__global__ void fill_trivial_rows_kernel(int nq, int q_offset, int rows_per_seq, int k, int32_t* idx) {
  const int b = blockIdx.y;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)rows_per_seq * k;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / k), slot = (int)(e - (int64_t)i * k);
    const int t = q_offset + i;
    idx[((int64_t)b * nq + i) * k + slot] = slot <= t ? slot : -1;
  }
}

cudaError_t launch_fill_trivial_rows(int B, int nq, int q_offset, int rows_per_seq, int k, int32_t* idx,
                                     cudaStream_t stream) {
  if (rows_per_seq <= 0 || B <= 0) return cudaSuccess;
  const int64_t n = (int64_t)rows_per_seq * k;
  int gx = (int)((n + 255) / 256);
  if (gx > 4096) gx = 4096;
  fill_trivial_rows_kernel<<<dim3(gx, B), 256, 0, stream>>>(nq, q_offset, rows_per_seq, k, idx);
  return cudaGetLastError();
}

__global__ void fill_f32_kernel(float* p, int64_t n, float v) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}

cudaError_t launch_fill_f32(float* p, int64_t n, float v, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  int gx = (int)((n + 255) / 256);
  if (gx > 8192) gx = 8192;
  fill_f32_kernel<<<gx, 256, 0, stream>>>(p, n, v);
  return cudaGetLastError();
}

// Exercises the bounded-wait path: waits on an mbarrier that nothing will
// complete; the wait gives up after timeout_ns and records kStatusTimeout.
__global__ void wait_selftest_kernel(DeviceStatus* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtl ctl{&abort_flag, timeout_ns, status};
    (void)mbar_wait(&bar, 0u, ctl, 0x7e57u);
  }
  __syncthreads();
}

cudaError_t launch_wait_selftest(DeviceStatus* status, uint64_t timeout_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace dsa
