// topk.cu -- standalone top-k over materialised score rows with per-row
// lengths (eq. (2) of page "2.2.1 · DSA 与索引器"; the page's §2 lists a
// separate radix top-k that handles variable-length rows via seq_lens), plus
// small helper kernels.
//
// One CTA (1024 threads) per row, two passes over the row in the usual case:
// a histogram of the row's scores over the coarse score bins finds the
// cut-off bin; one pass then writes every entry above that bin and gathers
// the cut-off bin's entries into shared memory, where the exact radix
// refinement on (key, position) runs.  (A cut-off bin too large for shared
// memory is refined over the row instead.)  Used by the decode step (64 rows
// of 4096..65536 scores) and by the debug path.
#include "kernels.h"
#include "select.cuh"

namespace dsa {

namespace {
constexpr int kRowThreads = 1024;
constexpr int kRowBins = 2048;        // refinement digit bins
constexpr int kBndCap = 4096;         // cut-off bin entries kept in shared memory
}  // namespace

__global__ void __launch_bounds__(kRowThreads, 1) topk_rows_kernel(const TopkRowsArgs a) {
  __shared__ uint32_t hist[kRowBins];
  __shared__ uint2 bnd[kBndCap];
  __shared__ SelectShared<kRowThreads> sh;
  const int row = blockIdx.x;
  const uint32_t tid = threadIdx.x, lane = tid & 31u;
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
  if (kk == 0 || kk == len) {
    // nothing to choose: every entry (or none) is selected
    SelectResult r;
    r.lo = kk > 0 ? 0u : 0xFFFFFFFFu;
    r.hi = 0xFFFFFFFFu;
    r.key_all_in = 1;
    r.pos_hi = 0;
    group_emit<kRowThreads>(get, kk > 0 ? len : 0, r, kk, a.k, idx_row, val_row, sh, tid, 0, a.status);
    return;
  }
  // ---- pass 1: coarse score-bin histogram of the row
  for (int i = (int)tid; i < kScoreBins; i += kRowThreads) hist[i] = 0u;
  __syncthreads();
  for (int j0 = 0; j0 < len; j0 += kRowThreads * kBatch) {
    uint32_t key[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * kRowThreads + (int)tid;
      key[u] = i < len ? float_to_key(src[i]) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * kRowThreads + (int)tid;
      if (i < len) atomicAdd(&hist[score_bin(key[u])], 1u);
    }
  }
  __syncthreads();
  if (!group_find<kRowThreads>(hist, kScoreBins, (uint32_t)kk, true, sh, tid, 0) && tid == 0)
    report_status(a.status, kStatusDeviceCheck, 0x5e1ec5u);
  const uint32_t b0 = sh.found_bin;
  const uint32_t need = (uint32_t)kk - sh.found_beyond;
  uint32_t blo, bhi;
  bin_key_range(b0, blo, bhi);
  // ---- pass 2: entries above the cut-off bin are selected outright; the
  // cut-off bin's entries go to shared memory
  if (tid == 0) {
    sh.out_count = 0u;
    sh.bnd_count = 0u;
  }
  __syncthreads();
  for (int j0 = 0; j0 < len; j0 += kRowThreads * kBatch) {
    uint32_t key[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * kRowThreads + (int)tid;
      key[u] = i < len ? float_to_key(src[i]) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * kRowThreads + (int)tid;
      const bool above = i < len && key[u] > bhi, on = i < len && key[u] >= blo && key[u] <= bhi;
      const uint32_t ma = __ballot_sync(0xffffffffu, above), mo = __ballot_sync(0xffffffffu, on);
      uint32_t base_a = 0, base_o = 0;
      if (lane == 0) {
        if (ma) base_a = atomicAdd(&sh.out_count, (uint32_t)__popc(ma));
        if (mo) base_o = atomicAdd(&sh.bnd_count, (uint32_t)__popc(mo));
      }
      base_a = __shfl_sync(0xffffffffu, base_a, 0);
      base_o = __shfl_sync(0xffffffffu, base_o, 0);
      const uint32_t below = (1u << lane) - 1u;
      if (above) {
        const uint32_t slot = base_a + __popc(ma & below);
        if (slot < (uint32_t)kk) {
          idx_row[slot] = i;
          if (val_row) val_row[slot] = key_to_float(key[u]);
        }
      }
      if (on) {
        const uint32_t slot = base_o + __popc(mo & below);
        if (slot < (uint32_t)kBndCap) bnd[slot] = make_uint2(key[u], (uint32_t)i);
      }
    }
  }
  __syncthreads();
  const uint32_t nb = sh.bnd_count;
  SelectResult r;
  r.lo = blo;
  r.hi = bhi;
  r.key_all_in = 1;
  r.pos_hi = 0;
  if (nb <= (uint32_t)kBndCap) {
    auto get_bnd = [](int i, uint32_t& key, uint32_t& pos) {
      const uint2 e = bnd[i];
      key = e.x;
      pos = e.y;
    };
    if (need != nb)
      r = group_refine<kRowThreads, kRowBins>(get_bnd, (int)nb, blo, bhi, need, (uint32_t)(len - 1), hist, sh, tid,
                                              0, a.status);
    group_emit_append<kRowThreads>(get_bnd, (int)nb, r, blo, bhi, kk, idx_row, val_row, sh, tid, 0);
  } else {
    // the cut-off bin does not fit: refine and emit over the row, taking only
    // entries inside the bin (those above it are already written)
    if (need != nb)
      r = group_refine<kRowThreads, kRowBins>(get, len, blo, bhi, need, (uint32_t)(len - 1), hist, sh, tid, 0,
                                              a.status);
    group_emit_append<kRowThreads>(get, len, r, blo, bhi, kk, idx_row, val_row, sh, tid, 0);
  }
  group_emit_finish<kRowThreads>(kk, a.k, idx_row, val_row, sh, tid, 0, a.status);
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


// ---------------------------------------------------------------------------
// Selection diagnostic: per row, how many valid entries of selection A also
// appear in selection B (the numerator of the set recall R_k = |T ∩ S| / k,
// eq. (14) of the same page, §3.1), and how many valid entries A has.  One
// row at a time per CTA: A's positions go into a shared-memory bitmap of
// max_pos bits, then B's entries are tested against it.  Slot order and -1
// slots are irrelevant; entries outside [0, max_pos) are not counted.
// ---------------------------------------------------------------------------
namespace {
constexpr int kOverlapThreads = 256;
}

__global__ void __launch_bounds__(kOverlapThreads) selection_overlap_kernel(int rows, int k, int max_pos,
                                                                            const int32_t* idx_a,
                                                                            const int32_t* idx_b, int32_t* inter,
                                                                            int32_t* count_a) {
  extern __shared__ uint32_t bits[];
  __shared__ uint32_t s_inter, s_count;
  const int words = (max_pos + 31) / 32;
  for (int r = blockIdx.x; r < rows; r += gridDim.x) {
    for (int i = threadIdx.x; i < words; i += kOverlapThreads) bits[i] = 0u;
    if (threadIdx.x == 0) {
      s_inter = 0u;
      s_count = 0u;
    }
    __syncthreads();
    const int32_t* a = idx_a + (int64_t)r * k;
    const int32_t* b = idx_b + (int64_t)r * k;
    uint32_t na = 0;
    for (int j = threadIdx.x; j < k; j += kOverlapThreads) {
      const int p = a[j];
      if (p >= 0 && p < max_pos) {
        atomicOr(&bits[p >> 5], 1u << (p & 31));
        ++na;
      }
    }
    __syncthreads();
    uint32_t hit = 0;
    for (int j = threadIdx.x; j < k; j += kOverlapThreads) {
      const int p = b[j];
      if (p >= 0 && p < max_pos && (bits[p >> 5] >> (p & 31)) & 1u) ++hit;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      hit += __shfl_xor_sync(0xffffffffu, hit, o);
      na += __shfl_xor_sync(0xffffffffu, na, o);
    }
    if ((threadIdx.x & 31u) == 0u) {
      atomicAdd(&s_inter, hit);
      atomicAdd(&s_count, na);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      inter[r] = (int32_t)s_inter;
      if (count_a) count_a[r] = (int32_t)s_count;
    }
    __syncthreads();   // the bitmap is cleared for the next row
  }
}

cudaError_t launch_selection_overlap(int rows, int k, int max_pos, const int32_t* idx_a, const int32_t* idx_b,
                                     int32_t* inter, int32_t* count_a, int grid, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const size_t smem = (size_t)((max_pos + 31) / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(selection_overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  selection_overlap_kernel<<<grid, kOverlapThreads, smem, stream>>>(rows, k, max_pos, idx_a, idx_b, inter, count_a);
  return cudaGetLastError();
}

}  // namespace dsa
