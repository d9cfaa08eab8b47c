// topk.cu -- standalone top-k over materialised score rows with per-row
// lengths (eq. (2) of page "2.2.1 · DSA 与索引器"; the page's §2 lists a
// separate radix top-k that handles variable-length rows via seq_lens), plus
// small helper kernels.
//
// One CTA (1024 threads) per row.  A long row (at least 8192 entries and 4k)
// first takes a 1/16 sample of itself and finds a cut-off key tau a little
// below the sample's estimate of the k-th largest key; one 16-byte-load pass
// over the row then gathers every entry with key >= tau into shared memory,
// where the exact radix select of select.cuh runs.  When at least k entries
// reach tau, every selected entry and every tie at the k-th key is among the
// gathered ones, so the result is the row's exact top-k; when fewer than k
// reach tau, or more than the shared buffer holds, the row falls back to the
// two-pass path.  The two-pass path (also used for short rows): a histogram of
// the row's scores over the coarse score bins finds the cut-off bin; one pass
// then writes every entry above that bin and gathers the cut-off bin's
// entries into shared memory, where the exact radix refinement on
// (key, position) runs.  (A cut-off bin too large for shared memory is refined
// over the row instead.)  Used by the decode step (64 rows of 4096..65536
// scores) and by the debug path.
#include "kernels.h"
#include "select.cuh"

namespace dsa {

namespace {
constexpr int kRowThreads = 1024;
constexpr int kRowBins = 2048;        // refinement digit bins
constexpr int kBndCap = 16384;        // cut-off bin entries kept in shared memory (two-pass path)
constexpr int kCandCap = 16384;       // gathered candidates (prefilter path)
constexpr int kSampleMax = 8192;      // sampled entries
constexpr int kSampleLong = 1024;     // sampled entries of a row of at least 16384
constexpr int kGatherBatch = 4;       // 16-byte loads in flight per thread in the gather pass
constexpr int kPrefilterMinLen = 8192;
constexpr size_t kTopkDynSmem = (size_t)kCandCap * sizeof(uint2);
static_assert(kBndCap <= kCandCap && kSampleMax * sizeof(uint32_t) <= kTopkDynSmem, "aliased buffers");
}  // namespace

__global__ void __launch_bounds__(kRowThreads, 1) topk_rows_kernel(const TopkRowsArgs a) {
  __shared__ uint32_t hist[kRowBins];
  __shared__ SelectShared<kRowThreads> sh;
  __shared__ uint32_t s_maxkey;   // largest key of the row (prefilter path)
  extern __shared__ __align__(16) uint8_t topk_dyn[];
  uint2* cand = reinterpret_cast<uint2*>(topk_dyn);     // prefilter candidates
  uint32_t* samp = reinterpret_cast<uint32_t*>(topk_dyn);  // sample keys (before the gather)
  uint2* bnd = cand;                                    // two-pass cut-off bin entries
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
    if (a.row_list) len = a.q_offset + a.row_list[row] % a.nq + 1;
    if (len > a.ncols) {   // a row cannot be longer than the matrix
      if (threadIdx.x == 0) report_status(a.status, kStatusDeviceCheck, 0x70E1u);
      len = a.ncols;
    }
  }
  if (len < 0) len = 0;
  const int kk = len < a.k ? len : a.k;
  const int64_t out_row = a.row_list ? (int64_t)a.row_list[row] : (int64_t)row;
  int32_t* idx_row = a.idx_out + out_row * a.k;
  float* val_row = a.val_out ? a.val_out + out_row * a.k : nullptr;
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
  // ---- prefilter for long rows
  const int head = min(len, (int)((((16u - ((uint32_t)reinterpret_cast<uintptr_t>(src) & 15u)) & 15u)) >> 2));
  const int nb4 = (len - head) >> 2;                    // 16-byte aligned body, in float4
  const float4* body = reinterpret_cast<const float4*>(src + head);
  if (len >= kPrefilterMinLen && len >= 4 * kk) {
    // the row is pulled into L2 now, for the gather pass after the sample
    if (tid < 32) {
      constexpr int64_t kChunk = 65536;
      const int64_t bytes = (int64_t)nb4 * 16;
      for (int64_t o = (int64_t)tid * kChunk; o < bytes; o += 32 * kChunk)
        prefetch_l2_bulk(reinterpret_cast<const char*>(body) + o, (uint32_t)min(kChunk, bytes - o));
    }
    if (tid == 0) s_maxkey = 0u;
    // 1024 sampled entries for long rows (1/16 of shorter ones)
    const int ns4 = nb4 >= 16 * (kSampleLong / 4) ? kSampleLong / 4 : min(nb4 >> 4, kSampleMax / 4);
    const int st = nb4 / ns4;                            // >= 16
    const int s_n = 4 * ns4;
    for (int j = (int)tid; j < ns4; j += kRowThreads) {
      const float4 v = body[(int64_t)j * st];
      samp[4 * j + 0] = float_to_key(v.x);
      samp[4 * j + 1] = float_to_key(v.y);
      samp[4 * j + 2] = float_to_key(v.z);
      samp[4 * j + 3] = float_to_key(v.w);
    }
    __syncthreads();
    // tau = the lower edge of the top-11-bit key bin holding the m-th largest
    // sampled key, m about 1.25 kk s/len plus a margin, so that more than kk
    // row entries reach it unless the sample is unrepresentative (one
    // histogram round: the exact select runs on the gathered entries)
    const int m = (int)((5LL * kk * s_n + 4LL * len - 1) / (4LL * len)) + 32;
    for (int i = (int)tid; i < kRowBins; i += kRowThreads) hist[i] = 0u;
    __syncthreads();
    for (int j = (int)tid; j < s_n; j += kRowThreads) atomicAdd(&hist[samp[j] >> 21], 1u);
    __syncthreads();
    if (!group_find<kRowThreads>(hist, kRowBins, (uint32_t)m, true, sh, tid, 0) && tid == 0)
      report_status(a.status, kStatusDeviceCheck, 0x5e1ecau);
    const uint32_t tau = sh.found_bin << 21;
    if (tid == 0) sh.bnd_count = 0u;
    __syncthreads();   // sample reads done before the buffer is reused
    for (int j0 = 0; j0 < nb4; j0 += kRowThreads * kGatherBatch) {
      float4 v[kGatherBatch];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int j = j0 + u * kRowThreads + (int)tid;
        v[u] = j < nb4 ? body[j] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      uint32_t n = 0, kmax = 0;
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int j = j0 + u * kRowThreads + (int)tid;
        if (j < nb4) {
          const uint32_t k0 = float_to_key(v[u].x), k1 = float_to_key(v[u].y), k2 = float_to_key(v[u].z),
                         k3 = float_to_key(v[u].w);
          n += (k0 >= tau) + (k1 >= tau) + (k2 >= tau) + (k3 >= tau);
          kmax = max(kmax, max(max(k0, k1), max(k2, k3)));
        }
      }
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if (lane == 0) atomicMax(&s_maxkey, kmax);
      uint32_t incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= (uint32_t)o) incl += t;
      }
      uint32_t base = 0;
      if (lane == 31 && incl) base = atomicAdd(&sh.bnd_count, incl);
      base = __shfl_sync(0xffffffffu, base, 31) + incl - n;
      if (n) {
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u) {
          const int j = j0 + u * kRowThreads + (int)tid;
          const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t key = float_to_key(f[c]);
            if (j < nb4 && key >= tau) {
              if (base < (uint32_t)kCandCap) cand[base] = make_uint2(key, (uint32_t)(head + 4 * j + c));
              ++base;
            }
          }
        }
      }
    }
    if (tid < 32) {   // the unaligned head and tail (at most 3 entries each)
      const int tail0 = head + 4 * nb4;
      const int i = tid < 3 ? (int)tid : tail0 + (int)tid - 3;
      const bool valid = tid < 3 ? i < head : (tid < 6 && i < len);
      const uint32_t key = valid ? float_to_key(src[i]) : 0u;
      const bool take = valid && key >= tau;
      if (take) atomicMax(&s_maxkey, key);
      const uint32_t mk = __ballot_sync(0xffffffffu, take);
      uint32_t base = 0;
      if (lane == 0 && mk) base = atomicAdd(&sh.bnd_count, (uint32_t)__popc(mk));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (take) {
        const uint32_t slot = base + __popc(mk & ((1u << lane) - 1u));
        if (slot < (uint32_t)kCandCap) cand[slot] = make_uint2(key, (uint32_t)i);
      }
    }
    __syncthreads();
    const uint32_t c = sh.bnd_count, kmax = s_maxkey;
    __syncthreads();   // every thread has read the count before the select reuses sh
    if (c >= (uint32_t)kk && c <= (uint32_t)kCandCap) {
      auto get_c = [cand](int i, uint32_t& key, uint32_t& pos) {
        const uint2 e = cand[i];
        key = e.x;
        pos = e.y;
      };
      // every candidate key lies in [tau, kmax]
      const SelectResult r = group_refine<kRowThreads, kRowBins>(get_c, (int)c, tau, max(tau, kmax), (uint32_t)kk,
                                                                 (uint32_t)(len - 1), hist, sh, tid, 0, a.status);
      group_emit<kRowThreads>(get_c, (int)c, r, kk, a.k, idx_row, val_row, sh, tid, 0, a.status);
      return;
    }
    // the sample misjudged the row: take the two-pass path below
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
  // one entry per thread (all lanes of the warp take part): above the
  // cut-off bin -> written to the output now; inside it -> shared memory
  auto classify = [&](bool valid, uint32_t key, int i) {
    const bool above = valid && key > bhi, on = valid && key >= blo && key <= bhi;
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
        if (val_row) val_row[slot] = key_to_float(key);
      }
    }
    if (on) {
      const uint32_t slot = base_o + __popc(mo & below);
      if (slot < (uint32_t)kBndCap) bnd[slot] = make_uint2(key, (uint32_t)i);
    }
  };
  // the 16-byte aligned body with 16-byte loads, then the head and tail;
  // per thread and batch of 16 entries: both counts, one warp scan of the
  // packed pair and one pair of shared atomics per warp
  for (int j0 = 0; j0 < nb4; j0 += kRowThreads * kGatherBatch) {
    float4 v[kGatherBatch];
#pragma unroll
    for (int u = 0; u < kGatherBatch; ++u) {
      const int j = j0 + u * kRowThreads + (int)tid;
      v[u] = j < nb4 ? body[j] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    uint32_t na = 0, no = 0;
#pragma unroll
    for (int u = 0; u < kGatherBatch; ++u) {
      const int j = j0 + u * kRowThreads + (int)tid;
      if (j < nb4) {
        const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t key = float_to_key(f[c]);
          na += key > bhi;
          no += key >= blo && key <= bhi;
        }
      }
    }
    const uint32_t packed = na | (no << 16);   // each count <= 16 per thread, <= 512 per warp
    uint32_t incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= (uint32_t)o) incl += t;
    }
    uint32_t base_a = 0, base_o = 0;
    if (lane == 31) {
      if (incl & 0xFFFFu) base_a = atomicAdd(&sh.out_count, incl & 0xFFFFu);
      if (incl >> 16) base_o = atomicAdd(&sh.bnd_count, incl >> 16);
    }
    const uint32_t excl = incl - packed;
    uint32_t pa = __shfl_sync(0xffffffffu, base_a, 31) + (excl & 0xFFFFu);
    uint32_t po = __shfl_sync(0xffffffffu, base_o, 31) + (excl >> 16);
    if (na | no) {
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int j = j0 + u * kRowThreads + (int)tid;
        const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t key = float_to_key(f[c]);
          if (j < nb4 && key > bhi) {
            if (pa < (uint32_t)kk) {
              idx_row[pa] = head + 4 * j + c;
              if (val_row) val_row[pa] = key_to_float(key);
            }
            ++pa;
          } else if (j < nb4 && key >= blo) {
            if (po < (uint32_t)kBndCap) bnd[po] = make_uint2(key, (uint32_t)(head + 4 * j + c));
            ++po;
          }
        }
      }
    }
  }
  if (tid < 32) {
    const int tail0 = head + 4 * nb4;
    const int i = tid < 3 ? (int)tid : tail0 + (int)tid - 3;
    const bool valid = tid < 3 ? i < head : (tid < 6 && i < len);
    classify(valid, valid ? float_to_key(src[i]) : 0u, i);
  }
  __syncthreads();
  const uint32_t nb = sh.bnd_count;
  SelectResult r;
  r.lo = blo;
  r.hi = bhi;
  r.key_all_in = 1;
  r.pos_hi = 0;
  if (nb <= (uint32_t)kBndCap) {
    auto get_bnd = [bnd](int i, uint32_t& key, uint32_t& pos) {
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
  cudaError_t e = setup_once_per_device([] {
    return cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTopkDynSmem);
  });
  if (e != cudaSuccess) return e;
  topk_rows_kernel<<<a.rows, kRowThreads, kTopkDynSmem, stream>>>(a);
  return cudaGetLastError();
}

// Rows whose history fits in the budget (t + 1 <= k) select every position:
// S_t = {0, ..., t}, the rest of the row is -1 (eq. (2), short history).
// Rows whose history holds at most k positions (t + 1 <= k) select all of
// it (eq. (2)): slot j holds j for j <= t, then -1.  One block per row (grid
// stride), 16-byte stores when the rows are 16-byte aligned.
__global__ void fill_trivial_rows_kernel(int nq, int q_offset, int rows_per_seq, int64_t nrows, int k, int32_t* idx,
                                         int vec4) {
  for (int64_t r = blockIdx.x; r < nrows; r += gridDim.x) {
    const int b = (int)(r / rows_per_seq), i = (int)(r - (int64_t)b * rows_per_seq);
    const int t = q_offset + i;
    int32_t* row = idx + ((int64_t)b * nq + i) * k;
    if (vec4) {
      for (int q = threadIdx.x; q < k / 4; q += blockDim.x) {
        const int s = 4 * q;
        reinterpret_cast<int4*>(row)[q] =
            make_int4(s <= t ? s : -1, s + 1 <= t ? s + 1 : -1, s + 2 <= t ? s + 2 : -1, s + 3 <= t ? s + 3 : -1);
      }
    } else {
      for (int s = threadIdx.x; s < k; s += blockDim.x) row[s] = s <= t ? s : -1;
    }
  }
}

cudaError_t launch_fill_trivial_rows(int B, int nq, int q_offset, int rows_per_seq, int k, int32_t* idx,
                                     cudaStream_t stream) {
  if (rows_per_seq <= 0 || B <= 0) return cudaSuccess;
  const int64_t nrows = (int64_t)B * rows_per_seq;
  const int vec4 = (k % 4 == 0 && (reinterpret_cast<uintptr_t>(idx) & 15u) == 0) ? 1 : 0;
  const int grid = (int)(nrows < 148 * 8 ? nrows : 148 * 8);
  fill_trivial_rows_kernel<<<grid, 256, 0, stream>>>(nq, q_offset, rows_per_seq, nrows, k, idx, vec4);
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
