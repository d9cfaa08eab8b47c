// indexer_scan.cu -- Lightning Indexer scores written densely, one query token
// per row (page "2.2.1 · DSA 与索引器", §1.1 eq. (1); decode step of §2).
//
// Used by the decode step (one new token per sequence scans every cached
// indexer key; the scores of one step are small, so they are written out and
// a separate select kernel takes the top-k) and by the debug entry point that
// materialises the causal prefill score matrix for small n.
//
// Per CTA: warp 0 = TMA producer, warp 1 = tcgen05 MMA issuer (and TMEM
// owner), warps 2..5 = epilogue (TMEM -> ReLU * w -> head sum -> global).
// The MMA computes D[128 keys x N] with keys on TMEM lanes and the token's
// heads on columns; two accumulators alternate so the epilogue of one tile
// overlaps the MMA of the next.  Work items are (row, run of key tiles),
// spread over a persistent grid.
#include "indexer_common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

constexpr int kScanStages = 4;
constexpr int kScanThreads = 192;
constexpr int kEpiWarp0 = 2;

struct ScanRow {
  int64_t key_base;
  int len;
  float* out;
};

__device__ __forceinline__ ScanRow scan_row(const ScanArgs& a, int r) {
  ScanRow g;
  if (a.mode == 0) {
    const int b = r / a.nq, i = r - b * a.nq;
    g.key_base = (int64_t)b * a.kv_len;
    g.len = a.q_offset + i + 1;
    g.out = a.out + (int64_t)r * a.kv_len;
  } else {
    const int64_t lo = a.cu_seqlens[r];
    g.key_base = lo;
    g.len = (int)(a.cu_seqlens[r + 1] - lo);
    g.out = a.out + lo;
  }
  return g;
}

// Item i -> (row, first tile, number of tiles); ntiles == 0 means empty.
__device__ __forceinline__ void scan_item(const ScanArgs& a, int item, int& row, int& t0, int& nt,
                                          ScanRow& g) {
  row = item / a.max_chunks;
  const int c = item - row * a.max_chunks;
  g = scan_row(a, row);
  const int tiles = (g.len + kTileKeys - 1) / kTileKeys;
  t0 = c * a.chunk_tiles;
  nt = tiles - t0;
  nt = nt < 0 ? 0 : (nt > a.chunk_tiles ? a.chunk_tiles : nt);
}

}  // namespace

template <int HI, bool FP8, int KB>
__global__ void __launch_bounds__(kScanThreads, 1)
    indexer_scan_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const ScanArgs a) {
  constexpr int N = HI < 16 ? 16 : HI;
  constexpr int kQBytes = N * KB * kSwizzleBytes;
  constexpr int kKBytes = kTileKeys * KB * kSwizzleBytes;
  constexpr uint32_t kTmemCols = (2 * N <= 32) ? 32 : (2 * N <= 64 ? 64 : (2 * N <= 128 ? 128 : 256));
  constexpr uint32_t kIdesc = instr_desc(ElemTraits<FP8>::kFormat, kTileKeys, N);
  constexpr int kElemsPerBlock = ElemTraits<FP8>::kElemsPerBlock;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sQ = sK + kScanStages * kKBytes;
  float* sW = reinterpret_cast<float*>(sQ + 2 * kQBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + 2 * HI);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + kScanStages;
  uint64_t* q_full = bars + 2 * kScanStages;
  uint64_t* q_empty = q_full + 2;
  uint64_t* acc_full = q_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};
  const int total_items = a.rows * a.max_chunks;
  const int ksteps = a.ksteps;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0, qslot = 0;
      uint32_t kphase = 0, qphase = 0;
      uint32_t k_last_parity[kScanStages], q_last_parity[2];
      bool k_issued[kScanStages], q_issued[2];
      for (int s = 0; s < kScanStages; ++s) k_issued[s] = false;
      q_issued[0] = q_issued[1] = false;
      bool ok = true;
      for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        int row, t0, nt;
        ScanRow g;
        scan_item(a, item, row, t0, nt, g);
        if (nt == 0) continue;
        if (!(ok = mbar_wait(&q_empty[qslot], qphase ^ 1u, ctl, 0x101))) break;
        mbar_arrive_expect_tx(&q_full[qslot], kQBytes);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sQ + qslot * kQBytes + kb * N * kSwizzleBytes, &tmap_q, &q_full[qslot], kb * kElemsPerBlock,
                      row * HI);
        q_issued[qslot] = true;
        q_last_parity[qslot] = qphase;
        if (++qslot == 2) { qslot = 0; qphase ^= 1u; }
        for (int t = 0; t < nt; ++t) {
          if (!(ok = mbar_wait(&k_empty[stage], kphase ^ 1u, ctl, 0x102))) break;
          mbar_arrive_expect_tx(&k_full[stage], kKBytes);
          const int y = (int)(g.key_base + (int64_t)(t0 + t) * kTileKeys);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sK + stage * kKBytes + kb * kTileKeys * kSwizzleBytes, &tmap_k, &k_full[stage],
                        kb * kElemsPerBlock, y);
          k_issued[stage] = true;
          k_last_parity[stage] = kphase;
          if (++stage == kScanStages) { stage = 0; kphase ^= 1u; }
        }
      }
      if (!ok) {
        // Let every copy this thread started land before the CTA exits.
        const WaitCtl drain{abort_flag, a.timeout_ns, nullptr};
        for (int s = 0; s < kScanStages; ++s)
          if (k_issued[s]) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&k_full[s]), k_last_parity[s]) &&
                   globaltimer_ns() - t0 < drain.timeout_ns) {
            }
          }
        for (int s = 0; s < 2; ++s)
          if (q_issued[s]) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&q_full[s]), q_last_parity[s]) &&
                   globaltimer_ns() - t0 < drain.timeout_ns) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0, qslot = 0, acc = 0;
      uint32_t kphase = 0, qphase = 0, aphase = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        int row, t0, nt;
        ScanRow g;
        scan_item(a, item, row, t0, nt, g);
        if (nt == 0) continue;
        if (!(ok = mbar_wait(&q_full[qslot], qphase, ctl, 0x201))) break;
        tc_fence_after();
        const uint32_t qaddr = smem_u32(sQ + qslot * kQBytes);
        for (int t = 0; t < nt; ++t) {
          if (!(ok = mbar_wait(&k_full[stage], kphase, ctl, 0x202))) break;
          if (!(ok = mbar_wait(&acc_empty[acc], aphase ^ 1u, ctl, 0x203))) break;
          tc_fence_after();
          issue_tile_mma<FP8>(tmem_base + acc * N, smem_u32(sK + stage * kKBytes), qaddr, N, ksteps, kIdesc);
          tc_commit(&acc_full[acc]);
          tc_commit(&k_empty[stage]);
          if (++stage == kScanStages) { stage = 0; kphase ^= 1u; }
          if (++acc == 2) { acc = 0; aphase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&q_empty[qslot]);
        if (++qslot == 2) { qslot = 0; qphase ^= 1u; }
      }
      // All MMAs this thread issued must finish before TMEM is released.
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0u) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // Same barrier sequence for every thread; a failed wait only disables work.
    const uint32_t ew = warp - kEpiWarp0;             // 0..3
    const uint32_t lane_grp = (warp & 3u) * 32u;      // TMEM lanes this warp may access
    const uint32_t et = ew * 32u + lane;              // 0..127
    int acc = 0;
    uint32_t aphase = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
      int row, t0, nt;
      ScanRow g;
      scan_item(a, item, row, t0, nt, g);
      if (nt == 0) continue;
      named_bar_sync(1, 128);
      if (et < (uint32_t)HI) {
        float wv = a.w[(int64_t)row * HI + et];
        if (FP8) wv *= a.q_scale[row];
        sW[et] = wv;
      }
      named_bar_sync(1, 128);
      for (int t = 0; t < nt; ++t) {
        const bool got = ok && mbar_wait(&acc_full[acc], aphase, ctl, 0x301);
        ok = __all_sync(0xffffffffu, got);
        if (ok) {
          tc_fence_after();
          uint32_t r[HI];
          tmem_load_heads<HI>(tmem_base + (lane_grp << 16) + acc * N, r);
          tmem_wait_ld(r);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[acc]);
          const int s = (t0 + t) * kTileKeys + (int)lane_grp + (int)lane;
          if (s < g.len) {
            float score = relu_weighted_head_sum<HI>(r, sW);
            if (FP8) score *= a.k_scale[g.key_base + s];
            g.out[s] = score + 0.0f;
          }
        }
        if (++acc == 2) { acc = 0; aphase ^= 1u; }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int HI, bool FP8, int KB>
static size_t scan_smem_bytes() {
  constexpr int N = HI < 16 ? 16 : HI;
  return 1024 + kScanStages * kTileKeys * KB * kSwizzleBytes + 2 * N * KB * kSwizzleBytes + 2 * HI * 4 +
         (2 * kScanStages + 9) * 8 + 16;
}

template <int HI, bool FP8, int KB>
static cudaError_t launch_scan_t(const CUtensorMap& tq, const CUtensorMap& tk, const ScanArgs& a, int grid,
                                 cudaStream_t stream) {
  const size_t smem = scan_smem_bytes<HI, FP8, KB>();
  auto kern = indexer_scan_kernel<HI, FP8, KB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kScanThreads, smem, stream>>>(tq, tk, a);
  return cudaGetLastError();
}

cudaError_t launch_indexer_scan(int HI, bool fp8, int kblocks, const CUtensorMap& tq, const CUtensorMap& tk,
                                const ScanArgs& a, int grid, cudaStream_t stream) {
#define DSA_SCAN_CASE(H)                                                     \
  case H:                                                                    \
    if (fp8) return launch_scan_t<H, true, 1>(tq, tk, a, grid, stream);     \
    if (kblocks == 1) return launch_scan_t<H, false, 1>(tq, tk, a, grid, stream); \
    return launch_scan_t<H, false, 2>(tq, tk, a, grid, stream);
  switch (HI) {
    DSA_SCAN_CASE(4)
    DSA_SCAN_CASE(8)
    DSA_SCAN_CASE(16)
    DSA_SCAN_CASE(32)
    DSA_SCAN_CASE(64)
    default:
      return cudaErrorInvalidValue;
  }
#undef DSA_SCAN_CASE
}

}  // namespace dsa
