// indexer_scan.cu -- Lightning Indexer scores written densely, one query token
// per row (page "2.2.1 · DSA 与索引器", §1.1 eq. (1); decode step of §2).
//
// Used by the decode step (one new token per sequence scans every cached
// indexer key; the scores of one step are small, so they are written out and
// a separate select kernel takes the top-k) and by the debug entry point that
// materialises the causal prefill score matrix for small n.
//
// Per CTA: warp 0 = TMA producer, warp 1 = tcgen05 MMA issuer (and TMEM
// owner), warps 2..9 = two epilogue warpgroups (TMEM -> ReLU * w -> head sum
// -> global); with an e4m3 cache, warp 10 stages each tile's per-key scales
// into a shared ring by cp.async, so no epilogue thread waits on them.  The MMA computes D[128 keys x N] with keys on TMEM lanes and
// the token's heads on columns into four accumulators used in turn; the two
// warpgroups take alternate tiles, so two tiles' epilogues run at once while
// the MMA fills the next ones.  Work items are (row, run of key tiles),
// spread over a persistent grid; the producer stages each item's q^I tile and
// its head weights w[t, :] together.
#include "indexer_common.cuh"
#include "kernels.h"

namespace dsa {

namespace {

// K tiles in flight: as many as shared memory holds beside the q tiles and
// the row prefix (11 tiles of 128-byte rows = 176 KB, 5 of 256-byte rows =
// 160 KB).  Under the scan's load the HBM latency is 2.5-4.5 us, so the bytes
// in flight per SM set the rate (a tile every 0.54 us with 128 KB in flight).
template <int KB>
constexpr int scan_stages() { return KB == 1 ? 11 : 5; }
constexpr int kEpiWarp0 = 2;
constexpr int kEpiWarps = 8;     // two warpgroups
constexpr int kScaleWarp = kEpiWarp0 + kEpiWarps;   // e4m3 only
constexpr int kScanAcc = 4;      // accumulators in TMEM
constexpr int kScaleStages = 8;  // tiles of key scales in flight
template <bool FP8>
constexpr int scan_threads() { return 32 * (kScaleWarp + (FP8 ? 1 : 0)); }

struct ScanRow {
  int64_t key_base;
  int len;
  int qrow;      // row of q^I / w / q_scale
  float* out;
};

__device__ __forceinline__ ScanRow scan_row(const ScanArgs& a, int r) {
  ScanRow g;
  if (a.mode == 0) {
    const int q = a.row_list ? a.row_list[r] : r;
    const int b = q / a.nq, i = q - b * a.nq;
    g.key_base = (int64_t)b * a.kv_len;
    g.len = a.q_offset + i + 1;
    g.qrow = q;
    g.out = a.out + (int64_t)r * a.kv_len;
  } else {
    const int64_t lo = a.cu_seqlens[r];
    g.key_base = lo;
    g.len = (int)(a.cu_seqlens[r + 1] - lo);
    g.qrow = r;
    g.out = a.out + lo;
  }
  return g;
}

// Item i -> (row, first tile, number of tiles); ntiles == 0 means empty.
// Ragged decode rows (balanced mode) number only the non-empty chunks:
// pre[r] = chunks of rows 0..r-1, so a persistent grid gets an even share of
// the real work whatever the length mix; otherwise every row has max_chunks
// item slots.
__device__ __forceinline__ void scan_item(const ScanArgs& a, int item, int& row, int& t0, int& nt,
                                          ScanRow& g, const int* pre, bool balanced) {
  int c;
  if (balanced) {
    int lo = 0, hi = a.rows;   // pre[lo] <= item < pre[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre[mid] <= item) lo = mid; else hi = mid;
    }
    row = lo;
    c = item - pre[lo];
  } else {
    row = item / a.max_chunks;
    c = item - row * a.max_chunks;
  }
  g = scan_row(a, row);
  const int tiles = (g.len + kTileKeys - 1) / kTileKeys;
  t0 = c * a.chunk_tiles;
  nt = tiles - t0;
  nt = nt < 0 ? 0 : (nt > a.chunk_tiles ? a.chunk_tiles : nt);
}

// Eq. (1) for this thread's key: sum_j w_j * ReLU(D_j) with four independent
// packed partial sums (the epilogue's critical path is this chain, one warp
// per SM sub-partition), the weights read four at a time from shared memory.
template <int HI>
__device__ __forceinline__ float scan_head_sum(const uint32_t (&acc)[HI], const float* w_smem) {
  static_assert(HI % 4 == 0, "heads come in fours");
  float2 p[2][2] = {{make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)},
                    {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)}};
#pragma unroll
  for (int j = 0; j < HI; j += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(w_smem + j);
    const float2 r0 = make_float2(fmaxf(__uint_as_float(acc[j]), 0.0f), fmaxf(__uint_as_float(acc[j + 1]), 0.0f));
    const float2 r1 = make_float2(fmaxf(__uint_as_float(acc[j + 2]), 0.0f), fmaxf(__uint_as_float(acc[j + 3]), 0.0f));
    const int c = (j >> 2) & 1;
    p[c][0] = ffma2(make_float2(w4.x, w4.y), r0, p[c][0]);
    p[c][1] = ffma2(make_float2(w4.z, w4.w), r1, p[c][1]);
  }
  return ((p[0][0].x + p[0][0].y) + (p[0][1].x + p[0][1].y)) + ((p[1][0].x + p[1][0].y) + (p[1][1].x + p[1][1].y));
}

}  // namespace

template <int HI, bool FP8, int KB>
__global__ void __launch_bounds__(scan_threads<FP8>(), 1)
    indexer_scan_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const ScanArgs a) {
  constexpr int N = HI < 16 ? 16 : HI;
  constexpr int kQBytes = N * KB * kSwizzleBytes;
  constexpr int kKBytes = kTileKeys * KB * kSwizzleBytes;
  constexpr uint32_t kTmemCols =
      (kScanAcc * N <= 32) ? 32 : (kScanAcc * N <= 64 ? 64 : (kScanAcc * N <= 128 ? 128 : 256));
  static_assert(kScanAcc * N <= 256, "accumulators exceed the TMEM allocation");
  constexpr uint32_t kWBytes = HI * 4;
  constexpr uint32_t kIdesc = instr_desc(ElemTraits<FP8>::kFormat, kTileKeys, N);
  constexpr int kElemsPerBlock = ElemTraits<FP8>::kElemsPerBlock;
  constexpr int kScanStages = scan_stages<KB>();

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sQ = sK + kScanStages * kKBytes;
  float* sW = reinterpret_cast<float*>(sQ + 2 * kQBytes);   // [2][HI], beside the two q^I slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + 2 * HI);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + kScanStages;
  uint64_t* q_full = bars + 2 * kScanStages;
  uint64_t* q_empty = q_full + 2;
  uint64_t* acc_full = q_empty + 2;
  uint64_t* acc_empty = acc_full + kScanAcc;
  uint64_t* mma_done = acc_empty + kScanAcc;
  uint64_t* ks_full = mma_done + 1;                 // [kScaleStages] (e4m3)
  uint64_t* ks_empty = ks_full + kScaleStages;      // [kScaleStages]
  float* sKS = reinterpret_cast<float*>(ks_empty + kScaleStages);   // [kScaleStages][128]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sKS + kScaleStages * kTileKeys);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  int* sPre = reinterpret_cast<int*>(tmem_slot + 4);   // [rows + 1] in balanced mode

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kScanStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1 + kEpiWarps);   // the MMA's commit and every epilogue warp
    }
    for (int s = 0; s < kScanAcc; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);              // the four warps of the warpgroup that reads it
    }
    mbar_init(mma_done, 1);
    for (int s = 0; s < kScaleStages; ++s) {
      mbar_init(&ks_full[s], 32);   // one cp.async arrival per lane of the scale warp
      mbar_init(&ks_empty[s], 4);   // the four warps of the warpgroup that reads the tile
    }
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
  // balanced numbering needs the ragged offsets and room for the prefix
  const bool balanced = a.balanced != 0 && a.mode == 1 && a.rows <= kScanMaxBalancedRows;
  if (balanced) {
    for (int r = threadIdx.x; r < a.rows; r += scan_threads<FP8>()) {
      const int64_t len = a.cu_seqlens[r + 1] - a.cu_seqlens[r];
      const int tiles = (int)((len + kTileKeys - 1) / kTileKeys);
      sPre[r + 1] = (tiles + a.chunk_tiles - 1) / a.chunk_tiles;
    }
    __syncthreads();
    if (warp == 0) {   // inclusive scan of the chunk counts, 32 rows at a time
      int carry = 0;
      for (int r0 = 1; r0 <= a.rows; r0 += 32) {
        const int r = r0 + (int)lane;
        int v = r <= a.rows ? sPre[r] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= (uint32_t)o) v += u;
        }
        if (r <= a.rows) sPre[r] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) sPre[0] = 0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};
  const int total_items = balanced ? sPre[a.rows] : a.rows * a.max_chunks;
  const int ksteps = a.ksteps;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // K^I is read once: evicted from L2 first, so the scores stay there
      const uint64_t k_policy = l2_policy_evict_first();
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
        scan_item(a, item, row, t0, nt, g, sPre, balanced);
        if (nt == 0) continue;
        if (!(ok = mbar_wait(&q_empty[qslot], qphase ^ 1u, ctl, 0x101))) break;
        mbar_arrive_expect_tx(&q_full[qslot], kQBytes + kWBytes);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(sQ + qslot * kQBytes + kb * N * kSwizzleBytes, &tmap_q, &q_full[qslot], kb * kElemsPerBlock,
                      g.qrow * HI);
        bulk_copy_g2s(smem_u32(sW + qslot * HI), a.w + (int64_t)g.qrow * HI, kWBytes, &q_full[qslot]);
        q_issued[qslot] = true;
        q_last_parity[qslot] = qphase;
        if (++qslot == 2) { qslot = 0; qphase ^= 1u; }
        for (int t = 0; t < nt; ++t) {
          if (!(ok = mbar_wait(&k_empty[stage], kphase ^ 1u, ctl, 0x102))) break;
          mbar_arrive_expect_tx(&k_full[stage], kKBytes);
          const int y = (int)(g.key_base + (int64_t)(t0 + t) * kTileKeys);
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d_hint(sK + stage * kKBytes + kb * kTileKeys * kSwizzleBytes, &tmap_k, &k_full[stage],
                             kb * kElemsPerBlock, y, k_policy);
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
      int stage = 0, qslot = 0;
      uint32_t kphase = 0, qphase = 0, n = 0;   // n: tile sequence number
      bool ok = true;
      for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
        int row, t0, nt;
        ScanRow g;
        scan_item(a, item, row, t0, nt, g, sPre, balanced);
        if (nt == 0) continue;
        if (!(ok = mbar_wait(&q_full[qslot], qphase, ctl, 0x201))) break;
        tc_fence_after();
        const uint32_t qaddr = smem_u32(sQ + qslot * kQBytes);
        for (int t = 0; t < nt; ++t) {
          const uint32_t acc = n % kScanAcc, aphase = (n / kScanAcc) & 1u;
          if (!(ok = mbar_wait(&k_full[stage], kphase, ctl, 0x202))) break;
          if (!(ok = mbar_wait(&acc_empty[acc], aphase ^ 1u, ctl, 0x203))) break;
          tc_fence_after();
          issue_tile_mma<FP8>(tmem_base + acc * N, smem_u32(sK + stage * kKBytes), qaddr, N, ksteps, kIdesc);
          tc_commit(&acc_full[acc]);
          tc_commit(&k_empty[stage]);
          if (++stage == kScanStages) { stage = 0; kphase ^= 1u; }
          ++n;
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
  } else if (FP8 && warp == (uint32_t)kScaleWarp) {
    // ------------------------------------------------------------ key scales (e4m3)
    // Tile n's 128 scales go to ring slot n % kScaleStages; lane l copies
    // keys l, l + 32, l + 64, l + 96 and its arrival fires when they land.
    uint32_t n = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total_items && ok; item += gridDim.x) {
      int row, t0, nt;
      ScanRow gr;
      scan_item(a, item, row, t0, nt, gr, sPre, balanced);
      for (int t = 0; t < nt; ++t, ++n) {
        const uint32_t ks = n % kScaleStages;
        const bool got = mbar_wait(&ks_empty[ks], ((n / kScaleStages) & 1u) ^ 1u, ctl, 0x401);
        if (!(ok = __all_sync(0xffffffffu, got))) break;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int key = (t0 + t) * kTileKeys + 32 * j + (int)lane;
          const bool in = key < gr.len;
          cp_async_4(smem_u32(sKS + ks * kTileKeys + 32 * j + lane), in ? a.k_scale + gr.key_base + key : a.k_scale,
                     in ? 4u : 0u);
        }
        cp_async_arrive_noinc(&ks_full[ks]);
      }
    }
    cp_async_wait_all();   // nothing may land after the CTA is gone
  } else {
    // ------------------------------------------------------------ epilogue
    // Same barrier sequence for every thread; a failed wait only disables work.
    // Warpgroup g takes the tiles whose sequence number n has n % 2 == g.
    const uint32_t g = (warp - kEpiWarp0) >> 2;       // 0..1
    // the scores are read again by the row top-k right after: kept in L2
    const uint64_t out_policy = l2_policy_evict_last();
    const uint32_t lane_grp = (warp & 3u) * 32u;      // TMEM lanes this warp may access
    int qslot = 0;
    uint32_t qphase = 0, n = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < total_items; item += gridDim.x) {
      int row, t0, nt;
      ScanRow gr;
      scan_item(a, item, row, t0, nt, gr, sPre, balanced);
      if (nt == 0) continue;
      // q_scale is requested before the wait so its latency hides behind it
      const float qs = FP8 ? __ldg(a.q_scale + gr.qrow) : 1.0f;
      const bool gotq = ok && mbar_wait(&q_full[qslot], qphase, ctl, 0x300);
      ok = __all_sync(0xffffffffu, gotq);
      const float* w_row = sW + qslot * HI;
      for (int t = 0; t < nt; ++t, ++n) {
        if ((n & 1u) != g) continue;
        const uint32_t acc = n % kScanAcc, aphase = (n / kScanAcc) & 1u;
        const int s = (t0 + t) * kTileKeys + (int)lane_grp + (int)lane;
        float kscale = 1.0f;
        if constexpr (FP8) {
          // the key's scale, staged by the scale warp
          const uint32_t ks = n % kScaleStages;
          const bool gs = ok && mbar_wait(&ks_full[ks], (n / kScaleStages) & 1u, ctl, 0x302);
          ok = __all_sync(0xffffffffu, gs);
          kscale = sKS[ks * kTileKeys + lane_grp + lane] * qs;
          __syncwarp();
          if (lane == 0) mbar_arrive(&ks_empty[ks]);
        }
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
          if (s < gr.len) {
            float score = scan_head_sum<HI>(r, w_row);
            if (FP8) score *= kscale;
            st_global_hint(gr.out + s, score + 0.0f, out_policy);
          }
        }
      }
      // this warp is done with the item's weights
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[qslot]);
      if (++qslot == 2) { qslot = 0; qphase ^= 1u; }
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
  return 1024 + scan_stages<KB>() * kTileKeys * KB * kSwizzleBytes + 2 * N * KB * kSwizzleBytes + 2 * HI * 4 +
         (2 * scan_stages<KB>() + 4 + 2 * kScanAcc + 1 + 2 * kScaleStages) * 8 + kScaleStages * kTileKeys * 4 + 16 +
         (kScanMaxBalancedRows + 1) * 4;
}

template <int HI, bool FP8, int KB>
static cudaError_t launch_scan_t(const CUtensorMap& tq, const CUtensorMap& tk, const ScanArgs& a, int grid,
                                 cudaStream_t stream) {
  const size_t smem = scan_smem_bytes<HI, FP8, KB>();
  auto kern = indexer_scan_kernel<HI, FP8, KB>;
  cudaError_t e = setup_once_per_device([&]() { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); });
  if (e != cudaSuccess) return e;
  kern<<<grid, scan_threads<FP8>(), smem, stream>>>(tq, tk, a);
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
