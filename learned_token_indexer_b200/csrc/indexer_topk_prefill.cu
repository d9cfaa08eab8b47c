// indexer_topk_prefill.cu -- fused Lightning Indexer + causal top-k for a
// prefill chunk: eqs. (1) and (2) of page "2.2.1 · DSA 与索引器" (§1.1), with
// the fusion the page's §2 asks for (score tiles are filtered while they are
// produced and merged into each row's final top-k; the B x n x n score
// matrix is never written).
//
// Work unit: a block of 8 consecutive query tokens of one sequence against
// all keys 0..t of its last token.  Persistent grid, heavy blocks first, snake
// order over CTAs.  Per CTA (18 warps):
//   warp 0      TMA producer: Q of the block (both groups, once), K tiles;
//   warp 1      tcgen05 MMA issuer, TMEM owner: for each 128-key tile and
//               each accumulator g, D_g[128 keys x T*HI] (+)= K Q_g^T, where
//               an accumulator holds T = 2 tokens (four accumulators of 2*HI
//               columns, one per epilogue warpgroup, when 2*HI >= 16) or
//               T = 4 tokens (two accumulators shared by all warpgroups);
//   warps 2..17 epilogue, 4 warpgroups; warpgroup j takes tokens 2j and
//               2j+1 (four accumulators) or j and 4+j (two), in MMA order:
//               TMEM -> ReLU * w -> head sum = I[t, s];
//               causal mask; then the streaming filter below; an accumulator
//               is released to the MMA issuer by the warpgroups that read it;
//               after the block's last tile the exact select (select.cuh)
//               writes idx (and scores).
// Streaming filter, per token: a 512-bin histogram of accepted scores over a
// monotone binning of the score (quarter-octaves for 2^-31 <= |x| < 2^31).
// bin_floor only rises: once at least k accepted entries lie in bins above
// bin_floor, no later key (higher position) in bin <= bin_floor can enter the
// top k, so such keys are dropped.  Accepted (key, position) pairs go to a
// per-(CTA, token slot) candidate buffer in global memory (L2 resident).
#include "indexer_common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace dsa {

namespace {

constexpr int kQB = 8;          // tokens per block
constexpr int kTA = 4;          // tokens per accumulator group
constexpr int kPrefillThreads = 576;   // producer, MMA, 4 epilogue warpgroups
constexpr int kHistBins = kScoreBins;  // streaming histogram bins (499 used)

// Raise a token's floor from its histogram (one warp): the bin where the
// running count of accepted scores, from the top bin down, first reaches k
// (at least k accepted scores lie in that bin or above, so nothing in a lower
// bin can enter the top k).  Lane l sums bins [512 - 16(l+1), 512 - 16l).
__device__ __forceinline__ void raise_floor(const uint32_t* hist, uint32_t k, uint32_t* floor_key, uint32_t lane) {
  constexpr int kPerLane = kHistBins / 32;
  const int b0 = kHistBins - kPerLane * ((int)lane + 1);
  uint32_t h[kPerLane];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < kPerLane; ++j) {
    h[j] = hist[b0 + j];
    local += h[j];
  }
  uint32_t incl = local;   // count from the top bin down to this lane's lowest bin
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= (uint32_t)o) incl += v;
  }
  const uint32_t reach = __ballot_sync(0xffffffffu, incl >= k);
  if (reach == 0u) return;   // fewer than k accepted so far
  const uint32_t L = (uint32_t)(__ffs(reach) - 1);
  if (lane == L) {
    // highest bin of this lane's range where the running count reaches k
    // (no early exit, so h stays in registers)
    uint32_t run = incl - local;
    int f = b0;
    bool found = false;
#pragma unroll
    for (int j = kPerLane - 1; j >= 0; --j) {
      run += h[j];
      const bool hit = !found && run >= k;
      f = hit ? b0 + j : f;
      found = found || hit;
    }
    uint32_t lo, hi;
    bin_key_range((uint32_t)f, lo, hi);
    if (lo > *floor_key) *floor_key = lo;
  }
}

// Accumulator plan: each TMEM accumulator holds the heads of kTPA tokens of
// the block (MMA N = kTPA * HI).  Two tokens per accumulator (four
// accumulators, one per epilogue warpgroup, which releases it alone) where the
// MMA shape allows it (N >= 16); four tokens otherwise, and in the wide plan
// (two accumulators, every warpgroup reading one token of each).  The wide
// plan halves the MMA instructions and the shared-memory reads of each K^I
// tile (it is read once per accumulator); measured on B200 with H^I = 64 it
// is faster with long histories (8192 queries against 32768 keys: 4.91 ->
// 4.80 ms) and slower with short ones (8192 against 8192: 0.896 -> 0.929 ms),
// so the launch picks it from the history length.
template <int HI, bool WIDE>
struct AccPlan {
  static constexpr int kTPA = (WIDE || 2 * HI < 16) ? 4 : 2;
  static constexpr int kNA = kQB / kTPA;
  static constexpr int kNP = kTPA * HI;
};

struct Block {
  int b, t0;      // sequence, first local query row
  int nvalid;     // valid tokens in the block (<= 8)
  int nt[4];      // key tiles per accumulator (0 = no valid token in it)
};

__device__ __forceinline__ bool block_of(const PrefillArgs& a, int r, Block& blk, int tpa) {
  // Round r of the snake schedule: CTA c takes item r*G + (c or G-1-c).
  const int G = gridDim.x;
  const int c = blockIdx.x;
  const int item = r * G + ((r & 1) ? (G - 1 - c) : c);
  const int per_seq = a.nblk - a.first_blk;
  if (item >= a.B * per_seq) return false;
  const int j = item / a.B;
  blk.b = item - j * a.B;
  const int bi = a.nblk - 1 - j;   // heaviest (last) blocks first
  blk.t0 = bi * kQB;
  blk.nvalid = min(kQB, a.nq - blk.t0);
  for (int g = 0; g < kQB / tpa; ++g) {
    const int last = min(blk.t0 + tpa * g + tpa - 1, a.nq - 1);
    if (blk.t0 + tpa * g >= a.nq) {
      blk.nt[g] = 0;
    } else {
      const int tmax = a.q_offset + last;
      blk.nt[g] = tmax / kTileKeys + 1;
    }
  }
  for (int g = kQB / tpa; g < 4; ++g) blk.nt[g] = 0;
  return true;
}

}  // namespace

template <int HI, bool FP8, int KB, int STAGES, bool WIDE>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    indexer_topk_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q,
                                const __grid_constant__ CUtensorMap tmap_k, const PrefillArgs a) {
  constexpr int N = kTA * HI;                                 // Q rows per TMA group (4 tokens)
  using Plan = AccPlan<HI, WIDE>;
  constexpr int kNA = Plan::kNA, kNP = Plan::kNP, kTPA = Plan::kTPA;
  constexpr int kQGroupBytes = N * KB * kSwizzleBytes;
  constexpr int kKBytes = kTileKeys * KB * kSwizzleBytes;
  constexpr uint32_t kTmemCols = (2 * N <= 32) ? 32 : (2 * N <= 64 ? 64 : (2 * N <= 128 ? 128 : (2 * N <= 256 ? 256 : 512)));
  constexpr uint32_t kIdesc = instr_desc(ElemTraits<FP8>::kFormat, kTileKeys, kNP);
  constexpr int kElemsPerBlock = ElemTraits<FP8>::kElemsPerBlock;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sQ = sK + STAGES * kKBytes;
  float* sW = reinterpret_cast<float*>(sQ + 2 * kQGroupBytes);            // [8][HI]
  uint32_t* sHist = reinterpret_cast<uint32_t*>(sW + kQB * HI);           // [8][512]
  uint32_t* sCnt = sHist + kQB * kHistBins;                               // [8][4 warps]
  uint32_t* sFloorKey = sCnt + kQB * 4;                                   // [8]
  SelectShared<128>* sSel = reinterpret_cast<SelectShared<128>*>(sFloorKey + kQB);  // [4]
  uint64_t* bars = reinterpret_cast<uint64_t*>(
      (reinterpret_cast<uintptr_t>(sSel + 4) + 7) & ~uintptr_t(7));
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + STAGES;
  uint64_t* q_full = bars + 2 * STAGES;
  uint64_t* q_empty = q_full + 1;
  uint64_t* acc_full = q_empty + 1;   // [kNA]
  uint64_t* acc_empty = acc_full + 4; // [kNA]
  uint64_t* mma_done = acc_empty + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int g = 0; g < kNA; ++g) {
      mbar_init(&acc_full[g], 1);
      mbar_init(&acc_empty[g], kNA == 4 ? 4 : 16);   // the owning warpgroup, or all four
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

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t kphase = 0, qphase = 0;
      uint32_t k_last_parity[STAGES];
      bool k_issued[STAGES];
      for (int s = 0; s < STAGES; ++s) k_issued[s] = false;
      bool q_issued = false;
      uint32_t q_last_parity = 0;
      bool ok = true;
      Block blk;
      for (int r = 0; ok && block_of(a, r, blk, kTPA); ++r) {
        if (!(ok = mbar_wait(q_empty, qphase ^ 1u, ctl, 0x1101))) break;
        mbar_arrive_expect_tx(q_full, 2 * kQGroupBytes);
        for (int g = 0; g < 2; ++g)
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sQ + g * kQGroupBytes + kb * N * kSwizzleBytes, &tmap_q, q_full, kb * kElemsPerBlock,
                        (blk.b * a.nq + blk.t0 + kTA * g) * HI);
        q_issued = true;
        q_last_parity = qphase;
        qphase ^= 1u;
        const int nt = max(max(blk.nt[0], blk.nt[1]), max(blk.nt[2], blk.nt[3]));
        for (int t = 0; t < nt; ++t) {
          if (!(ok = mbar_wait(&k_empty[stage], kphase ^ 1u, ctl, 0x1102))) break;
          mbar_arrive_expect_tx(&k_full[stage], kKBytes);
          const int y = blk.b * a.kv_len + t * kTileKeys;
          for (int kb = 0; kb < KB; ++kb)
            tma_load_2d(sK + stage * kKBytes + kb * kTileKeys * kSwizzleBytes, &tmap_k, &k_full[stage],
                        kb * kElemsPerBlock, y);
          k_issued[stage] = true;
          k_last_parity[stage] = kphase;
          if (++stage == STAGES) { stage = 0; kphase ^= 1u; }
        }
      }
      if (!ok) {
        for (int s = 0; s < STAGES; ++s)
          if (k_issued[s]) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&k_full[s]), k_last_parity[s]) && globaltimer_ns() - t0 < a.timeout_ns) {
            }
          }
        if (q_issued) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(smem_u32(q_full), q_last_parity) && globaltimer_ns() - t0 < a.timeout_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0;
      uint32_t kphase = 0, qphase = 0, aphase[4] = {0u, 0u, 0u, 0u};
      bool ok = true;
      Block blk;
      for (int r = 0; ok && block_of(a, r, blk, kTPA); ++r) {
        if (!(ok = mbar_wait(q_full, qphase, ctl, 0x1201))) break;
        qphase ^= 1u;
        tc_fence_after();
        const int nt = max(max(blk.nt[0], blk.nt[1]), max(blk.nt[2], blk.nt[3]));
        for (int t = 0; t < nt && ok; ++t) {
          if (!(ok = mbar_wait(&k_full[stage], kphase, ctl, 0x1202))) break;
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < kNA; ++g) {
            if (t >= blk.nt[g]) continue;
            if (!(ok = mbar_wait(&acc_empty[g], aphase[g] ^ 1u, ctl, 0x1203))) break;
            aphase[g] ^= 1u;
            tc_fence_after();
            // accumulator g holds Q rows [g*kNP, (g+1)*kNP): inside TMA group
            // (g*kTPA)/4 at row (g*kTPA)%4 * HI; K blocks are N rows apart
            const int grp = (g * kTPA) / kTA, row0 = ((g * kTPA) % kTA) * HI;
            issue_tile_mma<FP8>(tmem_base + g * kNP, smem_u32(sK + stage * kKBytes),
                                smem_u32(sQ + grp * kQGroupBytes + row0 * kSwizzleBytes), N, a.ksteps, kIdesc);
            tc_commit(&acc_full[g]);
          }
          if (!ok) break;
          tc_commit(&k_empty[stage]);
          if (++stage == STAGES) { stage = 0; kphase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(q_empty);
      }
      tc_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0u) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    // Four warpgroups, two block tokens each (token u of warpgroup j is block
    // slot st = ST(j, u)): with four accumulators warpgroup j owns accumulator
    // j (tokens 2j, 2j+1); with two, it takes token j of accumulator 0 and
    // token 4+j of accumulator 1.  Every thread of a warpgroup runs the same
    // sequence of named barriers; a wait that fails only turns the remaining
    // work into no-ops (no early exit, so no barrier is left short of threads).
    const uint32_t wg = (warp - 2) >> 2;                  // 0..3
    const uint32_t tid = (warp - 2 - 4 * wg) * 32 + lane; // 0..127 inside the warpgroup
    const uint32_t bar_id = 2 + wg;
    const uint32_t quarter = warp & 3u;                   // TMEM lane quarter of this warp
    const uint32_t lane_grp = quarter * 32u;
    const uint32_t key_in_tile = lane_grp + lane;
    SelectShared<128>& sel = sSel[wg];
    // block slot, accumulator and accumulator column of token u of this group
    auto ST = [&](int u) { return kNA == 4 ? 2 * (int)wg + u : kTA * u + (int)wg; };
    auto ACC = [&](int u) { return kNA == 4 ? (int)wg : u; };
    uint32_t aphase[2] = {0u, 0u};
    bool ok = true;
    Block blk;
    for (int r = 0; block_of(a, r, blk, kTPA); ++r) {
      named_bar_sync(bar_id, 128);
      int tok_t[2];
      bool tok_valid[2];
      int tok_nt[2];   // key tiles of the accumulator holding token u
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int li = blk.t0 + ST(u);
        tok_valid[u] = li < a.nq;
        tok_t[u] = a.q_offset + li;
        tok_nt[u] = blk.nt[ACC(u)];
      }
      for (int i = (int)tid; i < 2 * kHistBins; i += 128) {
        const int u = i / kHistBins;
        sHist[ST(u) * kHistBins + (i - u * kHistBins)] = 0u;
      }
      if (tid < 2u) sFloorKey[ST((int)tid)] = 0u;   // key 0: every score passes
      for (int i = (int)tid; i < 2 * HI; i += 128) {
        const int u = i / HI, h = i - u * HI;
        const int li = blk.t0 + ST(u);
        float wv = 0.0f;
        if (li < a.nq) {
          const int64_t row = (int64_t)blk.b * a.nq + li;
          wv = a.w[row * HI + h];
          if (FP8) wv *= a.q_scale[row];
        }
        sW[ST(u) * HI + h] = wv;
      }
      named_bar_sync(bar_id, 128);
      const int nt_max = max(tok_nt[0], tok_nt[1]);
      // accepted (key, position) pairs: this warp's sub-buffer of each token
      // (warp q of the group sees keys with s mod 128 in [32q, 32q + 32))
      uint2* cand_w[2];
      uint32_t cnt[2] = {0u, 0u};   // accepted entries (stored while below sub_cap)
      const uint32_t sub_cap = (uint32_t)(a.cand_cap / 4);
#pragma unroll
      for (int u = 0; u < 2; ++u)
        cand_w[u] = a.cand + ((int64_t)blockIdx.x * kQB + ST(u)) * a.cand_cap + quarter * (a.cand_cap / 4);
      for (int t = 0; t < nt_max; ++t) {
        const int s = t * kTileKeys + (int)key_in_tile;
        float ks = 1.0f;
        if (FP8 && ok) ks = (s < a.kv_len) ? a.k_scale[(int64_t)blk.b * a.kv_len + s] : 0.0f;
        float score[2] = {0.0f, 0.0f};
        if constexpr (kNA == 4) {
          // both tokens in this group's own accumulator: one wait, one release
          const bool got = ok && mbar_wait(&acc_full[wg], aphase[0], ctl, 0x1301);
          ok = __all_sync(0xffffffffu, got);
          aphase[0] ^= 1u;
          if (ok) {
            tc_fence_after();
            group_head_sums<HI, 2>(tmem_base + (lane_grp << 16) + wg * kNP, sW + ST(0) * HI, score, &acc_empty[wg],
                                   lane);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            if (t >= tok_nt[u]) continue;
            const bool got = ok && mbar_wait(&acc_full[u], aphase[u], ctl, 0x1301);
            ok = __all_sync(0xffffffffu, got);
            aphase[u] ^= 1u;
            if (!ok) continue;
            tc_fence_after();
            float sc[1];
            group_head_sums<HI, 1>(tmem_base + (lane_grp << 16) + u * kNP + wg * HI, sW + ST(u) * HI, sc,
                                   &acc_empty[u], lane);
            score[u] = sc[0];
          }
        }
        if (!ok) continue;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (t >= tok_nt[u]) continue;
          const float sc_u = FP8 ? score[u] * ks : score[u];
          // streaming filter: a key below the token's floor cannot be in its
          // top k (the floor only rises; another warp may raise it meanwhile)
          const int st = ST(u);
          const uint32_t key = float_to_key(sc_u);
          const uint32_t floor_key = *reinterpret_cast<volatile const uint32_t*>(&sFloorKey[st]);
          const bool acc = tok_valid[u] && s <= tok_t[u] && key >= floor_key;
          const uint32_t mask = __ballot_sync(0xffffffffu, acc);
          if (acc) {
            const uint32_t slot = cnt[u] + __popc(mask & ((1u << lane) - 1u));
            if (slot < sub_cap) cand_w[u][slot] = make_uint2(key, (uint32_t)s);
            // histogram of accepted scores, one atomic per distinct bin of the warp
            const uint32_t bin = score_bin(key);
            const uint32_t peers = __match_any_sync(mask, bin);
            if (lane == (uint32_t)(__ffs(peers) - 1)) atomicAdd(&sHist[st * kHistBins + bin], (uint32_t)__popc(peers));
          }
          cnt[u] += (uint32_t)__popc(mask);
          // raise the floor (every tile for the first 64 tiles, then on 4
          // tiles of every 16, where a long history has settled it; by a
          // warp that rotates with the tile so the four warps share the
          // work): the bin where the count of accepted scores from the top
          // first reaches k.  Two warps may raise one token's floor at once;
          // each value written is a valid floor (counts only grow), so a lost
          // update only admits more
          if (quarter == ((uint32_t)(t + 2 * u) & 3u) && (t < 64 || ((t >> 2) & 3) == 0))
            raise_floor(sHist + st * kHistBins, (uint32_t)a.k, &sFloorKey[st], lane);
        }
      }
      // per-warp candidate counts for the select
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (lane == 0) sCnt[ST(u) * 4 + quarter] = cnt[u];
      named_bar_sync(bar_id, 128);
      if (tid == 0) sel.aborted = *abort_flag;
      named_bar_sync(bar_id, 128);
      if (sel.aborted) continue;   // warpgroup-uniform: nothing below is valid
      // ---- exact select of each token's top min(k, t+1)
      for (int g = 0; g < 2; ++g) {
        if (!tok_valid[g] || tok_nt[g] == 0) continue;
        const int st = ST(g);
        const int kk = min(a.k, tok_t[g] + 1);
        const uint32_t c0 = sCnt[st * 4], c1 = sCnt[st * 4 + 1], c2 = sCnt[st * 4 + 2], c3 = sCnt[st * 4 + 3];
        const int64_t row = (int64_t)blk.b * a.nq + blk.t0 + st;
        const uint32_t sub_cap = (uint32_t)(a.cand_cap / 4);
        if (max(max(c0, c1), max(c2, c3)) > sub_cap) {
          // a sub-buffer overflowed (warpgroup-uniform): the row goes to the second pass
          if (tid == 0 && a.ovf_list) a.ovf_list[atomicAdd(a.ovf_count, 1u)] = (int32_t)row;
          continue;
        }
        const int m = (int)(c0 + c1 + c2 + c3);
        uint32_t* hist = sHist + st * kHistBins;
        const uint2* buf = a.cand + ((int64_t)blockIdx.x * kQB + st) * a.cand_cap;
        const int64_t sub = a.cand_cap / 4;
        // entry i of the token's candidates: the four warp sub-buffers in order
        auto get = [=](int i, uint32_t& key, uint32_t& pos) {
          uint32_t off = (uint32_t)i;
          int q = 0;
          if (off >= c0) {
            off -= c0;
            q = 1;
            if (off >= c1) {
              off -= c1;
              q = 2;
              if (off >= c2) {
                off -= c2;
                q = 3;
              }
            }
          }
          const uint2 e = buf[q * sub + off];
          key = e.x;
          pos = e.y;
        };
        // the filter keeps at least kk candidates, so the bin always exists;
        // a miss is reported and the row is emitted from bin 0 (in bounds)
        if (!group_find<128>(hist, kHistBins, (uint32_t)kk, true, sel, tid, bar_id) && tid == 0)
          report_status(a.status, kStatusDeviceCheck, 0x5e1ec6u);
        const uint32_t b0 = sel.found_bin;
        const uint32_t need = (uint32_t)kk - sel.found_beyond;
        named_bar_sync(bar_id, 128);   // hist of this token becomes scratch
        // One pass over the candidates: entries above the cut-off bin are
        // selected outright and written now; the cut-off bin's entries are
        // gathered into this group's scratch, where the refinement runs.
        int32_t* idx_row = a.idx_out + row * a.k;
        float* score_row = a.score_out ? a.score_out + row * a.k : nullptr;
        uint2* bnd = a.bnd + ((int64_t)blockIdx.x * 4 + wg) * a.cand_cap;
        if (tid == 0) {
          sel.out_count = 0u;
          sel.bnd_count = 0u;
        }
        named_bar_sync(bar_id, 128);
        for (int j0 = 0; j0 < m; j0 += 128 * kBatch) {
          uint32_t key[kBatch], pos[kBatch];
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            key[u] = 0u;
            pos[u] = 0u;
            const int i = j0 + u * 128 + (int)tid;
            if (i < m) get(i, key[u], pos[u]);
          }
          // the batch's classes first, then one warp scan of the packed
          // counts and one pair of shared atomics per warp (per-entry atomics
          // put a shared-atomic round trip on the chain of every entry)
          uint32_t abits = 0, obits = 0;
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            const int i = j0 + u * 128 + (int)tid;
            const uint32_t bin = score_bin(key[u]);
            abits |= (i < m && bin > b0) ? (1u << u) : 0u;
            obits |= (i < m && bin == b0) ? (1u << u) : 0u;
          }
          const uint32_t packed = (uint32_t)__popc(abits) | ((uint32_t)__popc(obits) << 16);
          uint32_t incl = packed;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t2 = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= (uint32_t)o) incl += t2;
          }
          uint32_t base_a = 0, base_o = 0;
          if (lane == 31) {
            if (incl & 0xFFFFu) base_a = atomicAdd(&sel.out_count, incl & 0xFFFFu);
            if (incl >> 16) base_o = atomicAdd(&sel.bnd_count, incl >> 16);
          }
          const uint32_t excl = incl - packed;
          uint32_t pa = __shfl_sync(0xffffffffu, base_a, 31) + (excl & 0xFFFFu);
          uint32_t po = __shfl_sync(0xffffffffu, base_o, 31) + (excl >> 16);
#pragma unroll
          for (int u = 0; u < kBatch; ++u) {
            if ((abits >> u) & 1u) {
              if (pa < (uint32_t)kk) {
                idx_row[pa] = (int32_t)pos[u];
                if (score_row) score_row[pa] = key_to_float(key[u]);
              }
              ++pa;
            } else if ((obits >> u) & 1u) {
              if (po < (uint32_t)a.cand_cap) bnd[po] = make_uint2(key[u], pos[u]);
              ++po;
            }
          }
        }
        named_bar_sync(bar_id, 128);
        const int nb = (int)min((uint32_t)a.cand_cap, sel.bnd_count);
        auto get_bnd = [bnd](int i, uint32_t& key, uint32_t& pos) {
          const uint2 e = bnd[i];
          key = e.x;
          pos = e.y;
        };
        SelectResult res;
        bin_key_range(b0, res.lo, res.hi);
        res.key_all_in = 1;
        res.pos_hi = 0;
        if (need != (uint32_t)nb)
          res = group_refine<128, kHistBins>(get_bnd, nb, res.lo, res.hi, need, (uint32_t)tok_t[g], hist, sel, tid,
                                             bar_id, a.status);
        uint32_t blo, bhi;
        bin_key_range(b0, blo, bhi);
        group_emit_append<128>(get_bnd, nb, res, blo, bhi, kk, idx_row, score_row, sel, tid, bar_id);
        group_emit_finish<128>(kk, a.k, idx_row, score_row, sel, tid, bar_id, a.status);
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

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int HI, bool FP8, int KB>
struct PrefillConfig {
  static constexpr int N = kTA * HI;
  static constexpr int kQBytes = 2 * N * KB * kSwizzleBytes;
  static constexpr int kKBytes = kTileKeys * KB * kSwizzleBytes;
  static constexpr int kFixed = 1024 /*align*/ + kQBytes + kQB * HI * 4 + kQB * kHistBins * 4 + 5 * kQB * 4 +
                                4 * (int)sizeof(SelectShared<128>) + 8 + 16 * 8 + 16;
  static constexpr int kBudget = 227 * 1024;
  static constexpr int kStagesFit = (kBudget - kFixed) / kKBytes;
  static constexpr int STAGES = kStagesFit > 6 ? 6 : kStagesFit;
  static_assert(STAGES >= 2, "not enough shared memory for two K stages");
  static constexpr int kSmem = kFixed + STAGES * kKBytes + 2 * STAGES * 8;
};

template <int HI, bool FP8, int KB, bool WIDE = false>
static cudaError_t launch_prefill_t(const CUtensorMap& tq, const CUtensorMap& tk, const PrefillArgs& a, int grid,
                                    cudaStream_t stream) {
  using C = PrefillConfig<HI, FP8, KB>;
  auto kern = indexer_topk_prefill_kernel<HI, FP8, KB, C::STAGES, WIDE>;
  cudaError_t e = setup_once_per_device([&]() { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem); });
  if (e != cudaSuccess) return e;
  kern<<<grid, kPrefillThreads, C::kSmem, stream>>>(tq, tk, a);
  return cudaGetLastError();
}

// History length (keys seen by the chunk's last query) from which bf16
// H^I = 64 launches take the wide plan.
constexpr int kWideMinKeys = 16384;

cudaError_t launch_indexer_topk_prefill(int HI, bool fp8, int kblocks, const CUtensorMap& tq,
                                        const CUtensorMap& tk, const PrefillArgs& a, int grid, cudaStream_t stream) {
#define DSA_PF_CASE(H)                                                          \
  case H:                                                                       \
    if (fp8) return launch_prefill_t<H, true, 1>(tq, tk, a, grid, stream);      \
    if (kblocks == 1) return launch_prefill_t<H, false, 1>(tq, tk, a, grid, stream); \
    if (H == 64 && a.q_offset + a.nq >= kWideMinKeys)                          \
      return launch_prefill_t<H, false, 2, true>(tq, tk, a, grid, stream);      \
    return launch_prefill_t<H, false, 2>(tq, tk, a, grid, stream);
  switch (HI) {
    DSA_PF_CASE(4)
    DSA_PF_CASE(8)
    DSA_PF_CASE(16)
    DSA_PF_CASE(32)
    DSA_PF_CASE(64)
    default:
      return cudaErrorInvalidValue;
  }
#undef DSA_PF_CASE
}

int prefill_block_tokens() { return kQB; }

}  // namespace dsa
