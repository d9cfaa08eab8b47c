// select.cuh -- exact top-k selection of one row by radix refinement, done by
// a group of NT threads that share a histogram in shared memory.
//
// Eq. (2) of page "2.2.1 · DSA 与索引器" (§1.1): S_t = TopK({I[t,s]}, min(k, t+1)).
// Entries are (key, pos) with key = order-preserving uint32 image of the
// score (-0.0 folded into +0.0) and pos the key position; the order is key
// descending, then position ascending (ties go to the lower position), so the
// selected set is unique.  The page (§2, top-k paragraph) names radix top-k as
// the usual way to avoid an O(t log t) sort; this is such a select:
//
//   1. keep an interval [lo, hi] of keys known to contain the cut-off key, and
//      `need` = how many entries inside the interval still have to be taken;
//   2. histogram the entries inside the interval by their next digit, find
//      the digit bin where the running count (from the top) reaches `need`,
//      and shrink the interval to that bin; stop early when the whole bin is
//      taken;
//   3. if the interval shrinks to one key with more entries than `need`,
//      refine the same way over positions (from the bottom: lowest first);
//   4. one output pass writes every selected entry in unspecified slot order.
#pragma once
#include "sm100.cuh"

namespace dsa {

// Entries read per thread per pass before they are processed (independent
// loads in flight).
constexpr int kBatch = 8;

// Coarse monotone binning of score keys (the order-preserving uint32 image of
// an fp32 score): quarter-octaves for 2^-31 <= |x| < 2^31, one bin for each
// tail and one for |x| < 2^-31.  Larger key <=> same or higher bin.
constexpr int kScoreBins = 512;      // bins 0..498 used
constexpr uint32_t kScoreLastBin = 498;

__device__ __forceinline__ uint32_t score_bin(uint32_t key) {
  const uint32_t k11 = key >> 21;
  if (k11 < 392u) return 0u;                    // x <= -2^31
  if (k11 < 640u) return 1u + (k11 - 392u);     // -2^31 < x <= -2^-31
  if (k11 < 1408u) return 249u;                 // |x| < 2^-31 (zeros)
  if (k11 < 1656u) return 250u + (k11 - 1408u); // 2^-31 <= x < 2^31
  return kScoreLastBin;                              // x >= 2^31
}

__device__ __forceinline__ void bin_key_range(uint32_t b, uint32_t& lo, uint32_t& hi) {
  uint32_t a, z;
  if (b == 0u) { a = 0u; z = 391u; }
  else if (b <= 248u) { a = z = 391u + b; }
  else if (b == 249u) { a = 640u; z = 1407u; }
  else if (b <= 497u) { a = z = 1408u + (b - 250u); }
  else { a = 1656u; z = 2047u; }
  lo = a << 21;
  hi = (z << 21) | 0x1FFFFFu;
}


struct SelectResult {
  uint32_t lo, hi;        // key interval of the cut-off
  uint32_t key_all_in;    // 1: every entry with key >= lo is selected
  uint32_t pos_hi;        // else: key == lo entries with pos <= pos_hi are selected
};

// Shared scratch of one selecting group.
template <int NT>
struct SelectShared {
  uint32_t warp_sum[NT / 32];
  uint32_t found_bin;
  uint32_t found_beyond;
  uint32_t out_count;
  uint32_t aborted;
  uint32_t bnd_count;
};

// Find the bin where the running count over `nbins` bins, traversed from the
// top (from_top) or from the bottom, first reaches `need` (1 <= need <= total).
// Result: sh.found_bin, sh.found_beyond = count strictly before it in
// traversal order.  All NT threads call it; it ends with a barrier.  Returns
// false (and leaves bin 0, nothing before it) when the bins hold fewer than
// `need` entries -- a broken caller invariant; callers report it and stop.
// Callers read the result before their next barrier and call again only
// after one.
template <int NT>
__device__ __forceinline__ bool group_find(const uint32_t* hist, int nbins, uint32_t need, bool from_top,
                                           SelectShared<NT>& sh, uint32_t tid, uint32_t bar_id) {
  constexpr uint32_t kNotFound = 0xFFFFFFFFu;
  if (tid == 0) {
    sh.found_bin = kNotFound;
    sh.found_beyond = 0u;
  }
  const int per = (nbins + NT - 1) / NT;
  const int i0 = (int)tid * per;
  uint32_t local = 0;
  for (int i = i0; i < i0 + per && i < nbins; ++i) local += hist[from_top ? nbins - 1 - i : i];
  const uint32_t lane = tid & 31u, w = tid >> 5;
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= (uint32_t)o) incl += v;
  }
  if (lane == 31) sh.warp_sum[w] = incl;
  named_bar_sync(bar_id, NT);
  // entries in the warps before this one: a scan over the warp sums
  // (a loop over them would be a chain of up to 31 shared loads)
  constexpr int NW = NT / 32;
  uint32_t wpre = 0;
  if constexpr (NW <= 4) {
    for (uint32_t j = 0; j < w; ++j) wpre += sh.warp_sum[j];
  } else {
    const uint32_t v = lane < (uint32_t)NW ? sh.warp_sum[lane] : 0u;
    uint32_t sc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= (uint32_t)o) sc += t;
    }
    wpre = __shfl_sync(0xffffffffu, sc - v, w);
  }
  uint32_t before = incl - local + wpre;
  if (before < need && need <= before + local) {
    uint32_t run = before;
    for (int i = i0; i < i0 + per && i < nbins; ++i) {
      const int b = from_top ? nbins - 1 - i : i;
      const uint32_t h = hist[b];
      if (run + h >= need) {
        sh.found_bin = (uint32_t)b;
        sh.found_beyond = run;
        break;
      }
      run += h;
    }
  }
  named_bar_sync(bar_id, NT);
  if (sh.found_bin != kNotFound) return true;
  named_bar_sync(bar_id, NT);   // every thread has seen the miss before it is cleared
  if (tid == 0) sh.found_bin = 0u;
  named_bar_sync(bar_id, NT);
  return false;
}

// Refine a cut-off inside [lo, hi] (need >= 1 entries to take there, entries
// above hi already counted).  `get(i, key, pos)` reads entry i < m.
// `hist` is NBINS uint32 of shared scratch owned by the group.
template <int NT, int NBINS, typename Get>
__device__ SelectResult group_refine(Get get, int m, uint32_t lo, uint32_t hi, uint32_t need, uint32_t pos_max,
                                     uint32_t* hist, SelectShared<NT>& sh, uint32_t tid, uint32_t bar_id,
                                     DeviceStatus* status) {
  SelectResult r;
  r.key_all_in = 0;
  r.pos_hi = 0;
  bool done = false;
  while (!done && lo < hi) {
    int s = 0;
    while (((hi >> s) - (lo >> s)) >= (uint32_t)NBINS) ++s;
    const uint32_t base = lo >> s;
    const int nb = (int)((hi >> s) - base) + 1;
    for (int i = (int)tid; i < nb; i += NT) hist[i] = 0u;
    named_bar_sync(bar_id, NT);
    for (int i0 = (int)tid; i0 < m; i0 += NT * kBatch) {
      uint32_t key[kBatch], pos[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        key[u] = 0u;
        pos[u] = 0u;
        if (i0 + u * NT < m) get(i0 + u * NT, key[u], pos[u]);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (i0 + u * NT < m && key[u] >= lo && key[u] <= hi) atomicAdd(&hist[(key[u] >> s) - base], 1u);
    }
    named_bar_sync(bar_id, NT);
    if (!group_find<NT>(hist, nb, need, true, sh, tid, bar_id)) {
      if (tid == 0) report_status(status, kStatusDeviceCheck, 0x5e1ec8u);
      r.lo = lo;
      r.hi = hi;
      r.key_all_in = 1;
      return r;
    }
    const uint32_t d = sh.found_bin;
    const uint32_t cnt = hist[d];
    need -= sh.found_beyond;
    const uint64_t nlo = (uint64_t)(base + d) << s;
    const uint64_t nhi = (((uint64_t)(base + d) + 1) << s) - 1;
    lo = nlo > lo ? (uint32_t)nlo : lo;
    hi = nhi < hi ? (uint32_t)nhi : hi;
    if (need == cnt) done = true;
    named_bar_sync(bar_id, NT);
  }
  r.lo = lo;
  r.hi = hi;
  if (done) {
    r.key_all_in = 1;
    return r;
  }
  // One key (lo == hi) holds more entries than needed: take the lowest positions.
  uint32_t plo = 0, phi = pos_max;
  bool pdone = false;
  while (!pdone) {
    int s = 0;
    while (((phi >> s) - (plo >> s)) >= (uint32_t)NBINS) ++s;
    const uint32_t base = plo >> s;
    const int nb = (int)((phi >> s) - base) + 1;
    for (int i = (int)tid; i < nb; i += NT) hist[i] = 0u;
    named_bar_sync(bar_id, NT);
    for (int i0 = (int)tid; i0 < m; i0 += NT * kBatch) {
      uint32_t key[kBatch], pos[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        key[u] = 0u;
        pos[u] = 0u;
        if (i0 + u * NT < m) get(i0 + u * NT, key[u], pos[u]);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (i0 + u * NT < m && key[u] == lo && pos[u] >= plo && pos[u] <= phi)
          atomicAdd(&hist[(pos[u] >> s) - base], 1u);
    }
    named_bar_sync(bar_id, NT);
    if (!group_find<NT>(hist, nb, need, false, sh, tid, bar_id)) {
      if (tid == 0) report_status(status, kStatusDeviceCheck, 0x5e1ec9u);
      break;
    }
    const uint32_t d = sh.found_bin;
    const uint32_t cnt = hist[d];
    need -= sh.found_beyond;
    const uint64_t nlo = (uint64_t)(base + d) << s;
    const uint64_t nhi = (((uint64_t)(base + d) + 1) << s) - 1;
    plo = nlo > plo ? (uint32_t)nlo : plo;
    phi = nhi < phi ? (uint32_t)nhi : phi;
    if (need == cnt) pdone = true;
    named_bar_sync(bar_id, NT);
  }
  r.pos_hi = phi;
  return r;
}

__device__ __forceinline__ bool selected(const SelectResult& r, uint32_t key, uint32_t pos) {
  if (key > r.hi) return true;
  if (key < r.lo) return false;
  return r.key_all_in || pos <= r.pos_hi;
}

// Write the selected entries (exactly kk of them) to idx_row[0..kk) in
// unspecified order, scores too if score_row != nullptr, then pad [kk, k)
// with -1 / -inf.  Output slots come from a group-wide scan of the per-warp
// counts of each batch (two barriers a batch, no shared atomics).
template <int NT, typename Get>
__device__ void group_emit(Get get, int m, const SelectResult& r, int kk, int k, int32_t* idx_row,
                           float* score_row, SelectShared<NT>& sh, uint32_t tid, uint32_t bar_id,
                           DeviceStatus* status) {
  constexpr int NW = NT / 32;
  const uint32_t lane = tid & 31u, w = tid >> 5;
  uint32_t run = 0;
  for (int j0 = 0; j0 < m; j0 += NT * kBatch) {
    uint32_t key[kBatch], pos[kBatch];
    uint32_t n = 0;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      key[u] = 0u;
      pos[u] = 0u;
      const int i = j0 + u * NT + (int)tid;
      if (i < m) get(i, key[u], pos[u]);
      n += (i < m && selected(r, key[u], pos[u])) ? 1u : 0u;
    }
    uint32_t incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= (uint32_t)o) incl += t;
    }
    if (lane == 31) sh.warp_sum[w] = incl;
    named_bar_sync(bar_id, NT);
    const uint32_t tw = lane < (uint32_t)NW ? sh.warp_sum[lane] : 0u;
    uint32_t sc = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= (uint32_t)o) sc += t;
    }
    uint32_t slot = run + __shfl_sync(0xffffffffu, sc - tw, w) + incl - n;
    run += __shfl_sync(0xffffffffu, sc, 31);
    named_bar_sync(bar_id, NT);   // warp_sum is free for the next batch
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * NT + (int)tid;
      if (i < m && selected(r, key[u], pos[u])) {
        if (slot < (uint32_t)kk) {
          idx_row[slot] = (int32_t)pos[u];
          if (score_row) score_row[slot] = key_to_float(key[u]);
        }
        ++slot;
      }
    }
  }
  // A selection that does not produce exactly kk entries is a library bug:
  // report it and leave no stale slot behind.
  const int got = (int)run;
  if (got != kk && tid == 0) report_status(status, kStatusDeviceCheck, 0x5e1ec7u);
  for (int j = (got < kk ? got : kk) + (int)tid; j < k; j += NT) {
    idx_row[j] = -1;
    if (score_row) score_row[j] = -__int_as_float(0x7f800000);
  }
  named_bar_sync(bar_id, NT);
}

// Append the selected entries with keys in [key_lo, key_hi] among entries
// [0, m) to idx_row / score_row at slots counted on from sh.out_count (which
// the caller has set and made visible with a barrier); no padding.  Slots
// come from a group-wide scan of the per-warp counts of each batch.
template <int NT, typename Get>
__device__ void group_emit_append(Get get, int m, const SelectResult& r, uint32_t key_lo, uint32_t key_hi, int kk,
                                  int32_t* idx_row, float* score_row, SelectShared<NT>& sh, uint32_t tid,
                                  uint32_t bar_id) {
  constexpr int NW = NT / 32;
  const uint32_t lane = tid & 31u, w = tid >> 5;
  uint32_t run = sh.out_count;
  for (int j0 = 0; j0 < m; j0 += NT * kBatch) {
    uint32_t key[kBatch], pos[kBatch];
    uint32_t n = 0;
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      key[u] = 0u;
      pos[u] = 0u;
      const int i = j0 + u * NT + (int)tid;
      if (i < m) get(i, key[u], pos[u]);
      n += (i < m && key[u] >= key_lo && key[u] <= key_hi && selected(r, key[u], pos[u])) ? 1u : 0u;
    }
    uint32_t incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= (uint32_t)o) incl += t;
    }
    if (lane == 31) sh.warp_sum[w] = incl;
    named_bar_sync(bar_id, NT);
    const uint32_t tw = lane < (uint32_t)NW ? sh.warp_sum[lane] : 0u;
    uint32_t sc = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= (uint32_t)o) sc += t;
    }
    uint32_t slot = run + __shfl_sync(0xffffffffu, sc - tw, w) + incl - n;
    run += __shfl_sync(0xffffffffu, sc, 31);
    named_bar_sync(bar_id, NT);   // warp_sum is free for the next batch
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = j0 + u * NT + (int)tid;
      if (i < m && key[u] >= key_lo && key[u] <= key_hi && selected(r, key[u], pos[u])) {
        if (slot < (uint32_t)kk) {
          idx_row[slot] = (int32_t)pos[u];
          if (score_row) score_row[slot] = key_to_float(key[u]);
        }
        ++slot;
      }
    }
  }
  named_bar_sync(bar_id, NT);   // every thread has read out_count
  if (tid == 0) sh.out_count = run;
  named_bar_sync(bar_id, NT);
}

// Check the emitted count (report a mismatch) and pad slots [count, k) with
// -1 / -inf.
template <int NT>
__device__ void group_emit_finish(int kk, int k, int32_t* idx_row, float* score_row, SelectShared<NT>& sh,
                                  uint32_t tid, uint32_t bar_id, DeviceStatus* status) {
  const int got = (int)sh.out_count;
  if (got != kk && tid == 0) report_status(status, kStatusDeviceCheck, 0x5e1ec7u);
  for (int j = (got < kk ? got : kk) + (int)tid; j < k; j += NT) {
    idx_row[j] = -1;
    if (score_row) score_row[j] = -__int_as_float(0x7f800000);
  }
  named_bar_sync(bar_id, NT);
}

}  // namespace dsa
