// latent_attn_dense.cu -- eq. (3) of page "2.2.1 · DSA 与索引器" computed over
// dense key tiles with a mask: the "masked MHA" way of running DSA that §2
// recommends for short prefill, where top-k, index materialisation and the
// irregular gather cost more than the attention they save.  Every query row
// sees the causal keys s <= t; a row with t + 1 > k additionally sees only
// its selected positions (a bitmask built from the index tensor), so the
// result is eq. (3) on the same selection.  Without an index tensor it is
// plain causal attention over the whole history, whose log-sum-exp gives the
// teacher mass coverage of eq. (15) (M_k = exp(lse_sparse - lse_dense) per
// head).
//
// Shape served here: 16 query heads sharing one latent row of 576 columns
// per position (key; the first 512 columns are the value).  A block of 8
// consecutive tokens x 16 heads = 128 rows sits on the tcgen05 M (TMEM
// lanes), so every key tile loaded from HBM/L2 feeds 8 tokens.  As in the
// decode kernel the output O = 128 x 512 fp32 would fill a CTA's TMEM, so a
// cluster of two CTAs splits the latent columns: CTA r keeps value columns
// [256r, 256r + 256) and rope columns [512 + 32r, +32), forms partial logits
// over them, and the two partials are exchanged through distributed shared
// memory and added, so both CTAs take identical softmax decisions and each
// accumulates its half of O.  The exchange is one 16 KB TMA bulk copy per
// warpgroup and tile from a local staging buffer into the other CTA's
// (double-buffered) receive buffer, counted by its mbarrier: per-thread
// 16-byte remote stores moved only about 8 bytes per clock and slowed the
// MMAs' shared-memory reads.  Key tiles of 64 positions arrive by TMA 2-D
// tile loads straight into the 128-byte swizzled layout (two stages).
//
// Warps: 0-7 softmax and output (warpgroup g: keys 32g..32g+31 of a tile,
// output columns 128g..128g+127; thread h owns row h = TMEM lane h), 8 issues
// the logits MMAs and owns TMEM, 9 issues P V, 10 issues the TMA loads.
// Blocks with the longest causal history are scheduled first.
#include "kernels.h"
#include "latent_attn.cuh"
#include "sm100.cuh"

namespace dsa {

namespace {

using lattn::pack_bf16x2;
using lattn::swz_off;

constexpr int kRows = 128;             // MMA M: kTok tokens x kH heads
constexpr int kH = 16;
constexpr int kTok = kRows / kH;       // 8
constexpr int kDqk = 576, kDv = 512;
constexpr int kTile = 64;              // keys per tile: N of the logits, K of P V
constexpr int kStages = 2;
constexpr int kSlotBytes = kTile * 128;
constexpr int kStageBytes = 5 * kSlotBytes;              // 4 value blocks + the rope block
constexpr int kPBytes = kRows * kTile * 2;
constexpr int kXHalf = kRows * 32 * 4;                   // one warpgroup's partial logits (16 KB)
constexpr int kXBytes = 2 * kXHalf;
constexpr uint32_t kXTx = kXBytes;
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 8, kPvWarp = 9, kTmaWarp = 10;
constexpr int kThreads = 11 * 32;
constexpr uint32_t kBarSoft = 2;                          // all softmax warps
constexpr uint32_t kBarHalf0 = 3;                         // + g: the softmax warps of warpgroup g

constexpr uint32_t kTmemO = 0;
constexpr uint32_t kTmemQ = 256;
constexpr uint32_t kTmemS = 448;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = instr_desc(1u, 128u, 64u);
constexpr uint32_t kIdescPV = instr_desc_bf16_bmn(128u, 256u);
constexpr float kRescaleThreshold = 8.0f;

struct Smem {
  uint8_t* stage;      // kStages x kStageBytes, 1024-aligned
  uint8_t* pbuf;       // 2 x kPBytes
  uint8_t* x;          // 2 x kXBytes: the other CTA's partial logits of tiles i % 2
  uint8_t* xs;         // kXBytes: this CTA's partial logits, staged for the copy
  float* tmax;         // 2 x 2 x kRows
  float* lsum;         // kRows
  uint64_t* full;      // kStages
  uint64_t* empty;     // kStages
  uint64_t* s_full;
  uint64_t* s_empty;
  uint64_t* p_full;    // 2
  uint64_t* o_done;    // 2
  uint64_t* x_full;    // 2
  uint64_t* drain;     // 2
  uint32_t* tmem_slot;
  volatile uint32_t* abort_flag;
};

constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 2;

__host__ __device__ constexpr size_t smem_bytes() {
  return 1024 + (size_t)kStages * kStageBytes + 2 * kPBytes + 3 * kXBytes + 5 * kRows * 4 + kNumBars * 8 + 64;
}

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.stage = p;
  p += kStages * kStageBytes;
  s.pbuf = p;
  p += 2 * kPBytes;
  s.x = p;
  p += 2 * kXBytes;
  s.xs = p;
  p += kXBytes;
  s.tmax = reinterpret_cast<float*>(p);
  p += 4 * kRows * 4;
  s.lsum = reinterpret_cast<float*>(p);
  p += kRows * 4;
  uint64_t* b = reinterpret_cast<uint64_t*>(p);
  s.full = b;
  b += kStages;
  s.empty = b;
  b += kStages;
  s.s_full = b++;
  s.s_empty = b++;
  s.p_full = b;
  b += 2;
  s.o_done = b;
  b += 2;
  s.x_full = b;
  b += 2;
  s.drain = b;
  b += 2;
  uint32_t* w = reinterpret_cast<uint32_t*>(b);
  s.tmem_slot = w;
  s.abort_flag = w + 1;
  return s;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    latent_attn_dense_kernel(const __grid_constant__ CUtensorMap tmap_lat, const DenseAttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const uint32_t warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  // cluster c -> (sequence, 8-token block), longest histories first
  const int c = (int)(blockIdx.x >> 1);
  const int b = c % a.B;
  const int tb = a.nblk - 1 - c / a.B;
  const int i0 = tb * kTok;
  const int ntok = min(kTok, a.nq - i0);
  const int t_last = a.q_offset + i0 + ntok - 1;
  const int T = t_last / kTile + 1;                  // key tiles 0 .. T-1 hold every causal key
  const int64_t key_row0 = (int64_t)b * a.kv_len;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(sm.s_full, 1);
    mbar_init(sm.s_empty, kSoftWarps);
    for (int j = 0; j < 2; ++j) {
      mbar_init(&sm.p_full[j], kSoftWarps);
      mbar_init(&sm.o_done[j], 1);
      mbar_init(&sm.x_full[j], 1);
      mbar_init(&sm.drain[j], 1);
    }
    *sm.abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kTmaWarp && lane == 0) tma_prefetch_desc(&tmap_lat);
  if (warp == kMmaWarp) {
    tmem_alloc(sm.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  const WaitCtl ctl{sm.abort_flag, a.timeout_ns, a.status};

  if (warp < 4) {
    // this CTA's query columns of the block's 128 rows into TMEM; rows past
    // the chunk's end repeat its first row (their outputs are not written)
    const uint32_t lrow = (warp & 3u) * 32u;
    const int tok = (int)(tid / kH) < ntok ? (int)(tid / kH) : 0;
    const uint16_t* qrow = a.q + (((int64_t)b * a.nq + i0 + tok) * kH + (tid % kH)) * kDqk;
    const uint4* qv = reinterpret_cast<const uint4*>(qrow + 256 * rank);
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = __ldg(qv + cc * 8 + j);
        r[4 * j] = v.x;
        r[4 * j + 1] = v.y;
        r[4 * j + 2] = v.z;
        r[4 * j + 3] = v.w;
      }
      tmem_st_32x32b_x32(tmem + (lrow << 16) + kTmemQ + 32 * cc, r);
    }
    {
      const uint4* qr = reinterpret_cast<const uint4*>(qrow + 512 + 32 * rank);
      uint32_t r[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = __ldg(qr + j);
        r[4 * j] = v.x;
        r[4 * j + 1] = v.y;
        r[4 * j + 2] = v.z;
        r[4 * j + 3] = v.w;
      }
      tmem_st_32x32b_x16(tmem + (lrow << 16) + kTmemQ + 128, r);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();

  if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax + output
    const uint32_t g = warp >> 2;
    const uint32_t h = tid & 127u;                 // row = token h / 16, head h % 16
    const uint32_t lrow = (warp & 3u) * 32u;
    const int my_tok = (int)(h / kH);
    const bool row_live = my_tok < ntok;
    const int i_row = i0 + (row_live ? my_tok : 0);
    const int t = a.q_offset + i_row;               // absolute position of the row's token
    const bool use_sel = a.sel_bits != nullptr && t + 1 > a.k;
    const uint64_t* sel = use_sel ? a.sel_bits + ((int64_t)b * a.nq + i_row) * a.kv_tiles : nullptr;
    // row h of a warpgroup's 16 KB block of partial logits: 128 bytes, its
    // 16-byte chunks XOR-swizzled by h so that 8 rows cover every bank
    const uint32_t x_row = g * (uint32_t)kXHalf + h * 128u;
    const uint32_t x_peer0 = map_to_cta(smem_u32(sm.x + g * kXHalf), peer);
    const uint32_t xfull_peer0 = map_to_cta(smem_u32(&sm.x_full[0]), peer);
    const bool leader = (tid & 127u) == 0u;       // issues its warpgroup's copy
    const float cs = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      const uint32_t xs = (uint32_t)i & 1u;
      if (tid == 0) mbar_arrive_expect_tx(&sm.x_full[xs], kXTx);
      // the row's valid keys in this half tile: causal, then the selection
      const int kb = i * kTile + 32 * (int)g;
      uint32_t mk = 0u;
      if (row_live) {
        const int lim = t - kb;                     // keys kb .. kb + lim are causal
        mk = lim >= 31 ? 0xffffffffu : (lim < 0 ? 0u : (0xffffffffu >> (31 - lim)));
        if (use_sel) mk &= (uint32_t)(__ldg(sel + i) >> (32 * g));
      }
      float s[32];
      ok = ok && mbar_wait(sm.s_full, (uint32_t)i & 1u, ctl, 0x2501);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + (lrow << 16) + kTmemS + 32u * g, r);
        tmem_wait_ld(r);
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = __uint_as_float(r[j]);
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.s_empty);
      // stage this warpgroup's partial logits (after its previous copy has
      // read the staging buffer), then one bulk copy into the other CTA
      if (leader) bulk_wait_read_all();
      named_bar_sync(kBarHalf0 + g, 128);
      if (ok) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(sm.xs + x_row + ((j ^ (h & 7u)) << 4)) =
              make_float4(s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
        fence_proxy_async_smem();
      }
      named_bar_sync(kBarHalf0 + g, 128);
      if (leader && ok) {
        bulk_s2cluster(x_peer0 + xs * kXBytes, smem_u32(sm.xs + g * kXHalf), kXHalf, xfull_peer0 + xs * 8u);
        bulk_commit_group();
      }
      ok = ok && mbar_wait_cluster(&sm.x_full[xs], (uint32_t)(i >> 1) & 1u, ctl, 0x2502);
      if (ok) {
        const uint8_t* xr = sm.x + xs * kXBytes + x_row;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = *reinterpret_cast<const float4*>(xr + ((j ^ (h & 7u)) << 4));
          s[4 * j] += v.x;
          s[4 * j + 1] += v.y;
          s[4 * j + 2] += v.z;
          s[4 * j + 3] += v.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 z = ffma2(make_float2(s[2 * j], s[2 * j + 1]), make_float2(cs, cs), make_float2(0.0f, 0.0f));
        s[2 * j] = z.x;
        s[2 * j + 1] = z.y;
      }
      float mt = -INFINITY;
      if (mk == 0xffffffffu) {
#pragma unroll
        for (int j = 0; j < 32; ++j) mt = fmaxf(mt, s[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          s[j] = ((mk >> j) & 1u) ? s[j] : -INFINITY;
          mt = fmaxf(mt, s[j]);
        }
      }
      float* tm = sm.tmax + ((uint32_t)i & 1u) * 2 * kRows;
      tm[g * kRows + h] = mt;
      named_bar_sync(kBarSoft, kSoftWarps * 32);
      mt = fmaxf(mt, tm[(g ^ 1u) * kRows + h]);
      float alpha = 1.0f;
      bool rescale = false;
      if (mt > m_run + kRescaleThreshold) {
        if (m_run != -INFINITY) {
          alpha = ex2_approx(m_run - mt);
          rescale = true;
        }
        m_run = mt;
      }
      const float msub = (m_run == -INFINITY) ? 0.0f : m_run;
      uint32_t p[16];
      float2 lsum = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 z = ffma2(make_float2(s[2 * j], s[2 * j + 1]), make_float2(1.0f, 1.0f), make_float2(-msub, -msub));
        const float2 e = make_float2(ex2_approx(z.x), ex2_approx(z.y));
        p[j] = pack_bf16x2(e.x, e.y);
        // the denominator sums the unrounded probabilities (its log is the lse)
        lsum = ffma2(e, make_float2(1.0f, 1.0f), lsum);
      }
      l_run = l_run * alpha + (lsum.x + lsum.y);
      const uint32_t pb = (uint32_t)i & 1u;
      if (i >= 2) ok = ok && mbar_wait(&sm.o_done[pb], (uint32_t)((i - 2) >> 1) & 1u, ctl, 0x2503);
      const bool any_rescale = __any_sync(0xffffffffu, rescale);
      if (any_rescale && i >= 1)
        ok = ok && mbar_wait(&sm.o_done[pb ^ 1u], (uint32_t)((i - 1) >> 1) & 1u, ctl, 0x2504);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        if (any_rescale) {
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t o[32];
            const uint32_t col = kTmemO + 128u * g + 32u * cc;
            tmem_ld_32x32b_x32(tmem + (lrow << 16) + col, o);
            tmem_wait_ld(o);
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
            tmem_st_32x32b_x32(tmem + (lrow << 16) + col, o);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        uint8_t* pbase = sm.pbuf + pb * kPBytes;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(pbase + swz_off(h, 4u * g + (uint32_t)j)) =
              make_uint4(p[4 * j], p[4 * j + 1], p[4 * j + 2], p[4 * j + 3]);
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[pb]);
    }
    if (leader) bulk_wait_read_all();
    if (g == 1) sm.lsum[h] = l_run;
    named_bar_sync(kBarSoft, kSoftWarps * 32);
    if (g == 0) sm.lsum[h] += l_run;
    named_bar_sync(kBarSoft, kSoftWarps * 32);
    const float l_tot = sm.lsum[h];
    ok = ok && mbar_wait(&sm.o_done[(T - 1) & 1], (uint32_t)((T - 1) >> 1) & 1u, ctl, 0x2505);
    ok = __all_sync(0xffffffffu, ok);
    const float inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
    const int64_t orow_idx = ((int64_t)b * a.nq + i_row) * kH + (h % kH);
    uint16_t* orow = a.out + orow_idx * kDv + 256 * rank + 128 * g;
    if (ok) tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t o[32];
      if (ok) {
        tmem_ld_32x32b_x32(tmem + (lrow << 16) + kTmemO + 128u * g + 32u * cc, o);
        tmem_wait_ld(o);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
      if (row_live) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * j]) * inv_l, __uint_as_float(o[8 * j + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * j + 2]) * inv_l, __uint_as_float(o[8 * j + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * j + 4]) * inv_l, __uint_as_float(o[8 * j + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * j + 6]) * inv_l, __uint_as_float(o[8 * j + 7]) * inv_l);
          dst[j] = v;
        }
      }
    }
    if (row_live && rank == 0 && g == 0 && a.lse != nullptr)
      a.lse[orow_idx] = l_tot > 0.0f ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ logits issuer
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < T && ok; ++i) {
        ok = mbar_wait(&sm.full[i % kStages], (uint32_t)(i / kStages) & 1u, ctl, 0x2511);
        if (ok && i >= 1) ok = mbar_wait(sm.s_empty, (uint32_t)(i - 1) & 1u, ctl, 0x2512);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sbase = smem_u32(sm.stage + (i % kStages) * kStageBytes);
#pragma unroll
        for (int k = 0; k < 18; ++k) {
          const uint32_t a_col = k < 16 ? 8u * k : 128u + 8u * (k - 16);
          const uint32_t slot = k < 16 ? (uint32_t)k / 4u : 4u;
          const uint32_t koff = k < 16 ? 32u * (k % 4) : 64u * rank + 32u * (k - 16);
          mma_bf16_ts(tmem + kTmemS, tmem + kTmemQ + a_col, smem_desc_sw128(sbase + slot * kSlotBytes + koff),
                      kIdescS, k > 0 ? 1u : 0u);
        }
        tc_commit(sm.s_full);
      }
      tc_commit(&sm.drain[0]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&sm.drain[0]), 0u) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ P V issuer
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < T && ok; ++i) {
        const uint32_t pb = (uint32_t)i & 1u;
        if (!(ok = mbar_wait(&sm.p_full[pb], (uint32_t)(i >> 1) & 1u, ctl, 0x2513))) break;
        tc_fence_after();
        const uint32_t sbase = smem_u32(sm.stage + (i % kStages) * kStageBytes);
        const uint32_t pbase = smem_u32(sm.pbuf + pb * kPBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss(tmem + kTmemO, smem_desc_sw128(pbase + 32u * k), smem_desc_sw128_mn(sbase + 2048u * k, kSlotBytes),
                      kIdescPV, (i > 0 || k > 0) ? 1u : 0u);
        tc_commit(&sm.o_done[pb]);
        tc_commit(&sm.empty[i % kStages]);
      }
      tc_commit(&sm.drain[1]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&sm.drain[1]), 0u) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ TMA loads of the key tiles
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int i = 0; i < T; ++i) {
        const int st = i % kStages;
        if (!(ok = mbar_wait(&sm.empty[st], ((uint32_t)(i / kStages) & 1u) ^ 1u, ctl, 0x2521))) break;
        mbar_arrive_expect_tx(&sm.full[st], (uint32_t)kStageBytes);
        uint8_t* dst = sm.stage + st * kStageBytes;
        const int y = (int)(key_row0 + (int64_t)i * kTile);
#pragma unroll
        for (int j = 0; j < 4; ++j) tma_load_2d(dst + j * kSlotBytes, &tmap_lat, &sm.full[st], (4 * (int)rank + j) * 64, y);
        tma_load_2d(dst + 4 * kSlotBytes, &tmap_lat, &sm.full[st], 512, y);
        issued = i + 1;
      }
      if (!ok) {   // let the loads in flight land before the CTA exits
        const uint64_t t0 = globaltimer_ns();
        for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
          while (!mbar_try_wait(smem_u32(&sm.full[i % kStages]), (uint32_t)(i / kStages) & 1u) &&
                 globaltimer_ns() - t0 < a.timeout_ns) {
          }
      }
    }
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync_all();
}

// Selection bitmask of the rows that need one (t + 1 > k): bit s of word
// [b, i, s / 64] is set when row i selected position s.  Indices outside
// [-1, kv_len) are skipped and reported.
__global__ void selection_bits_kernel(int B, int nq, int q_offset, int kv_len, int k, int kv_tiles, int i0,
                                      const int32_t* __restrict__ idx, unsigned long long* __restrict__ bits,
                                      DeviceStatus* status) {
  // rows i0 .. nq-1 of each sequence (the first rows with t + 1 > k)
  const int per_seq = nq - i0;
  const int64_t total = (int64_t)B * per_seq * k;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t rr = e / k;
    const int b = (int)(rr / per_seq);
    const int64_t row = (int64_t)b * nq + i0 + (rr - (int64_t)b * per_seq);
    const int p = idx[row * k + (e - rr * k)];
    if (p == -1) continue;
    if (p < 0 || p >= kv_len) {
      report_status(status, kStatusDeviceCheck, 0xA77E);
      continue;
    }
    atomicOr(bits + row * kv_tiles + (p >> 6), 1ull << (p & 63));
  }
}

// Teacher mass coverage per row (eq. (15)): a head's dense probabilities
// on the selection sum to exp(lse_sparse - lse_dense); the aggregate teacher
// (heads summed, L1-normalised) covers their mean.
__global__ void mass_coverage_kernel(int rows, int H, const float* __restrict__ lse_s, const float* __restrict__ lse_d,
                                     float* __restrict__ m_out, float* __restrict__ per_head, float* __restrict__ mn) {
  for (int r = blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += gridDim.x * blockDim.x) {
    float sum = 0.0f, lo = INFINITY;
    for (int h = 0; h < H; ++h) {
      const float ls = lse_s[(int64_t)r * H + h], ld = lse_d[(int64_t)r * H + h];
      const float m = ls == -INFINITY ? 0.0f : expf(ls - ld);
      if (per_head != nullptr) per_head[(int64_t)r * H + h] = m;
      sum += m;
      lo = fminf(lo, m);
    }
    if (m_out != nullptr) m_out[r] = sum / (float)H;
    if (mn != nullptr) mn[r] = lo;
  }
}

cudaError_t launch_mass_coverage(int rows, int H, const float* lse_sparse, const float* lse_dense, float* m_out,
                                 float* per_head_out, float* min_out, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int grid = (rows + 255) / 256 < 1184 ? (rows + 255) / 256 : 1184;
  mass_coverage_kernel<<<grid, 256, 0, stream>>>(rows, H, lse_sparse, lse_dense, m_out, per_head_out, min_out);
  return cudaGetLastError();
}

size_t latent_attn_dense_smem() { return smem_bytes(); }

cudaError_t launch_latent_attn_dense(const CUtensorMap& tmap_lat, const DenseAttnArgs& a, const int32_t* idx,
                                     cudaStream_t stream) {
  if (a.sel_bits != nullptr) {
    // only rows with t + 1 > k read a selection: i >= k - q_offset
    const int i0 = a.k - a.q_offset > 0 ? a.k - a.q_offset : 0;
    cudaError_t e = cudaMemsetAsync(const_cast<uint64_t*>(a.sel_bits), 0,
                                    (size_t)a.B * a.nq * a.kv_tiles * sizeof(uint64_t), stream);
    if (e != cudaSuccess) return e;
    const int64_t total = (int64_t)a.B * (a.nq - i0) * a.k;
    const int grid = (int)((total + 255) / 256 < 4096 ? (total + 255) / 256 : 4096);
    selection_bits_kernel<<<grid, 256, 0, stream>>>(a.B, a.nq, a.q_offset, a.kv_len, a.k, a.kv_tiles, i0, idx,
                                                    reinterpret_cast<unsigned long long*>(const_cast<uint64_t*>(a.sel_bits)),
                                                    a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = smem_bytes();
  cudaError_t e = setup_once_per_device([smem]() {
    return cudaFuncSetAttribute(latent_attn_dense_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * (unsigned)(a.B * a.nblk), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, latent_attn_dense_kernel, tmap_lat, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dsa
