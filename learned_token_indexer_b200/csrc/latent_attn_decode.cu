// latent_attn_decode.cu -- eq. (3) of page "2.2.1 · DSA 与索引器" for a decode
// step, in the MQA form of its §2: every query head of a sequence attends the
// same selected rows of that sequence's latent cache, with its own logits
// and softmax.  Shape served here: 128 query heads, latent rows of 576
// columns (the key), whose first 512 columns are the value.
//
// Engine: tcgen05 with the 128 heads on the MMA's M (TMEM lanes), so one
// gathered latent row feeds every head.  The output block O = 128 x 512 fp32
// alone would fill a CTA's 512 TMEM columns, so each sequence is served by a
// cluster of two CTAs that split the latent columns, not the work:
//   CTA r holds value columns [256r, 256r + 256) and rope columns
//   [512 + 32r, 512 + 32r + 32) of each selected row and of the queries.
//   Per tile of 64 selected rows it forms the partial logits over its own
//   columns, S_r = Q_r C_r^T (M 128 x N 64, K 288), sends them to the other
//   CTA (one 16 KB TMA bulk copy per warpgroup from a local staging buffer,
//   counted by the receiver's mbarrier) and adds the partial it receives,
//   so both CTAs hold the same full logits
//   S = S_0 + S_1 (the same fp32 sum on both sides), take the same softmax
//   decisions, and accumulate O_r += P C_r[:, value]  (M 128 x N 256, K 64)
//   for their own half of the value columns.  No row is gathered twice and no
//   product is computed twice.
//
// Gather: the selected rows sit in HBM in random order.  Each row's 512-byte
// value half arrives with one TMA bulk copy (the copy engine keeps enough
// bytes in flight for HBM latency; 16-byte cp.async per thread does not) in
// a row-major staging ring; eight warps then move it, 16 bytes per thread,
// into the 128-byte swizzled layout the MMA reads.  That tile is the K-major
// B operand of the logits (rows = keys) and the MN-major B operand of P V
// (rows = keys = the reduction dimension).  The 64-byte rope part goes
// straight to its swizzled place with cp.async.
//
// Warps: 0-7 softmax and output (warpgroup g handles keys 32g..32g+31 of
// every tile and value columns 128g..128g+127 of the output; thread h of a
// warpgroup owns head h = TMEM lane h); 8 issues the logits MMAs and owns
// TMEM; 9 issues P V; 10 issues the bulk copies; 11 the rope copies and the
// slot mask; 12-19 convert staged rows.  Registers move to the softmax warps
// with setmaxnreg.  The queries and P live in TMEM (the A operands of the
// logits and of P V).  Online softmax in base 2
// with a lazy reference maximum: O and l are rescaled only when a tile's
// maximum exceeds the reference by more than 2^8.
#include <cuda_bf16.h>

#include "kernels.h"
#include "latent_attn.cuh"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kHeads = 128;            // MMA M
constexpr int kDqk = 576, kDv = 512;
constexpr int kTile = 64;              // selected rows per tile: N of the logits, K of P V
constexpr int kSwz = 2;                // swizzled operand tiles
constexpr int kRaw = 2;                // row-major staging tiles
constexpr int kSlotBytes = kTile * 128;                  // one 64-column block of a tile (8 KB)
constexpr int kSwzBytes = 5 * kSlotBytes;                // 4 value blocks + the rope block
constexpr int kRowBytes = 512;                           // a row's value half for this CTA
constexpr int kRawBytes = kTile * kRowBytes;
constexpr int kXHalf = kHeads * 32 * 4;                  // one warpgroup's partial logits (16 KB)
constexpr int kXBytes = 2 * kXHalf;
constexpr uint32_t kXTx = kXBytes;                       // bytes the other CTA sends per tile
constexpr int kSoftWarps = 8;
constexpr int kMmaWarp = 8;                               // logits issuer, TMEM owner
constexpr int kPvWarp = 9;                                // P V issuer
constexpr int kFetchWarp = 10;                            // bulk copies of the value halves
constexpr int kRopeWarp = 11;                             // rope copies, slot mask, index checks
constexpr int kConvWarp0 = 12;
constexpr int kConv = 256;                                // warps 12-19
constexpr int kThreads = kConvWarp0 * 32 + kConv;        // 640
constexpr int kChunksPerConv = kTile * (kRowBytes / 16) / kConv;   // 8
static_assert(kTile * (kRowBytes / 16) % kConv == 0, "staged chunks must split evenly");
// register split: the launch gives every thread kLaunchRegs; the softmax
// warpgroups take kRegsSoft, the three others kRegsOther (sums must match,
// or the increase would wait forever)
constexpr int kLaunchRegs = 96;
constexpr int kRegsSoft = 168, kRegsOther = 48;
static_assert(2 * kRegsSoft + 3 * kRegsOther == 5 * kLaunchRegs, "register split must match the launch");
constexpr uint32_t kBarSoft = 2;                          // named barrier of the softmax warps
constexpr uint32_t kBarHalf0 = 3;                         // + g: the softmax warps of warpgroup g

// TMEM columns (512 allocated)
constexpr uint32_t kTmemO = 0;       // 256 fp32: O for this CTA's value columns
constexpr uint32_t kTmemQ = 256;     // 144: queries, bf16 pairs (128 value + 16 rope)
constexpr uint32_t kTmemP = 416;     // 32: P, bf16 pairs (A operand of P V)
constexpr uint32_t kTmemS = 448;     // 64 fp32: partial logits
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = instr_desc(1u, 128u, 64u);          // K-major x K-major, M 128, N 64
constexpr uint32_t kIdescPV = instr_desc_bf16_bmn(128u, 256u);   // A (TMEM), B MN-major, M 128, N 256
constexpr float kRescaleThreshold = 8.0f;                         // log2 units

struct Smem {
  uint8_t* swz;        // kSwz x kSwzBytes, 1024-aligned
  uint8_t* raw;        // kRaw x kRawBytes: value halves, one 512-byte row per slot
  uint8_t* x;          // kXBytes: the other CTA's partial logits (two 16 KB warpgroup halves)
  uint8_t* xs;         // kXBytes: this CTA's partial logits, staged for the copy
  float* tmax;         // 2 x 2 x kHeads: each warpgroup's tile maximum per head (by tile parity)
  float* lsum;         // kHeads: warpgroup 1's softmax denominator at the end
  uint32_t* mask;      // kSwz x 2: valid slots of the tile
  uint64_t* swz_full;  // kSwz: converted value blocks + rope blocks + mask
  uint64_t* swz_empty; // kSwz: P V of the tile is done
  uint64_t* raw_full;  // kRaw: bulk copies landed
  uint64_t* raw_empty; // kRaw: converted
  uint64_t* s_full;
  uint64_t* s_empty;
  uint64_t* p_full;    // P of the tile is in TMEM
  uint64_t* o_done;    // P V of the tile is done
  uint64_t* x_full;    // the other CTA's partial for the tile is in x
  uint64_t* x_empty;   // the other CTA has read what this CTA wrote into it
  uint64_t* drain;     // 2: every MMA of the logits / P V issuer is done
  int* last_valid;
  uint32_t* tmem_slot;
  volatile uint32_t* abort_flag;
};

constexpr int kNumBars = 2 * kSwz + 2 * kRaw + 2 + 2 + 2 + 2 + 2;

__host__ __device__ constexpr size_t smem_bytes() {
  return 1024 + (size_t)kSwz * kSwzBytes + (size_t)kRaw * kRawBytes + 2 * kXBytes + 5 * kHeads * 4 +
         kSwz * 8 + kNumBars * 8 + 64;
}

__device__ __forceinline__ Smem carve(uint8_t* raw) {
  Smem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.swz = p;
  p += kSwz * kSwzBytes;
  s.raw = p;
  p += kRaw * kRawBytes;
  s.x = p;
  p += kXBytes;
  s.xs = p;
  p += kXBytes;
  s.tmax = reinterpret_cast<float*>(p);
  p += 4 * kHeads * 4;
  s.lsum = reinterpret_cast<float*>(p);
  p += kHeads * 4;
  s.mask = reinterpret_cast<uint32_t*>(p);
  p += kSwz * 8;
  uint64_t* b = reinterpret_cast<uint64_t*>(p);
  s.swz_full = b;
  b += kSwz;
  s.swz_empty = b;
  b += kSwz;
  s.raw_full = b;
  b += kRaw;
  s.raw_empty = b;
  b += kRaw;
  s.s_full = b++;
  s.s_empty = b++;
  s.p_full = b++;
  s.o_done = b++;
  s.x_full = b++;
  s.x_empty = b++;
  s.drain = b;
  b += 2;
  uint32_t* w = reinterpret_cast<uint32_t*>(b);
  s.last_valid = reinterpret_cast<int*>(w);
  s.tmem_slot = w + 1;
  s.abort_flag = w + 2;
  return s;
}


using lattn::pack_bf16x2;
using lattn::regs_dec;
using lattn::regs_inc;
using lattn::swz_off;

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) latent_attn_decode_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sm = carve(smem_raw);
  const uint32_t warp = warp_id(), lane = lane_id(), tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int b = blockIdx.x >> 1;
  const int64_t base = a.cu_seqlens[b];
  const int L = (int)(a.cu_seqlens[b + 1] - base);
  const int32_t* idx = a.idx + (int64_t)b * a.k;

  if (tid == 0) {
    for (int s = 0; s < kSwz; ++s) {
      mbar_init(&sm.swz_full[s], kConv / 32 + 32 + 1);   // conversion warps, rope lanes, the mask
      mbar_init(&sm.swz_empty[s], 1);
    }
    for (int s = 0; s < kRaw; ++s) {
      mbar_init(&sm.raw_full[s], 1);
      mbar_init(&sm.raw_empty[s], kConv / 32);
    }
    mbar_init(sm.s_full, 1);
    mbar_init(sm.s_empty, kSoftWarps);
    mbar_init(sm.p_full, kSoftWarps);
    mbar_init(sm.o_done, 1);
    for (int j = 0; j < 2; ++j) mbar_init(&sm.drain[j], 1);
    mbar_init(sm.x_full, 1);    // one local arrival (with the byte count) + the other CTA's bytes
    mbar_init(sm.x_empty, 1);   // one arrival from the other CTA per tile
    *sm.last_valid = -1;
    *sm.abort_flag = 0u;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sm.tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  // Tiles to process: up to the last slot holding a usable position (both
  // CTAs of the pair read the same indices, so they agree).
  {
    int last = -1;
    for (int j = tid; j < a.k; j += kThreads) {
      const int p = idx[j];
      if (p >= 0 && p < L) last = j;
    }
    if (last >= 0) atomicMax(sm.last_valid, last);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sm.tmem_slot;
  const int T = (*sm.last_valid + kTile) / kTile;    // 0 when nothing is selected
  const WaitCtl ctl{sm.abort_flag, a.timeout_ns, a.status};

  if (warp < 4) {
    // the queries of this CTA's columns into TMEM (A operand of the logits)
    const uint32_t lrow = (warp & 3u) * 32u;
    const uint16_t* qrow = a.q + ((int64_t)b * kHeads + tid) * kDqk;
    const uint4* qv = reinterpret_cast<const uint4*>(qrow + 256 * rank);
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint4 v = __ldg(qv + c * 8 + j);
        r[4 * j] = v.x;
        r[4 * j + 1] = v.y;
        r[4 * j + 2] = v.z;
        r[4 * j + 3] = v.w;
      }
      tmem_st_32x32b_x32(tmem + (lrow << 16) + kTmemQ + 32 * c, r);
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
  // both CTAs' barriers are initialised before any remote store
  cluster_sync_all();

  if (warp < kSoftWarps)
    regs_inc<kRegsSoft>();
  else
    regs_dec<kRegsOther>();

  if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax + output
    const uint32_t g = warp >> 2;                 // key half of the tile / value quarter of the output
    const uint32_t h = tid & 127u;                // head = TMEM lane
    const uint32_t lrow = (warp & 3u) * 32u;
    // row h of a warpgroup's 16 KB block of partial logits: 128 bytes, its
    // 16-byte chunks XOR-swizzled by h so that 8 rows cover every bank
    const uint32_t x_row = g * (uint32_t)kXHalf + h * 128u;
    const uint32_t x_peer = map_to_cta(smem_u32(sm.x + g * kXHalf), peer);
    const uint32_t xfull_peer = map_to_cta(smem_u32(sm.x_full), peer);
    const uint32_t xempty_peer = map_to_cta(smem_u32(sm.x_empty), peer);
    const bool leader = (tid & 127u) == 0u;       // issues its warpgroup's copy
    const float c = a.scale_log2;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      const int st = i % kSwz;
      const uint32_t sph = (uint32_t)(i / kSwz) & 1u;
      if (tid == 0) mbar_arrive_expect_tx(sm.x_full, kXTx);
      float s[32];
      ok = ok && mbar_wait(sm.s_full, (uint32_t)i & 1u, ctl, 0x2401);
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
      // exchange partial logits with the other CTA of the pair: wait until it
      // has read the previous tile's, then write this tile's into it
      // (and this warpgroup's previous copy has read the staging buffer)
      if (leader) {
        if (i >= 1) ok = ok && mbar_wait_cluster(sm.x_empty, (uint32_t)(i - 1) & 1u, ctl, 0x2402);
        bulk_wait_read_all();
      }
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
        bulk_s2cluster(x_peer, smem_u32(sm.xs + g * kXHalf), kXHalf, xfull_peer);
        bulk_commit_group();
      }
      ok = ok && mbar_wait_cluster(sm.x_full, (uint32_t)i & 1u, ctl, 0x2403);
      if (ok) {
        const uint8_t* xr = sm.x + x_row;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = *reinterpret_cast<const float4*>(xr + ((j ^ (h & 7u)) << 4));
          s[4 * j] += v.x;
          s[4 * j + 1] += v.y;
          s[4 * j + 2] += v.z;
          s[4 * j + 3] += v.w;
        }
      }
      // the tile's valid slots (written before swz_full completes)
      ok = ok && mbar_wait(&sm.swz_full[st], sph, ctl, 0x2404);
      const uint32_t mk = sm.mask[2 * st + g];
      // z = scale * log2(e) * logit, -inf on unused slots
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float2 z = ffma2(make_float2(s[2 * j], s[2 * j + 1]), make_float2(c, c), make_float2(0.0f, 0.0f));
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
      // tile maximum over both key halves (the buffer alternates with the
      // tile parity, so a slow reader never sees the next tile's value)
      float* tm = sm.tmax + ((uint32_t)i & 1u) * 2 * kHeads;
      tm[g * kHeads + h] = mt;
      named_bar_sync(kBarSoft, kSoftWarps * 32);
      // every softmax thread has read x: the other CTA may write the next
      // tile's (signalled by a thread that issues no bulk copy: a
      // cluster-scope release by the copy's issuer would wait for the copy)
      if (tid == 96) mbar_arrive_cluster(xempty_peer);
      mt = fmaxf(mt, tm[(g ^ 1u) * kHeads + h]);
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
      // P V of the previous tile must be done before O is rescaled and P replaced
      if (i >= 1) ok = ok && mbar_wait(sm.o_done, (uint32_t)(i - 1) & 1u, ctl, 0x2405);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
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
        }
        // keys 32g..32g+31 of the tile are P columns 16g..16g+15 (bf16 pairs)
        tmem_st_32x32b_x16(tmem + (lrow << 16) + kTmemP + 16u * g, p);
        tmem_wait_st();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(sm.p_full);
    }
    if (leader) bulk_wait_read_all();
    // output: O / l for this warpgroup's value columns; lse from rank 0
    if (g == 1) sm.lsum[h] = l_run;
    named_bar_sync(kBarSoft, kSoftWarps * 32);
    if (g == 0) sm.lsum[h] += l_run;
    named_bar_sync(kBarSoft, kSoftWarps * 32);
    const float l_tot = sm.lsum[h];
    if (T >= 1) ok = ok && mbar_wait(sm.o_done, (uint32_t)(T - 1) & 1u, ctl, 0x2407);
    ok = __all_sync(0xffffffffu, ok);
    const float inv_l = l_tot > 0.0f ? 1.0f / l_tot : 0.0f;
    uint16_t* orow = a.out + ((int64_t)b * kHeads + h) * kDv + 256 * rank + 128 * g;
    if (T >= 1 && ok) tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t o[32];
      if (T >= 1 && ok) {
        tmem_ld_32x32b_x32(tmem + (lrow << 16) + kTmemO + 128u * g + 32u * cc, o);
        tmem_wait_ld(o);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
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
    if (rank == 0 && g == 0 && a.lse != nullptr)
      a.lse[(int64_t)b * kHeads + h] = l_tot > 0.0f ? (m_run + log2f(l_tot)) * 0.6931471805599453f : -INFINITY;
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ logits issuer
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < T && ok; ++i) {
        ok = mbar_wait(&sm.swz_full[i % kSwz], (uint32_t)(i / kSwz) & 1u, ctl, 0x2411);
        if (ok && i >= 1) ok = mbar_wait(sm.s_empty, (uint32_t)(i - 1) & 1u, ctl, 0x2412);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sbase = smem_u32(sm.swz + (i % kSwz) * kSwzBytes);
#pragma unroll
        for (int t = 0; t < 18; ++t) {
          const uint32_t a_col = t < 16 ? 8u * t : 128u + 8u * (t - 16);
          const uint32_t slot = t < 16 ? (uint32_t)t / 4u : 4u;
          const uint32_t koff = t < 16 ? 32u * (t % 4) : 64u * rank + 32u * (t - 16);
          mma_bf16_ts(tmem + kTmemS, tmem + kTmemQ + a_col, smem_desc_sw128(sbase + slot * kSlotBytes + koff),
                      kIdescS, t > 0 ? 1u : 0u);
        }
        tc_commit(sm.s_full);
      }
      // every MMA this thread issued completes before TMEM is released
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
        if (!(ok = mbar_wait(sm.p_full, (uint32_t)i & 1u, ctl, 0x2413))) break;
        tc_fence_after();
        const uint32_t sbase = smem_u32(sm.swz + (i % kSwz) * kSwzBytes);
#pragma unroll
        for (int t = 0; t < 4; ++t)
          mma_bf16_ts(tmem + kTmemO, tmem + kTmemP + 8u * t, smem_desc_sw128_mn(sbase + 2048u * t, kSlotBytes),
                      kIdescPV, (i > 0 || t > 0) ? 1u : 0u);
        tc_commit(sm.o_done);
        tc_commit(&sm.swz_empty[i % kSwz]);
      }
      tc_commit(&sm.drain[1]);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&sm.drain[1]), 0u) && globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
    __syncwarp();
  } else if (warp == kFetchWarp) {
    // ------------------------------------------------------------ bulk copies of the value halves
    // Unusable slots copy the sequence's first row (finite values that the
    // softmax masks out), so every tile moves the same byte count.
    bool ok = true;
    int issued = 0;
    for (int i = 0; i < T; ++i) {
      const int r = i % kRaw;
      ok = ok && mbar_wait(&sm.raw_empty[r], ((uint32_t)(i / kRaw) & 1u) ^ 1u, ctl, 0x2421);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      if (lane == 0) mbar_arrive_expect_tx(&sm.raw_full[r], (uint32_t)kRawBytes);
      __syncwarp();
      const uint32_t dst0 = smem_u32(sm.raw + r * kRawBytes);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int n = half * 32 + (int)lane;
        const int j = i * kTile + n;
        const int p = j < a.k ? idx[j] : -1;
        const int64_t row = base + ((p >= 0 && p < L) ? p : 0);
        bulk_copy_g2s(dst0 + n * kRowBytes, a.latent + row * kDqk + 256 * rank, kRowBytes, &sm.raw_full[r]);
      }
      issued = i + 1;
    }
    // copies in flight land before the CTA exits (their full barriers track them)
    if (!ok) {
      const uint64_t t0 = globaltimer_ns();
      for (int i = issued - kRaw < 0 ? 0 : issued - kRaw; i < issued; ++i)
        while (!mbar_try_wait(smem_u32(&sm.raw_full[i % kRaw]), (uint32_t)(i / kRaw) & 1u) &&
               globaltimer_ns() - t0 < a.timeout_ns) {
        }
    }
  } else if (warp == kRopeWarp) {
    // ------------------------------------------------------------ rope parts, slot mask, index checks
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      const int st = i % kSwz;
      ok = ok && mbar_wait(&sm.swz_empty[st], ((uint32_t)(i / kSwz) & 1u) ^ 1u, ctl, 0x2431);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const uint32_t rope = smem_u32(sm.swz + st * kSwzBytes + 4 * kSlotBytes);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const uint32_t n = (uint32_t)half * 32u + lane;
        const int j = i * kTile + (int)n;
        const int p = j < a.k ? idx[j] : -1;
        const bool valid = p >= 0 && p < L;
        if (j < a.k && !valid && p != -1) report_status(a.status, kStatusDeviceCheck, 0xA77E);
        const uint16_t* src = a.latent + (base + (valid ? p : 0)) * kDqk + 512 + 32 * rank;
#pragma unroll
        for (int q = 0; q < 4; ++q) cp_async_16(rope + swz_off(n, 4u * rank + q), src + 8 * q);
        const uint32_t m = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) sm.mask[2 * st + half] = m;
      }
      cp_async_arrive_noinc(&sm.swz_full[st]);
      if (lane == 0) mbar_arrive(&sm.swz_full[st]);
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ staged rows -> swizzled value blocks
    const uint32_t pt = tid - kConvWarp0 * 32;    // 0..255
    bool ok = true;
    for (int i = 0; i < T; ++i) {
      const int r = i % kRaw, st = i % kSwz;
      ok = ok && mbar_wait(&sm.raw_full[r], (uint32_t)(i / kRaw) & 1u, ctl, 0x2441);
      ok = ok && mbar_wait(&sm.swz_empty[st], ((uint32_t)(i / kSwz) & 1u) ^ 1u, ctl, 0x2442);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const uint8_t* src = sm.raw + r * kRawBytes;
      uint8_t* dst = sm.swz + st * kSwzBytes;
      uint4 v[kChunksPerConv];
#pragma unroll
      for (int q = 0; q < kChunksPerConv; ++q) {
        const uint32_t id = pt + kConv * q;            // 32 chunks per row
        v[q] = *reinterpret_cast<const uint4*>(src + (id >> 5) * kRowBytes + (id & 31u) * 16u);
      }
#pragma unroll
      for (int q = 0; q < kChunksPerConv; ++q) {
        const uint32_t id = pt + kConv * q;
        const uint32_t n = id >> 5, ch = id & 31u;
        *reinterpret_cast<uint4*>(dst + (ch >> 3) * kSlotBytes + swz_off(n, ch & 7u)) = v[q];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.raw_empty[r]);
        mbar_arrive(&sm.swz_full[st]);
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // the other CTA may still write into this CTA's shared memory until it is done
  cluster_sync_all();
}

size_t latent_attn_decode_smem() { return smem_bytes(); }

cudaError_t launch_latent_attn_decode(const AttnArgs& a, cudaStream_t stream) {
  // the warpgroups' register budgets add up to the launch allocation; a
  // build that allocated differently would make the increase wait forever
  const size_t smem = smem_bytes();
  cudaError_t e = setup_once_per_device([smem]() {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, latent_attn_decode_kernel);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(latent_attn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2u * (unsigned)a.rows, 1, 1);
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
  e = cudaLaunchKernelEx(&cfg, latent_attn_decode_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dsa
