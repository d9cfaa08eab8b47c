// sparse_attn.cu -- eq. (3) of page "2.2.1 · DSA 与索引器" (§1.1): for each
// query row, every head attends the latent rows its selector picked, with its
// own QK logits and softmax (the indexer scores are not reused); the value is
// the first Dv columns of each selected latent row.  All heads of a row share
// the selected set (the shared key of §1.1), so one gather of a row serves
// every head of the group.
//
// Engine choice (measured on B200): a work item has only 16 heads, so the
// logits product is 16 x keys x Dqk.  tcgen05.mma costs >= ~46 cycles per
// instruction whatever its shape, which caps an N = 16 product at ~1.4K
// FLOP/clk/SM; warp-level mma.sync m16n8k16 sustains ~1.9K FLOP/clk/SM and
// lets the 16 x Dqk query live in registers for the whole row, so it is used
// here.  The selected rows of one sequence sit in L2 (its latent tensor is a
// few MB), so the gather is bounded by L2 -> SM bandwidth: one TMA bulk copy
// per row, issued from four warps, sustains ~13 TB/s per GPU where 16-byte
// cp.async from the same four warps reaches ~5.
//
// Work item = (query row, group of 16 heads); persistent grid, one CTA per SM,
// three warpgroups that work on consecutive chunks of 64 selected rows at once:
//   WG0 producer: validate and compact the row's indices, prefetch the row's
//       queries into L2, then gather the selected latent rows (16 per warp,
//       one bulk copy per row) into three stages of padded rows (1168-byte
//       pitch: eight consecutive rows start in eight different bank groups,
//       so ldmatrix needs no swizzle);
//   WG1 logits + softmax: the 16 x Dqk query as register-resident A
//       fragments; warp w forms the logits of keys 16w..16w+15 of chunk c
//       (S = Q C^T; even and odd k-steps in separate accumulators, each
//       fragment loaded one step ahead of its MMAs), the warps agree on the
//       per-head running max through shared memory (base-2 exponent), then
//       hand the bf16 probabilities P and the per-head rescale factor to WG2;
//   WG2 values: warp w accumulates O for value columns [128w, 128w+128)
//       (O = alpha O + P V) in fp32 registers for chunk c - 1 while WG1 works
//       on chunk c, and writes the normalised output at the end of the row.
// Registers are rebalanced between the warpgroups (setmaxnreg): the logits
// group holds the query fragments, the value group the output accumulators.
// Loop trip counts are fixed at the largest supported shape (Dqk 576, Dv
// 512): columns past Dqk are zero in both operands (zeroed shared memory and
// zero query fragments) and value columns past Dv are computed, not stored.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kChunk = 64;                 // keys per chunk
constexpr int NH = 16;                     // heads per work item (mma M)
constexpr int kStages = 3;
constexpr int kMaxDqk = 576;
constexpr int kKsteps = kMaxDqk / 16;      // 36
constexpr int kMaxDv = 512;
constexpr int kPitch = kMaxDqk * 2 + 16;   // 1168 bytes per gathered row
constexpr int kStageBytes = kChunk * kPitch;
constexpr int kMaxK = 2048;
constexpr int kThreads = 384;
constexpr int kProd = 128;                 // producer threads (warps 0-3)
constexpr int kRowsPerWarp = kChunk / 4;   // rows copied per producer warp and chunk
constexpr int kPBytes = NH * kChunk * 2;
// per-thread register budgets after the split; their sum over the three
// warpgroups equals the launch allocation (168 per thread)
constexpr int kLaunchRegs = 168;
constexpr int kRegsProd = 56, kRegsLogits = 240, kRegsValues = 208;
static_assert(kRegsProd + kRegsLogits + kRegsValues == 3 * kLaunchRegs, "register split must match the launch");

struct TokInfo {
  uint32_t nvalid;
  uint32_t nchunks;
};

// Logits group -> value group, one per chunk (single slot, guarded by the
// p_full / p_empty barriers together with P).
struct Msg {
  int32_t item;        // work item of the chunk; -1: no more work
  uint32_t flags;      // bit 0: first chunk of the item, bit 1: last chunk
  float alpha[NH];     // factor on the running output before this chunk
  float inv_l[NH];     // last chunk: 1 / softmax denominator (0 if empty)
};
constexpr uint32_t kFirst = 1u, kLast = 2u;

__device__ __forceinline__ void row_geometry(const AttnArgs& a, int r, int64_t& base_row, int& len) {
  if (a.mode == 0) {
    base_row = (int64_t)(r / a.nq) * a.kv_len;
    len = a.kv_len;
  } else {
    base_row = a.cu_seqlens[r];
    len = (int)(a.cu_seqlens[r + 1] - base_row);
  }
}

template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// Byte offset of (row r, 16-byte chunk ch) of the 128-byte-row P tile, chunks
// XOR-swizzled by the row so the rows one ldmatrix reads fall in distinct
// bank groups.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t ch) { return r * 128u + ((ch ^ (r & 7u)) << 4); }

// Output rows of heads g and g+8 of an item, value columns 128w + 8j + 2c4.
__device__ __forceinline__ void store_out(const AttnArgs& a, int r, int hg, uint32_t w, uint32_t g, uint32_t c4,
                                          const float (&o)[16][4], float i_lo, float i_hi) {
  const int h_lo = hg * NH + (int)g, h_hi = h_lo + 8;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int v = (int)w * 128 + j * 8 + 2 * (int)c4;
    if (v < a.Dv) {
      if (h_lo < a.H)
        *reinterpret_cast<uint32_t*>(a.out + ((int64_t)r * a.H + h_lo) * a.Dv + v) =
            pack_bf16(o[j][0] * i_lo, o[j][1] * i_lo);
      if (h_hi < a.H)
        *reinterpret_cast<uint32_t*>(a.out + ((int64_t)r * a.H + h_hi) * a.Dv + v) =
            pack_bf16(o[j][2] * i_hi, o[j][3] * i_hi);
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* sC = base;                                                  // [3][64 rows][1168 B]
  uint8_t* sP = sC + kStages * kStageBytes;                            // [16 heads][64 keys] bf16, swizzled
  uint16_t* sList = reinterpret_cast<uint16_t*>(sP + kPBytes);         // [kMaxK] compacted slot numbers
  TokInfo* sTok = reinterpret_cast<TokInfo*>(sList + kMaxK);           // [2]
  float* sMax = reinterpret_cast<float*>(sTok + 2);                    // [2 parities][4 warps][16]
  float* sSum = sMax + 2 * 4 * NH;                                     // [4 warps][16]
  Msg* sMsg = reinterpret_cast<Msg*>(sSum + 4 * NH);
  uint32_t* sWarpCnt = reinterpret_cast<uint32_t*>(sMsg + 1);          // [4]
  uint32_t* sBcast = sWarpCnt + 4;                                     // [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(sBcast + 2) + 7) & ~uintptr_t(7));
  uint64_t* st_full = bars;                  // [3] (4 producer warps + transaction bytes)
  uint64_t* st_empty = bars + kStages;       // [3] (4 value warps)
  uint64_t* tok_full = bars + 2 * kStages;   // [2] (1 producer thread)
  uint64_t* tok_empty = tok_full + 2;        // [2] (4 logits warps)
  uint64_t* p_full = tok_empty + 2;          // (128 logits threads)
  uint64_t* p_empty = p_full + 1;            // (4 value warps)
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(p_empty + 1);

  const uint32_t warp = warp_id(), lane = lane_id();
  // A row shorter than the pitch (Dqk < 576) leaves the tail of its slot as
  // written here: zero, which the fixed-length loops then add nothing from.
  for (uint32_t i = threadIdx.x; i < (uint32_t)(kStages * kStageBytes / 16); i += kThreads)
    reinterpret_cast<uint4*>(sC)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&st_full[i], 4);
      mbar_init(&st_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tok_full[i], 1);
      mbar_init(&tok_empty[i], 4);
    }
    mbar_init(p_full, 128);
    mbar_init(p_empty, 4);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  fence_proxy_async_smem();   // the zeros are ordered before the bulk copies
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};
  const int hg_count = (a.H + NH - 1) / NH;
  const int items = a.rows * hg_count;

  if (warp < 4) {
    // ================================================================ producer
    // A failed wait only disables work: every producer thread still runs the
    // same sequence of named barriers.
    regs_dec<kRegsProd>();
    const uint32_t pt = threadIdx.x;    // 0..127
    const uint32_t row_bytes = (uint32_t)a.Dqk * 2u;
    int tslot = 0, stage = 0;
    uint32_t tphase = 0, sphase = 0;
    bool ok = true;
    int last_phase[kStages];            // parity of this warp's last copies per stage, -1 none
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int r = item / hg_count, hg = item - r * hg_count;
      int64_t base_row;
      int len;
      row_geometry(a, r, base_row, len);
      const int32_t* idx_row = a.idx + (int64_t)r * a.k;
      {  // the logits group reads this item's queries next: bring them into L2
        const int h0 = hg * NH, nh = min(NH, a.H - h0);
        const char* q0 = reinterpret_cast<const char*>(a.q + ((int64_t)r * a.H + h0) * a.Dqk);
        const int lines = (nh * a.Dqk * 2 + 127) / 128;
        for (int i = (int)pt; i < lines; i += kProd) prefetch_l2(q0 + (int64_t)i * 128);
      }
      // ---- compact the valid indices (slot order kept) into sList
      named_bar_sync(2, kProd);          // the previous row's list is no longer read
      constexpr int kPer = kMaxK / kProd;  // 16 slots per thread
      uint32_t vmask = 0;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int slot = (int)pt * kPer + e;
        const int p = slot < a.k ? __ldg(idx_row + slot) : -1;
        if (slot < a.k && (p < -1 || p >= len)) report_status(a.status, kStatusDeviceCheck, 0xA77Eu);
        if (p >= 0 && p < len) vmask |= 1u << e;
      }
      const uint32_t mycnt = __popc(vmask);
      uint32_t incl = mycnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= (uint32_t)o) incl += v;
      }
      if (lane == 31) sWarpCnt[warp] = incl;
      named_bar_sync(2, kProd);
      uint32_t off = incl - mycnt, nvalid = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint32_t c = sWarpCnt[w];
        if ((uint32_t)w < warp) off += c;
        nvalid += c;
      }
#pragma unroll
      for (int e = 0; e < kPer; ++e)
        if (vmask & (1u << e)) sList[off++] = (uint16_t)(pt * kPer + e);
      named_bar_sync(2, kProd);
      const uint32_t nchunks = (nvalid + kChunk - 1) / kChunk;
      if (pt == 0) {
        if (ok) ok = mbar_wait(&tok_empty[tslot], tphase ^ 1u, ctl, 0x2101);
        sTok[tslot].nvalid = ok ? nvalid : 0u;
        sTok[tslot].nchunks = ok ? nchunks : 0u;
        mbar_arrive(&tok_full[tslot]);
      }
      if (++tslot == 2) { tslot = 0; tphase ^= 1u; }
      // ---- gather: warp w copies rows 16w..16w+15 of every chunk, one bulk
      // copy per row from lanes 0..15.  The row number of the next chunk is
      // fetched while the stage is awaited.
      const uint32_t rr = warp * kRowsPerWarp + (lane & (kRowsPerWarp - 1));
      auto fetch_row = [&](uint32_t c) -> int64_t {
        const uint32_t slot = c * kChunk + rr;
        return (lane < (uint32_t)kRowsPerWarp && slot < nvalid) ? base_row + __ldg(idx_row + sList[slot]) : -1;
      };
      int64_t row = nchunks > 0 ? fetch_row(0) : -1;
      for (uint32_t c = 0; c < nchunks; ++c) {
        int got = 1;
        if (lane == 0 && ok) got = mbar_wait(&st_empty[stage], sphase ^ 1u, ctl, 0x2102) ? 1 : 0;
        ok = ok && __shfl_sync(0xffffffffu, got, 0) != 0;
        if (ok) {
          const uint32_t mine = __ballot_sync(0xffffffffu, row >= 0);
          if (lane == 0) mbar_arrive_expect_tx(&st_full[stage], (uint32_t)__popc(mine) * row_bytes);
          __syncwarp();
          if (row >= 0)
            bulk_copy_g2s(smem_u32(sC + stage * kStageBytes + rr * kPitch), a.latent + row * a.Dqk, row_bytes,
                          &st_full[stage]);
          last_phase[stage] = (int)sphase;
        }
        if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        if (c + 1 < nchunks) row = fetch_row(c + 1);
      }
    }
    if (*abort_flag != 0u && lane == 0) {
      // stopped early: give this warp's copies in flight time to land before
      // the CTA exits (bounded; a stage another warp never armed stays open)
#pragma unroll
      for (int s = 0; s < kStages; ++s)
        if (last_phase[s] >= 0) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(smem_u32(&st_full[s]), (uint32_t)last_phase[s]) &&
                 globaltimer_ns() - t0 < a.timeout_ns) {
          }
        }
    }
  } else if (warp < 8) {
    // ================================================================ logits
    // Every logits thread runs the same sequence of named barriers (chunk
    // counts are broadcast); a failed wait only leaves stale data behind.
    regs_inc<kRegsLogits>();
    const uint32_t sw = warp - 4;                 // 0..3
    const uint32_t g = lane >> 2, c4 = lane & 3u; // mma fragment coordinates
    const uint32_t mi = lane >> 3;                // ldmatrix matrix this lane addresses
    int tslot = 0, stage = 0;
    uint32_t tphase = 0, sphase = 0, pphase = 0;
    const uint32_t sC0 = smem_u32(sC);
    // ldmatrix row = key 16sw + 8(mi>>1) + (lane&7), 8-column half (mi&1)
    const uint32_t s_off = (sw * 16 + (mi >> 1) * 8 + (lane & 7u)) * kPitch + (mi & 1u) * 16;
    uint32_t parity = 0;                          // chunk parity (sMax double buffer)
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int r = item / hg_count, hg = item - r * hg_count;
      // queries of this head group -> A fragments (rows g, g+8; heads past H
      // and columns past Dqk are zero)
      uint32_t qa[kKsteps][4];
      {
        const int h0 = hg * NH + (int)g, h1 = h0 + 8;
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)r * a.H + h0) * a.Dqk);
        const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)r * a.H + h1) * a.Dqk);
        const bool v0 = h0 < a.H, v1 = h1 < a.H;
        const int kst = a.Dqk / 16;
#pragma unroll
        for (int ks = 0; ks < kKsteps; ++ks) {
          const bool in = ks < kst;
          const int e = ks * 8 + (int)c4;           // 32-bit element index (2 bf16 each)
          qa[ks][0] = (in && v0) ? __ldg(q0 + e) : 0u;
          qa[ks][1] = (in && v1) ? __ldg(q1 + e) : 0u;
          qa[ks][2] = (in && v0) ? __ldg(q0 + e + 4) : 0u;
          qa[ks][3] = (in && v1) ? __ldg(q1 + e + 4) : 0u;
        }
      }
      (void)mbar_wait(&tok_full[tslot], tphase, ctl, 0x2301);
      named_bar_sync(1, 128);
      if (threadIdx.x == kProd) {
        const bool ab = *abort_flag != 0u;
        sBcast[0] = ab ? 0u : sTok[tslot].nvalid;
        sBcast[1] = ab ? 0u : sTok[tslot].nchunks;
      }
      named_bar_sync(1, 128);
      const uint32_t nvalid = sBcast[0], nchunks = sBcast[1];
      __syncwarp();
      if (lane == 0) mbar_arrive(&tok_empty[tslot]);
      if (++tslot == 2) { tslot = 0; tphase ^= 1u; }

      if (nchunks == 0) {
        // nothing selected: zero output, log-sum-exp -inf
        float z[16][4];
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j][0] = z[j][1] = z[j][2] = z[j][3] = 0.0f;
        store_out(a, r, hg, sw, g, c4, z, 0.0f, 0.0f);
        if (a.lse && sw == 0 && c4 == 0) {
          const int h_lo = hg * NH + (int)g, h_hi = h_lo + 8;
          if (h_lo < a.H) a.lse[(int64_t)r * a.H + h_lo] = -INFINITY;
          if (h_hi < a.H) a.lse[(int64_t)r * a.H + h_hi] = -INFINITY;
        }
        continue;
      }
      float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;   // heads g, g+8
      for (uint32_t c = 0; c < nchunks; ++c) {
        (void)mbar_wait(&st_full[stage], sphase, ctl, 0x2302);
        const uint32_t cbase = sC0 + stage * kStageBytes;
        // ---- S = Q C^T for keys 16sw..16sw+15 (n-tiles 0, 1)
        float sa[2][2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int j = 0; j < 2; ++j) sa[i][j][0] = sa[i][j][1] = sa[i][j][2] = sa[i][j][3] = 0.0f;
        {
          uint32_t bc[4], bn[4];
          ldsm_x4(cbase + s_off, bc);
#pragma unroll
          for (int ks = 0; ks < kKsteps; ++ks) {
            if (ks + 1 < kKsteps) ldsm_x4(cbase + s_off + (ks + 1) * 32, bn);
            mma16816(sa[ks & 1][0], qa[ks], bc[0], bc[1]);
            mma16816(sa[ks & 1][1], qa[ks], bc[2], bc[3]);
            if (ks + 1 < kKsteps) {
#pragma unroll
              for (int i = 0; i < 4; ++i) bc[i] = bn[i];
            }
          }
        }
        float s0[4], s1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          s0[i] = sa[0][0][i] + sa[1][0][i];
          s1[i] = sa[0][1][i] + sa[1][1][i];
        }
        if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        // ---- mask, scale, chunk max per head
        const uint32_t kbase = c * kChunk + sw * 16 + 2 * c4;   // key of s0[0]
        const bool k00 = kbase < nvalid, k01 = kbase + 1 < nvalid, k10 = kbase + 8 < nvalid,
                   k11 = kbase + 9 < nvalid;
        const float sl = a.scale_log2;
        s0[0] = k00 ? s0[0] * sl : -INFINITY;
        s0[1] = k01 ? s0[1] * sl : -INFINITY;
        s0[2] = k00 ? s0[2] * sl : -INFINITY;
        s0[3] = k01 ? s0[3] * sl : -INFINITY;
        s1[0] = k10 ? s1[0] * sl : -INFINITY;
        s1[1] = k11 ? s1[1] * sl : -INFINITY;
        s1[2] = k10 ? s1[2] * sl : -INFINITY;
        s1[3] = k11 ? s1[3] * sl : -INFINITY;
        float mx_lo = fmaxf(fmaxf(s0[0], s0[1]), fmaxf(s1[0], s1[1]));
        float mx_hi = fmaxf(fmaxf(s0[2], s0[3]), fmaxf(s1[2], s1[3]));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        float* smx = sMax + parity * 4 * NH;
        if (c4 == 0) {
          smx[sw * NH + g] = mx_lo;
          smx[sw * NH + g + 8] = mx_hi;
        }
        named_bar_sync(1, 128);   // every warp's chunk maxima are visible
        const float cm_lo = fmaxf(fmaxf(smx[g], smx[NH + g]), fmaxf(smx[2 * NH + g], smx[3 * NH + g]));
        const float cm_hi =
            fmaxf(fmaxf(smx[g + 8], smx[NH + g + 8]), fmaxf(smx[2 * NH + g + 8], smx[3 * NH + g + 8]));
        parity ^= 1u;
        const float mn_lo = fmaxf(m_lo, cm_lo), mn_hi = fmaxf(m_hi, cm_hi);
        const float al_lo = (m_lo == -INFINITY) ? 0.0f : exp2f(m_lo - mn_lo);
        const float al_hi = (m_hi == -INFINITY) ? 0.0f : exp2f(m_hi - mn_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;
        const float mu_lo = mn_lo == -INFINITY ? 0.0f : mn_lo;
        const float mu_hi = mn_hi == -INFINITY ? 0.0f : mn_hi;
        const float p00 = exp2f(s0[0] - mu_lo), p01 = exp2f(s0[1] - mu_lo);
        const float p02 = exp2f(s0[2] - mu_hi), p03 = exp2f(s0[3] - mu_hi);
        const float p10 = exp2f(s1[0] - mu_lo), p11 = exp2f(s1[1] - mu_lo);
        const float p12 = exp2f(s1[2] - mu_hi), p13 = exp2f(s1[3] - mu_hi);
        l_lo = l_lo * al_lo + (p00 + p01 + p10 + p11);
        l_hi = l_hi * al_hi + (p02 + p03 + p12 + p13);
        const bool last = c + 1 == nchunks;
        float il_lo = 0.0f, il_hi = 0.0f;
        if (last) {
          // softmax denominators of the row: quad sums, then across warps
          float t_lo = l_lo, t_hi = l_hi;
          t_lo += __shfl_xor_sync(0xffffffffu, t_lo, 1);
          t_lo += __shfl_xor_sync(0xffffffffu, t_lo, 2);
          t_hi += __shfl_xor_sync(0xffffffffu, t_hi, 1);
          t_hi += __shfl_xor_sync(0xffffffffu, t_hi, 2);
          if (c4 == 0) {
            sSum[sw * NH + g] = t_lo;
            sSum[sw * NH + g + 8] = t_hi;
          }
          named_bar_sync(1, 128);
          const float L_lo = sSum[g] + sSum[NH + g] + sSum[2 * NH + g] + sSum[3 * NH + g];
          const float L_hi = sSum[g + 8] + sSum[NH + g + 8] + sSum[2 * NH + g + 8] + sSum[3 * NH + g + 8];
          il_lo = L_lo > 0.0f ? 1.0f / L_lo : 0.0f;
          il_hi = L_hi > 0.0f ? 1.0f / L_hi : 0.0f;
          if (a.lse && sw == 0 && c4 == 0) {
            const float ln2 = 0.69314718055994531f;
            const int h_lo = hg * NH + (int)g, h_hi = h_lo + 8;
            if (h_lo < a.H) a.lse[(int64_t)r * a.H + h_lo] = L_lo > 0.0f ? (m_lo + log2f(L_lo)) * ln2 : -INFINITY;
            if (h_hi < a.H) a.lse[(int64_t)r * a.H + h_hi] = L_hi > 0.0f ? (m_hi + log2f(L_hi)) * ln2 : -INFINITY;
          }
        }
        // ---- hand P and the factors to the value group once it has taken
        // the previous chunk's
        (void)mbar_wait(p_empty, pphase ^ 1u, ctl, 0x2303);
        {
          const uint32_t k0 = sw * 16 + 2 * c4;   // keys k0, k0+1 (n-tile 0) and k0+8, k0+9 (n-tile 1)
          *reinterpret_cast<uint32_t*>(sP + swz(g, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p00, p01);
          *reinterpret_cast<uint32_t*>(sP + swz(g + 8, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p02, p03);
          *reinterpret_cast<uint32_t*>(sP + swz(g, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p10, p11);
          *reinterpret_cast<uint32_t*>(sP + swz(g + 8, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p12, p13);
        }
        if (sw == 0 && c4 == 0) {
          sMsg->alpha[g] = al_lo;
          sMsg->alpha[g + 8] = al_hi;
          sMsg->inv_l[g] = il_lo;
          sMsg->inv_l[g + 8] = il_hi;
        }
        if (sw == 0 && lane == 0) {
          sMsg->item = item;
          sMsg->flags = (c == 0 ? kFirst : 0u) | (last ? kLast : 0u);
        }
        mbar_arrive(p_full);
        pphase ^= 1u;
      }
    }
    // no more work for the value group
    (void)mbar_wait(p_empty, pphase ^ 1u, ctl, 0x2304);
    if (sw == 0 && lane == 0) sMsg->item = -1;
    mbar_arrive(p_full);
  } else {
    // ================================================================ values
    regs_inc<kRegsValues>();
    const uint32_t vw = warp - 8;                 // 0..3
    const uint32_t g = lane >> 2, c4 = lane & 3u;
    const uint32_t mi = lane >> 3;
    int stage = 0;
    uint32_t sphase = 0, pphase = 0;
    const uint32_t sC0 = smem_u32(sC), sP0 = smem_u32(sP);
    // key 8(mi&1) + (lane&7) of each 16-key step, value columns 128vw + 8(mi>>1)
    const uint32_t v_off = ((mi & 1u) * 8 + (lane & 7u)) * kPitch + (vw * 128 + (mi >> 1) * 8) * 2;
    // P: head (lane&15), 8-key half (lane>>4) of each 16-key step
    const uint32_t p_row = lane & 15u, p_half = lane >> 4;
    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    for (;;) {
      if (!mbar_wait(p_full, pphase, ctl, 0x2401)) break;
      pphase ^= 1u;
      const int item = sMsg->item;
      if (item < 0) break;
      const uint32_t flags = sMsg->flags;
      const float al_lo = sMsg->alpha[g], al_hi = sMsg->alpha[g + 8];
      const float il_lo = sMsg->inv_l[g], il_hi = sMsg->inv_l[g + 8];
      if (flags & kFirst) {
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
      } else if (al_lo != 1.0f || al_hi != 1.0f) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          o[j][0] *= al_lo;
          o[j][1] *= al_lo;
          o[j][2] *= al_hi;
          o[j][3] *= al_hi;
        }
      }
      // the stage's bytes landed before the logits group released P (this
      // wait returns at once; it only makes the ordering explicit)
      (void)mbar_wait(&st_full[stage], sphase, ctl, 0x2402);
      const uint32_t cbase = sC0 + stage * kStageBytes;
      // ---- O[:, 128vw .. 128vw+127] += P (16 x 64) V (64 x 128); each
      // fragment is loaded one step ahead of the MMAs that use it
      {
        uint32_t pa[4], pn[4], vc[4], vn[4];
        ldsm_x4(sP0 + swz(p_row, p_half), pa);
        ldsm_x4_t(cbase + v_off, vc);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            const bool lastf = kk == kChunk / 16 - 1 && j == 14;
            if (j == 0 && kk + 1 < kChunk / 16) ldsm_x4(sP0 + swz(p_row, (uint32_t)(kk + 1) * 2u + p_half), pn);
            if (!lastf) {
              const int nkk = j == 14 ? kk + 1 : kk, nj = j == 14 ? 0 : j + 2;
              ldsm_x4_t(cbase + v_off + nkk * 16 * kPitch + nj * 16, vn);
            }
            mma16816(o[j], pa, vc[0], vc[1]);
            mma16816(o[j + 1], pa, vc[2], vc[3]);
            if (!lastf) {
#pragma unroll
              for (int i = 0; i < 4; ++i) vc[i] = vn[i];
              if (j == 14) {
#pragma unroll
                for (int i = 0; i < 4; ++i) pa[i] = pn[i];
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&st_empty[stage]);
        mbar_arrive(p_empty);
      }
      if (++stage == kStages) { stage = 0; sphase ^= 1u; }
      if (flags & kLast) {
        const int r = item / hg_count, hg = item - r * hg_count;
        store_out(a, r, hg, vw, g, c4, o, il_lo, il_hi);
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static size_t attn_smem() {
  return 128 + (size_t)kStages * kStageBytes + kPBytes + kMaxK * 2 + 2 * sizeof(TokInfo) + (3 * 4 * NH) * 4 +
         sizeof(Msg) + 6 * 4 + 8 + (2 * kStages + 6) * 8 + 8;
}

cudaError_t launch_sparse_attn(const AttnArgs& a, int grid, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.nh != NH || a.Dqk > kMaxDqk || a.Dqk % 16 != 0 || a.k > kMaxK || a.Dv > kMaxDv)
    return cudaErrorInvalidValue;
  // the warpgroups' register budgets add up to the launch allocation; a
  // build that allocated differently would make the increase wait forever
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, sparse_attn_kernel);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const size_t smem = attn_smem();
  e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  sparse_attn_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
