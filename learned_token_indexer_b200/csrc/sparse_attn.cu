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
// lets the query live in registers for the whole row, so it is used here.
// The selected rows of one sequence sit in L2 (its latent tensor is a few
// MB), so the gather is bounded by L2 -> SM bandwidth: one TMA bulk copy per
// row, issued from four warps, sustains ~13 TB/s per GPU where 16-byte
// cp.async from the same four warps reaches ~5.
//
// Work item = (query row, group of 16 heads); persistent grid, one CTA per SM,
// four warpgroups working on consecutive chunks of 64 selected rows at once:
//   WG0-1 producers: validate the row's indices into per-32-slot validity
//       masks and prefix counts, prefetch the row's queries into L2, then
//       gather the selected latent rows (8 per warp, one bulk copy per row;
//       bulk copies from one warp issue one after another) into three
//       stages of padded rows (1168-byte pitch: eight consecutive rows start
//       in eight different bank groups, so ldmatrix needs no swizzle);
//   WG2 logits: warp w owns keys 16w..16w+15 of every chunk.  It forms their
//       logits (S = Q C^T, the 16 x Dqk query as register-resident A
//       fragments), keeps its own running max per head (base-2 exponent) and
//       emits bf16 P = 2^(S - M_w) relative to that max, with M_w, into one of
//       two hand-off slots.  The warps never wait for one another inside a row;
//       they combine their softmax denominators once, at the row's end;
//   WG3 values: warp w accumulates O for value columns [128w, 128w+128)
//       (O += P V) in fp32 registers against a reference max R per head: it
//       raises R to the largest M_w of the chunk, rescales O by 2^(R_old - R),
//       and multiplies each logits warp's 16-key block of P by 2^(M_w - R)
//       before its MMAs.  At the row's end R equals the row max, so O / L is
//       the softmax-weighted sum.
// In the MMA loops even and odd k-steps go to separate accumulators and every
// fragment is requested two steps ahead of its MMAs; the next row's queries
// are requested as soon as the current row's last logits are formed.
// Registers are rebalanced between the warpgroups (setmaxnreg).  Loop trip
// counts are fixed at the largest supported shape (Dqk 576, Dv 512): columns
// past Dqk are zero in both operands (zeroed shared memory and zero query
// fragments) and value columns past Dv are computed, not stored.
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
constexpr int kBlocks = kMaxK / 32;        // 32-slot validity blocks of an index row
constexpr int kThreads = 512;
constexpr int kProdWarps = 8;              // producer warps 0-7 (two warpgroups)
constexpr int kProd = kProdWarps * 32;
constexpr int kRowsPerWarp = kChunk / kProdWarps;   // rows copied per producer warp and chunk
constexpr int kPBytes = NH * kChunk * 2;
constexpr int kSlots = 2;                  // logits -> values hand-off slots
// per-thread register budgets after the split; their sum over the four
// warpgroups equals the launch allocation (128 per thread)
constexpr int kLaunchRegs = 128;
constexpr int kRegsProd = 56, kRegsLogits = 232, kRegsValues = 168;
static_assert(2 * kRegsProd + kRegsLogits + kRegsValues == 4 * kLaunchRegs, "register split must match the launch");

// named barriers (0 is __syncthreads)
constexpr uint32_t kBarLogits = 1, kBarProd = 2;

struct TokInfo {
  uint32_t nvalid;
  uint32_t nchunks;
};

// Logits group -> value group, one per chunk, with the chunk's P.
struct Msg {
  int32_t item;          // work item of the chunk; -1: no more work
  uint32_t flags;        // bit 0: first chunk of the item, bit 1: last chunk
  float m[4][NH];        // running max of each logits warp after this chunk (-inf: none yet)
  float inv_l[NH];       // last chunk: 1 / softmax denominator at the row max (0 if empty)
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
// lane-wise bf16 product of two packed pairs, rounded to nearest
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t x, uint32_t y) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(y));
  return d;
}
// Byte offset of (row r, 16-byte chunk ch) of the 128-byte-row P tile, chunks
// XOR-swizzled by the row so the rows one ldmatrix reads fall in distinct
// bank groups.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t ch) { return r * 128u + ((ch ^ (r & 7u)) << 4); }

// Position of the (rank+1)-th set bit of m (rank < popc(m)).
__device__ __forceinline__ uint32_t nth_set_bit(uint32_t m, uint32_t rank) {
  uint32_t pos = 0;
#pragma unroll
  for (uint32_t w = 16; w > 0; w >>= 1) {
    const uint32_t low = __popc(m & ((1u << w) - 1u));
    if (rank >= low) {
      rank -= low;
      m >>= w;
      pos += w;
    }
  }
  return pos;
}

// Query fragments of one item (rows g, g+8 of the head group; heads past H
// and columns past Dqk are zero).
__device__ __forceinline__ void load_q(const AttnArgs& a, int hg_count, int item, uint32_t g, uint32_t c4,
                                       uint32_t (&qa)[kKsteps][4]) {
  const int r = item / hg_count, hg = item - r * hg_count;
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

// Logits of keys 16w..16w+15: s0 = n-tile 0 (keys +0..7), s1 = n-tile 1
// (keys +8..15).
__device__ __forceinline__ void logits(uint32_t row_addr, const uint32_t (&qa)[kKsteps][4], float (&s0)[4],
                                       float (&s1)[4]) {
  float sa[2][2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) sa[i][j][0] = sa[i][j][1] = sa[i][j][2] = sa[i][j][3] = 0.0f;
  // fragments of step i live in b[i % 3], requested two steps ahead
  uint32_t b[3][4];
  ldsm_x4(row_addr, b[0]);
  ldsm_x4(row_addr + 32, b[1]);
#pragma unroll
  for (int i = 0; i < kKsteps; ++i) {
    if (i + 2 < kKsteps) ldsm_x4(row_addr + (i + 2) * 32, b[(i + 2) % 3]);
    mma16816(sa[i & 1][0], qa[i], b[i % 3][0], b[i % 3][1]);
    mma16816(sa[i & 1][1], qa[i], b[i % 3][2], b[i % 3][3]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s0[i] = sa[0][0][i] + sa[1][0][i];
    s1[i] = sa[0][1][i] + sa[1][1][i];
  }
}

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
  uint8_t* sP = sC + kStages * kStageBytes;                            // [2 slots][16 heads][64 keys] bf16
  Msg* sMsg = reinterpret_cast<Msg*>(sP + kSlots * kPBytes);           // [2 slots]
  uint32_t* sMask = reinterpret_cast<uint32_t*>(sMsg + kSlots);        // [64] validity of 32-slot blocks
  uint32_t* sPre = sMask + kBlocks;                                    // [65] valid entries before each block
  TokInfo* sTok = reinterpret_cast<TokInfo*>(sPre + kBlocks + 1);      // [2]
  float* sFin = reinterpret_cast<float*>(sTok + 2);                    // [2][4 warps][16] row-end max, sum
  uint32_t* sWarpCnt = reinterpret_cast<uint32_t*>(sFin + 2 * 4 * NH); // [8]
  uint32_t* sBcast = sWarpCnt + kProdWarps;                            // [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(sBcast + 2) + 7) & ~uintptr_t(7));
  uint64_t* st_full = bars;                  // [3] (8 producer warps + transaction bytes)
  uint64_t* st_empty = bars + kStages;       // [3] (4 value warps)
  uint64_t* tok_full = bars + 2 * kStages;   // [2] (1 producer thread)
  uint64_t* tok_empty = tok_full + 2;        // [2] (4 logits warps)
  uint64_t* p_full = tok_empty + 2;          // [2] (128 logits threads)
  uint64_t* p_empty = p_full + kSlots;       // [2] (4 value warps)
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(p_empty + kSlots);

  const uint32_t warp = warp_id(), lane = lane_id();
  // A row shorter than the pitch (Dqk < 576) leaves the tail of its slot as
  // written here: zero, which the fixed-length loops then add nothing from.
  for (uint32_t i = threadIdx.x; i < (uint32_t)(kStages * kStageBytes / 16); i += kThreads)
    reinterpret_cast<uint4*>(sC)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&st_full[i], kProdWarps);
      mbar_init(&st_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tok_full[i], 1);
      mbar_init(&tok_empty[i], 4);
    }
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 4);
    }
    *abort_flag = 0u;
    mbar_fence_init();
  }
  fence_proxy_async_smem();   // the zeros are ordered before the bulk copies
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};
  const int hg_count = (a.H + NH - 1) / NH;
  const int items = a.rows * hg_count;
  const uint32_t g = lane >> 2, c4 = lane & 3u;   // mma fragment coordinates
  const uint32_t mi = lane >> 3;                  // ldmatrix matrix this lane addresses
  const uint32_t sC0 = smem_u32(sC), sP0 = smem_u32(sP);

  if (warp < (uint32_t)kProdWarps) {
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
      // ---- validity masks: thread pt owns slots [8pt, 8pt + 8); four threads
      // (consecutive lanes) make one 32-slot block
      named_bar_sync(kBarProd, kProd);   // the previous row's masks are no longer read
      constexpr int kPer = kMaxK / kProd;
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
      static_assert(kPer == 8, "four threads per 32-slot block");
      const uint32_t m1 = __shfl_down_sync(0xffffffffu, vmask, 1);
      const uint32_t m2 = __shfl_down_sync(0xffffffffu, vmask, 2);
      const uint32_t m3 = __shfl_down_sync(0xffffffffu, vmask, 3);
      if (lane == 31) sWarpCnt[warp] = incl;
      named_bar_sync(kBarProd, kProd);
      uint32_t off = incl - mycnt, nvalid = 0;
#pragma unroll
      for (int w = 0; w < kProdWarps; ++w) {
        const uint32_t c = sWarpCnt[w];
        if ((uint32_t)w < warp) off += c;
        nvalid += c;
      }
      if ((pt & 3u) == 0u) {
        sMask[pt >> 2] = vmask | (m1 << 8) | (m2 << 16) | (m3 << 24);
        sPre[pt >> 2] = off;
      }
      if (pt == 0) sPre[kBlocks] = nvalid;
      named_bar_sync(kBarProd, kProd);
      const uint32_t nchunks = (nvalid + kChunk - 1) / kChunk;
      if (pt == 0) {
        if (ok) ok = mbar_wait(&tok_empty[tslot], tphase ^ 1u, ctl, 0x2101);
        sTok[tslot].nvalid = ok ? nvalid : 0u;
        sTok[tslot].nchunks = ok ? nchunks : 0u;
        mbar_arrive(&tok_full[tslot]);
      }
      if (++tslot == 2) { tslot = 0; tphase ^= 1u; }
      // ---- gather: warp w copies rows 8w..8w+7 of every chunk, one bulk
      // copy per row from lanes 0..7 (bulk copies from one warp are issued one
      // after another, so eight warps share the issuing).  The j-th valid slot is found from the
      // prefix counts and the block's mask; the next chunk's row number is
      // fetched while the stage is awaited.
      const uint32_t rr = warp * kRowsPerWarp + (lane & (kRowsPerWarp - 1));
      auto fetch_row = [&](uint32_t c) -> int64_t {
        const uint32_t j = c * kChunk + rr;
        if (lane >= (uint32_t)kRowsPerWarp || j >= nvalid) return -1;
        uint32_t lo = 0, hi = kBlocks;   // sPre[lo] <= j < sPre[hi]
#pragma unroll
        for (int it = 0; it < 6; ++it) {
          const uint32_t mid = (lo + hi) >> 1;
          if (sPre[mid] <= j) lo = mid; else hi = mid;
        }
        const uint32_t slot = lo * 32u + nth_set_bit(sMask[lo], j - sPre[lo]);
        return base_row + __ldg(idx_row + slot);
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
  } else if (warp < (uint32_t)kProdWarps + 4) {
    // ================================================================ logits
    // Every thread of the group runs the same sequence of named barriers
    // (chunk counts are broadcast); a failed wait only leaves stale data.
    regs_inc<kRegsLogits>();
    const uint32_t sw = warp - kProdWarps;
    const uint32_t s_off = (sw * 16 + (mi >> 1) * 8 + (lane & 7u)) * kPitch + (mi & 1u) * 16;
    int tslot = 0, stage = 0, slot = 0;
    uint32_t tphase = 0, sphase = 0, pphase = 0;
    uint32_t qa[kKsteps][4];
    if ((int)blockIdx.x < items) load_q(a, hg_count, blockIdx.x, g, c4, qa);
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int r = item / hg_count, hg = item - r * hg_count;
      const int next_item = item + (int)gridDim.x;
      (void)mbar_wait(&tok_full[tslot], tphase, ctl, 0x2301);
      named_bar_sync(kBarLogits, 128);
      if (threadIdx.x == (uint32_t)kProd) {
        const bool ab = *abort_flag != 0u;
        sBcast[0] = ab ? 0u : sTok[tslot].nvalid;
        sBcast[1] = ab ? 0u : sTok[tslot].nchunks;
      }
      named_bar_sync(kBarLogits, 128);
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
        if (next_item < items) load_q(a, hg_count, next_item, g, c4, qa);
        continue;
      }
      // this warp's running max and denominator of heads g, g+8
      float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;
      for (uint32_t c = 0; c < nchunks; ++c) {
        (void)mbar_wait(&st_full[stage], sphase, ctl, 0x2302);
        float s0[4], s1[4];
        logits(sC0 + stage * kStageBytes + s_off, qa, s0, s1);
        if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        const bool last = c + 1 == nchunks;
        if (last && next_item < items) load_q(a, hg_count, next_item, g, c4, qa);
        // ---- mask, scale, running max of this warp's keys
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
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
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
        float il_lo = 0.0f, il_hi = 0.0f;
        if (last) {
          // the row's denominators at the row max: every warp's (max, sum)
          float t_lo = l_lo, t_hi = l_hi;
          t_lo += __shfl_xor_sync(0xffffffffu, t_lo, 1);
          t_lo += __shfl_xor_sync(0xffffffffu, t_lo, 2);
          t_hi += __shfl_xor_sync(0xffffffffu, t_hi, 1);
          t_hi += __shfl_xor_sync(0xffffffffu, t_hi, 2);
          float* fm = sFin;            // [4][16] maxima
          float* fl = sFin + 4 * NH;   // [4][16] sums
          if (c4 == 0) {
            fm[sw * NH + g] = m_lo;
            fm[sw * NH + g + 8] = m_hi;
            fl[sw * NH + g] = t_lo;
            fl[sw * NH + g + 8] = t_hi;
          }
          named_bar_sync(kBarLogits, 128);
          float R_lo = -INFINITY, R_hi = -INFINITY;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            R_lo = fmaxf(R_lo, fm[w * NH + g]);
            R_hi = fmaxf(R_hi, fm[w * NH + g + 8]);
          }
          float L_lo = 0.0f, L_hi = 0.0f;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const float ml = fm[w * NH + g], mh = fm[w * NH + g + 8];
            if (ml != -INFINITY) L_lo += fl[w * NH + g] * exp2f(ml - R_lo);
            if (mh != -INFINITY) L_hi += fl[w * NH + g + 8] * exp2f(mh - R_hi);
          }
          named_bar_sync(kBarLogits, 128);   // sFin is reused by the next row
          il_lo = L_lo > 0.0f ? 1.0f / L_lo : 0.0f;
          il_hi = L_hi > 0.0f ? 1.0f / L_hi : 0.0f;
          if (a.lse && sw == 0 && c4 == 0) {
            const float ln2 = 0.69314718055994531f;
            const int h_lo = hg * NH + (int)g, h_hi = h_lo + 8;
            if (h_lo < a.H) a.lse[(int64_t)r * a.H + h_lo] = L_lo > 0.0f ? (R_lo + log2f(L_lo)) * ln2 : -INFINITY;
            if (h_hi < a.H) a.lse[(int64_t)r * a.H + h_hi] = L_hi > 0.0f ? (R_hi + log2f(L_hi)) * ln2 : -INFINITY;
          }
        }
        // ---- hand P (relative to this warp's max) and the max over
        (void)mbar_wait(&p_empty[slot], pphase ^ 1u, ctl, 0x2303);
        uint8_t* P = sP + slot * kPBytes;
        Msg* msg = sMsg + slot;
        {
          const uint32_t k0 = sw * 16 + 2 * c4;   // keys k0, k0+1 (n-tile 0) and k0+8, k0+9 (n-tile 1)
          *reinterpret_cast<uint32_t*>(P + swz(g, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p00, p01);
          *reinterpret_cast<uint32_t*>(P + swz(g + 8, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p02, p03);
          *reinterpret_cast<uint32_t*>(P + swz(g, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p10, p11);
          *reinterpret_cast<uint32_t*>(P + swz(g + 8, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p12, p13);
        }
        if (c4 == 0) {
          msg->m[sw][g] = m_lo;
          msg->m[sw][g + 8] = m_hi;
          if (sw == 0) {
            msg->inv_l[g] = il_lo;
            msg->inv_l[g + 8] = il_hi;
          }
        }
        if (sw == 0 && lane == 0) {
          msg->item = item;
          msg->flags = (c == 0 ? kFirst : 0u) | (last ? kLast : 0u);
        }
        mbar_arrive(&p_full[slot]);
        if (++slot == kSlots) { slot = 0; pphase ^= 1u; }
      }
    }
    // no more work for the value group
    (void)mbar_wait(&p_empty[slot], pphase ^ 1u, ctl, 0x2304);
    if (sw == 0 && lane == 0) sMsg[slot].item = -1;
    mbar_arrive(&p_full[slot]);
  } else {
    // ================================================================ values
    regs_inc<kRegsValues>();
    const uint32_t vw = warp - kProdWarps - 4;
    int stage = 0, slot = 0;
    uint32_t sphase = 0, pphase = 0;
    // key 8(mi&1) + (lane&7) of each 16-key step, value columns 128vw + 8(mi>>1)
    const uint32_t v_off = ((mi & 1u) * 8 + (lane & 7u)) * kPitch + (vw * 128 + (mi >> 1) * 8) * 2;
    // P: head (lane&15), 8-key half (lane>>4) of each 16-key step
    const uint32_t p_row = lane & 15u, p_half = lane >> 4;
    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
    float R_lo = -INFINITY, R_hi = -INFINITY;    // reference max of heads g, g+8
    for (;;) {
      if (!mbar_wait(&p_full[slot], pphase, ctl, 0x2401)) break;
      const Msg* msg = sMsg + slot;
      const int item = msg->item;
      if (item < 0) break;
      const uint32_t flags = msg->flags;
      float wm_lo[4], wm_hi[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        wm_lo[w] = msg->m[w][g];
        wm_hi[w] = msg->m[w][g + 8];
      }
      const float il_lo = msg->inv_l[g], il_hi = msg->inv_l[g + 8];
      // raise the reference to the chunk's largest warp max, rescale O
      float rn_lo = fmaxf(fmaxf(wm_lo[0], wm_lo[1]), fmaxf(wm_lo[2], wm_lo[3]));
      float rn_hi = fmaxf(fmaxf(wm_hi[0], wm_hi[1]), fmaxf(wm_hi[2], wm_hi[3]));
      if (flags & kFirst) {
#pragma unroll
        for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
      } else {
        rn_lo = fmaxf(rn_lo, R_lo);
        rn_hi = fmaxf(rn_hi, R_hi);
        const float al_lo = exp2f(R_lo - rn_lo), al_hi = exp2f(R_hi - rn_hi);
        if (al_lo != 1.0f || al_hi != 1.0f) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            o[j][0] *= al_lo;
            o[j][1] *= al_lo;
            o[j][2] *= al_hi;
            o[j][3] *= al_hi;
          }
        }
      }
      R_lo = rn_lo;
      R_hi = rn_hi;
      // factor of each logits warp's block: 2^(M_w - R) (0 while M_w = -inf),
      // as a bf16 pair per head row
      uint32_t f_lo[4], f_hi[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float a_lo = wm_lo[w] == -INFINITY ? 0.0f : exp2f(wm_lo[w] - R_lo);
        const float a_hi = wm_hi[w] == -INFINITY ? 0.0f : exp2f(wm_hi[w] - R_hi);
        f_lo[w] = pack_bf16(a_lo, a_lo);
        f_hi[w] = pack_bf16(a_hi, a_hi);
      }
      // the stage's bytes landed before the logits group released P (this
      // wait returns at once; it only makes the ordering explicit)
      (void)mbar_wait(&st_full[stage], sphase, ctl, 0x2402);
      const uint32_t cbase = sC0 + stage * kStageBytes;
      const uint32_t pbase = sP0 + slot * kPBytes;
      // ---- O[:, 128vw .. 128vw+127] += P (16 x 64) V (64 x 128)
      {
        // step t = 8 kk + j/2 covers keys 16kk.. (logits warp kk) and value
        // columns 16(j/2)..; its fragments live in vb[t % 3], requested two
        // steps ahead; the scaled P fragments of step kk live in pa[kk & 1]
        constexpr int kSteps = (kChunk / 16) * 8;
        auto v_addr = [&](int t) { return cbase + v_off + (t >> 3) * 16 * kPitch + (t & 7) * 32; };
        auto load_p = [&](int kk, uint32_t (&p)[4]) {
          ldsm_x4(pbase + swz(p_row, (uint32_t)kk * 2u + p_half), p);
          p[0] = mul_bf16x2(p[0], f_lo[kk]);
          p[1] = mul_bf16x2(p[1], f_hi[kk]);
          p[2] = mul_bf16x2(p[2], f_lo[kk]);
          p[3] = mul_bf16x2(p[3], f_hi[kk]);
        };
        uint32_t pa[2][4], vb[3][4];
        load_p(0, pa[0]);
        ldsm_x4_t(v_addr(0), vb[0]);
        ldsm_x4_t(v_addr(1), vb[1]);
#pragma unroll
        for (int t = 0; t < kSteps; ++t) {
          const int kk = t >> 3, j = (t & 7) * 2;
          if (j == 0 && kk + 1 < kChunk / 16) load_p(kk + 1, pa[(kk + 1) & 1]);
          if (t + 2 < kSteps) ldsm_x4_t(v_addr(t + 2), vb[(t + 2) % 3]);
          mma16816(o[j], pa[kk & 1], vb[t % 3][0], vb[t % 3][1]);
          mma16816(o[j + 1], pa[kk & 1], vb[t % 3][2], vb[t % 3][3]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&st_empty[stage]);
        mbar_arrive(&p_empty[slot]);
      }
      if (++stage == kStages) { stage = 0; sphase ^= 1u; }
      if (++slot == kSlots) { slot = 0; pphase ^= 1u; }
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
  return 128 + (size_t)kStages * kStageBytes + kSlots * (kPBytes + sizeof(Msg)) + (2 * kBlocks + 1) * 4 +
         2 * sizeof(TokInfo) + 2 * 4 * NH * 4 + (kProdWarps + 2) * 4 + 8 + (2 * kStages + 4 + 2 * kSlots) * 8 + 8;
}

cudaError_t launch_sparse_attn(const AttnArgs& a, int grid, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.nh != NH || a.Dqk > kMaxDqk || a.Dqk % 16 != 0 || a.k > kMaxK || a.Dv > kMaxDv)
    return cudaErrorInvalidValue;
  // the warpgroups' register budgets add up to the launch allocation; a
  // build that allocated differently would make the increase wait forever
  const size_t smem = attn_smem();
  cudaError_t e = setup_once_per_device([smem]() {
    cudaFuncAttributes fa;
    cudaError_t r = cudaFuncGetAttributes(&fa, sparse_attn_kernel);
    if (r != cudaSuccess) return r;
    if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
    return cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  });
  if (e != cudaSuccess) return e;
  sparse_attn_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
