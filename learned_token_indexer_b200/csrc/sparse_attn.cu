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
// here.  (Products with >= 128 rows per operand run on tcgen05 elsewhere.)
//
// Work item = (query row, group of 16 heads); persistent grid, one CTA per SM.
//   warps 0-3  producer: validate and compact the row's indices, then gather
//              the selected latent rows 64 at a time with 16-byte cp.async into
//              three 72 KB stages (128B-swizzled 64-column blocks);
//   warps 4-7  compute: the 16 x Dqk query as register-resident A fragments;
//              warp w forms the logits of keys 16w..16w+15 of the chunk
//              (S = Q C^T), the per-head running max / rescale (base-2
//              exponent) is shared through shared memory, probabilities go to
//              shared memory in bf16, and warp w accumulates O for value
//              columns [128w, 128w+128) (O += P V) in fp32 registers.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kChunk = 64;            // keys per chunk
constexpr int NH = 16;                // heads per work item (mma M)
constexpr int kStages = 3;
constexpr int kMaxCB = 9;             // 64-column blocks per row (Dqk <= 576)
constexpr int kBlockBytes = kChunk * 128;
constexpr int kStageBytes = kMaxCB * kBlockBytes;
constexpr int kMaxK = 2048;
constexpr int kMaxKsteps = kMaxCB * 4;  // 16-column steps of Dqk
constexpr int kThreads = 256;
constexpr int kProd = 128;             // producer threads (warps 0-3)
constexpr int kPBytes = NH * kChunk * 2;

struct TokInfo {
  uint32_t nvalid;
  uint32_t nchunks;
};

__device__ __forceinline__ void row_geometry(const AttnArgs& a, int r, int64_t& base_row, int& len) {
  if (a.mode == 0) {
    base_row = (int64_t)(r / a.nq) * a.kv_len;
    len = a.kv_len;
  } else {
    base_row = a.cu_seqlens[r];
    len = (int)(a.cu_seqlens[r + 1] - base_row);
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// Byte offset of (row r, 16-byte chunk ch) inside a 128B-swizzled block.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t ch) { return r * 128u + ((ch ^ (r & 7u)) << 4); }

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) sparse_attn_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // the 128B swizzle here is address arithmetic (cp.async / ldmatrix), so
  // 128-byte alignment of the blocks is enough
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* sC = base;                                                  // [3][9][64][128B]
  uint8_t* sP = sC + kStages * kStageBytes;                            // [2][16 heads][64 keys] bf16, swizzled
  uint16_t* sList = reinterpret_cast<uint16_t*>(sP + 2 * kPBytes);     // [kMaxK] compacted slot numbers
  TokInfo* sTok = reinterpret_cast<TokInfo*>(sList + kMaxK);           // [2]
  float* sMax = reinterpret_cast<float*>(sTok + 2);                    // [2][4 warps][16]
  float* sSum = sMax + 2 * 4 * NH;                                     // [4][16]
  uint32_t* sWarpCnt = reinterpret_cast<uint32_t*>(sSum + 4 * NH);     // [4]
  uint32_t* sBcast = sWarpCnt + 4;                                     // [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(sBcast + 2) + 7) & ~uintptr_t(7));
  uint64_t* st_full = bars;               // [3] (producer threads, cp.async arrive)
  uint64_t* st_empty = bars + kStages;    // [3] (4 compute warps)
  uint64_t* tok_full = bars + 2 * kStages;   // [2]
  uint64_t* tok_empty = tok_full + 2;        // [2] (4 compute warps)
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(tok_empty + 2);

  const uint32_t warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&st_full[i], kProd);
      mbar_init(&st_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tok_full[i], 1);
      mbar_init(&tok_empty[i], 4);
    }
    *abort_flag = 0u;
    mbar_fence_init();
  }
  __syncthreads();
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};
  const int hg_count = (a.H + NH - 1) / NH;
  const int items = a.rows * hg_count;
  const int CB = a.cb;

  if (warp < 4) {
    // ------------------------------------------------------------------ producer
    const uint32_t pt = threadIdx.x;    // 0..127
    int tslot = 0, stage = 0;
    uint32_t tphase = 0, sphase = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int r = item / hg_count;
      int64_t base_row;
      int len;
      row_geometry(a, r, base_row, len);
      const int32_t* idx_row = a.idx + (int64_t)r * a.k;
      // ---- compact the valid indices (slot order kept) into sList
      named_bar_sync(2, kProd);          // the previous row's list is no longer read
      constexpr int kPer = kMaxK / kProd;  // 16 slots per thread
      int32_t pos[kPer];
      uint32_t vmask = 0;
#pragma unroll
      for (int e = 0; e < kPer; ++e) {
        const int slot = (int)pt * kPer + e;
        const int p = slot < a.k ? __ldg(idx_row + slot) : -1;
        if (slot < a.k && (p < -1 || p >= len)) report_status(a.status, kStatusDeviceCheck, 0xA77Eu);
        pos[e] = p;
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
      // ---- gather 64 selected rows per chunk.  Thread pt copies 16-byte
      // chunk (pt & 7) of every 128-byte block of rows (pt >> 3) + 16j,
      // j = 0..3: eight consecutive lanes cover one 128-byte segment.  The
      // four row numbers of the next chunk are fetched while waiting for a
      // free stage, so no global load sits between the copies.
      const uint32_t ch = pt & 7u, r0 = pt >> 3;
      int64_t rows[4];
      auto fetch_rows = [&](uint32_t c) {
        const uint32_t nk = min((uint32_t)kChunk, nvalid - c * kChunk);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t rr = r0 + 16u * j;
          rows[j] = base_row + __ldg(idx_row + sList[c * kChunk + (rr < nk ? rr : 0u)]);
        }
      };
      if (nchunks > 0) fetch_rows(0);
      for (uint32_t c = 0; c < nchunks; ++c) {
        if (ok) ok = mbar_wait(&st_empty[stage], sphase ^ 1u, ctl, 0x2102);
        if (ok) {
          uint8_t* dst = sC + stage * kStageBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t rr = r0 + 16u * j;
            const uint16_t* src = a.latent + rows[j] * a.Dqk;
            for (int cb = 0; cb < CB; ++cb) {
              const int col = cb * 64 + (int)ch * 8;
              const bool in = col < a.Dqk;
              cp_async16(smem_u32(dst + cb * kBlockBytes + swz(rr, ch)), src + (in ? col : 0), in ? 16u : 0u);
            }
          }
        }
        cp_async_arrive_noinc(&st_full[stage]);
        if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        if (c + 1 < nchunks) fetch_rows(c + 1);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else {
    // ------------------------------------------------------------------ compute
    const uint32_t cw = warp - 4;                 // 0..3
    const uint32_t g = lane >> 2, c4 = lane & 3u; // mma fragment coordinates
    const int ksteps = a.ksteps;
    int tslot = 0, stage = 0;
    uint32_t tphase = 0, sphase = 0, pbuf = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
      const int r = item / hg_count, hg = item - r * hg_count;
      // queries of this head group -> A fragments (rows g, g+8; heads past H are zero)
      uint32_t qa[kMaxKsteps][4];
      {
        const int h0 = hg * NH + (int)g, h1 = h0 + 8;
        const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)r * a.H + h0) * a.Dqk);
        const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)r * a.H + h1) * a.Dqk);
        const bool v0 = h0 < a.H, v1 = h1 < a.H;
#pragma unroll
        for (int ks = 0; ks < kMaxKsteps; ++ks) {
          const bool in = ks < ksteps;
          const int e = ks * 8 + (int)c4;           // 32-bit element index (2 bf16 each)
          qa[ks][0] = (in && v0) ? __ldg(q0 + e) : 0u;
          qa[ks][1] = (in && v1) ? __ldg(q1 + e) : 0u;
          qa[ks][2] = (in && v0) ? __ldg(q0 + e + 4) : 0u;
          qa[ks][3] = (in && v1) ? __ldg(q1 + e + 4) : 0u;
        }
      }
      // the chunk count is broadcast after a barrier so every compute warp runs
      // the same number of barriers (0 chunks after a failed wait)
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

      float o[16][4];
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
      float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;   // heads g, g+8

      for (uint32_t c = 0; c < nchunks; ++c) {
        (void)mbar_wait(&st_full[stage], sphase, ctl, 0x2302);
        const uint32_t cbase = smem_u32(sC + stage * kStageBytes);
        // ---- S = Q C^T for keys 16cw..16cw+15 (two n-tiles of 8 keys)
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
        {
          // ldmatrix x4: matrices (keys 0-7, dims 0-7), (keys 0-7, dims 8-15),
          //                        (keys 8-15, dims 0-7), (keys 8-15, dims 8-15)
          const uint32_t mi = lane >> 3;
          const uint32_t key = cw * 16 + (mi >> 1) * 8 + (lane & 7);
          const uint32_t dh = mi & 1;   // which 8-dim half of the 16-dim step
#pragma unroll
          for (int ks = 0; ks < kMaxKsteps; ++ks) {
            if (ks < ksteps) {
              const uint32_t cb = (uint32_t)ks >> 2, ch = ((uint32_t)ks & 3u) * 2u + dh;
              uint32_t b0, b1, b2, b3;
              ldsm_x4(cbase + cb * kBlockBytes + swz(key, ch), b0, b1, b2, b3);
              mma16816(s0, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b0, b1);
              mma16816(s1, qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], b2, b3);
            }
          }
        }
        // ---- mask, scale, chunk max per head
        const uint32_t kbase = c * kChunk + cw * 16 + 2 * c4;   // key of s0[0]
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
        float* smx = sMax + pbuf * 4 * NH;
        if (c4 == 0) {
          smx[cw * NH + g] = mx_lo;
          smx[cw * NH + g + 8] = mx_hi;
        }
        named_bar_sync(1, 128);
        const float cm_lo = fmaxf(fmaxf(smx[g], smx[NH + g]), fmaxf(smx[2 * NH + g], smx[3 * NH + g]));
        const float cm_hi =
            fmaxf(fmaxf(smx[g + 8], smx[NH + g + 8]), fmaxf(smx[2 * NH + g + 8], smx[3 * NH + g + 8]));
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
        // P[head][key] (bf16), row = head, 128 bytes per row, swizzled 16-byte chunks
        {
          uint8_t* P = sP + pbuf * kPBytes;
          const uint32_t k0 = cw * 16 + 2 * c4;   // keys k0, k0+1 (n-tile 0) and k0+8, k0+9 (n-tile 1)
          *reinterpret_cast<uint32_t*>(P + swz(g, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p00, p01);
          *reinterpret_cast<uint32_t*>(P + swz(g + 8, k0 >> 3) + (k0 & 7) * 2) = pack_bf16(p02, p03);
          *reinterpret_cast<uint32_t*>(P + swz(g, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p10, p11);
          *reinterpret_cast<uint32_t*>(P + swz(g + 8, (k0 + 8) >> 3) + (k0 & 7) * 2) = pack_bf16(p12, p13);
        }
        // rescale the running output
        if (al_lo != 1.0f || al_hi != 1.0f) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            o[j][0] *= al_lo;
            o[j][1] *= al_lo;
            o[j][2] *= al_hi;
            o[j][3] *= al_hi;
          }
        }
        named_bar_sync(1, 128);
        // ---- O[:, 128cw .. 128cw+127] += P (16 x 64) V (64 x 128)
        {
          const uint32_t pbase = smem_u32(sP + pbuf * kPBytes);
          const uint32_t mi = lane >> 3;
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk) {
            uint32_t a0, a1, a2, a3;
            // A = P rows (heads) 0-15, keys 16kk..16kk+15
            ldsm_x4(pbase + swz(lane & 15u, (uint32_t)kk * 2u + (lane >> 4)), a0, a1, a2, a3);
            const uint32_t key = kk * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
              const uint32_t v0 = cw * 128 + j * 8 + (mi >> 1) * 8;   // value column of this matrix
              if ((int)v0 < a.Dv) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(cbase + (v0 >> 6) * kBlockBytes + swz(key, (v0 & 63) >> 3), b0, b1, b2, b3);
                mma16816(o[j], a0, a1, a2, a3, b0, b1);
                mma16816(o[j + 1], a0, a1, a2, a3, b2, b3);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&st_empty[stage]);
        if (++stage == kStages) { stage = 0; sphase ^= 1u; }
        pbuf ^= 1u;
      }
      // ---- finish the row: O / l, log-sum-exp
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
      l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
      l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
      if (c4 == 0) {
        sSum[cw * NH + g] = l_lo;
        sSum[cw * NH + g + 8] = l_hi;
      }
      named_bar_sync(1, 128);
      const float L_lo = sSum[g] + sSum[NH + g] + sSum[2 * NH + g] + sSum[3 * NH + g];
      const float L_hi = sSum[g + 8] + sSum[NH + g + 8] + sSum[2 * NH + g + 8] + sSum[3 * NH + g + 8];
      named_bar_sync(1, 128);   // sSum is reused by the next row
      const float i_lo = L_lo > 0.0f ? 1.0f / L_lo : 0.0f, i_hi = L_hi > 0.0f ? 1.0f / L_hi : 0.0f;
      const int h_lo = hg * NH + (int)g, h_hi = h_lo + 8;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int v = (int)cw * 128 + j * 8 + 2 * (int)c4;
        if (v < a.Dv) {
          if (h_lo < a.H)
            *reinterpret_cast<uint32_t*>(a.out + ((int64_t)r * a.H + h_lo) * a.Dv + v) =
                pack_bf16(o[j][0] * i_lo, o[j][1] * i_lo);
          if (h_hi < a.H)
            *reinterpret_cast<uint32_t*>(a.out + ((int64_t)r * a.H + h_hi) * a.Dv + v) =
                pack_bf16(o[j][2] * i_hi, o[j][3] * i_hi);
        }
      }
      if (a.lse && cw == 0 && c4 == 0) {
        const float ln2 = 0.69314718055994531f;
        if (h_lo < a.H) a.lse[(int64_t)r * a.H + h_lo] = L_lo > 0.0f ? (m_lo + log2f(L_lo)) * ln2 : -INFINITY;
        if (h_hi < a.H) a.lse[(int64_t)r * a.H + h_hi] = L_hi > 0.0f ? (m_hi + log2f(L_hi)) * ln2 : -INFINITY;
      }
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static size_t attn_smem() {
  return 128 + (size_t)kStages * kStageBytes + 2 * kPBytes + kMaxK * 2 + 2 * sizeof(TokInfo) +
         (2 * 4 * NH + 4 * NH) * 4 + 6 * 4 + 8 + (2 * kStages + 4) * 8 + 8;
}

cudaError_t launch_sparse_attn(const AttnArgs& a, int grid, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.nh != NH || a.cb > kMaxCB || a.k > kMaxK || a.Dv > 512) return cudaErrorInvalidValue;
  const size_t smem = attn_smem();
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  sparse_attn_kernel<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
