// sparse_attn.cu -- eq. (3) of page "2.2.1 · DSA 与索引器" (§1.1): attention of
// every query head over the latent rows the selector picked, with its own
// QK logits and softmax (the indexer scores are not reused), the value being
// the first Dv columns of each selected latent row.  All heads of a token
// share one selected set (the key is shared, §1.1), so one gather of a row
// serves every head of the group.
//
// CTA = (query row, group of 16 heads), 4 warps.  Selected rows are gathered
// 32 at a time into shared memory with 16-byte cp.async (invalid slots are
// zero-filled), double buffered.  Warp w computes the logits of keys
// 8w..8w+7 for the 16 heads (bf16 mma.sync m16n8k16, fp32 accumulate); all
// warps then share the chunk's logits through shared memory, run the online
// softmax (base-2 exponent, running max / sum per head) and accumulate
// P.V for their quarter of the value columns.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kAttnThreads = 128;
constexpr int kHeadsPerCta = 16;
constexpr int kChunk = 32;
constexpr int kSPitch = kChunk + 1;     // fp32 logits row pitch
constexpr int kPPitch = kChunk + 8;     // bf16 probability row pitch (80 bytes)

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

}  // namespace

template <int DV>
__global__ void __launch_bounds__(kAttnThreads) sparse_attn_kernel(const AttnArgs a) {
  constexpr int kOT = DV / 32;    // 8-column O tiles per warp (each warp owns DV/4 columns)
  const int row = blockIdx.x;
  const int hg = blockIdx.y;
  const int Dqk = a.Dqk;
  const int pitch = Dqk * 2 + 16;            // bytes per smem row
  const int pieces = Dqk / 8;                // 16-byte pieces per row
  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t g = lane >> 2, c4 = lane & 3u;

  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* sQ = smem;                                  // [16][pitch]
  uint8_t* sC = sQ + kHeadsPerCta * pitch;             // [2][32][pitch]
  float* sS = reinterpret_cast<float*>(sC + 2 * kChunk * pitch);            // [2][16][33]
  uint16_t* sP = reinterpret_cast<uint16_t*>(sS + 2 * kHeadsPerCta * kSPitch); // [2][16][40]
  int32_t* sIdx = reinterpret_cast<int32_t*>(sP + 2 * kHeadsPerCta * kPPitch);  // [2][32]

  // Row geometry.
  const uint16_t* lat;
  int len;
  if (a.mode == 0) {
    lat = a.latent + (int64_t)(row / a.nq) * a.kv_len * Dqk;
    len = a.kv_len;
  } else {
    const int64_t lo = a.cu_seqlens[row];
    lat = a.latent + lo * Dqk;
    len = (int)(a.cu_seqlens[row + 1] - lo);
  }
  const int32_t* idx_row = a.idx + (int64_t)row * a.k;

  // Q rows of this head group (heads past H are zero).
  const int h0 = hg * kHeadsPerCta;
  for (int e = threadIdx.x; e < kHeadsPerCta * pieces; e += kAttnThreads) {
    const int hr = e / pieces, pc = e - hr * pieces;
    const bool v = h0 + hr < a.H;
    const uint16_t* src = a.q + ((int64_t)row * a.H + (v ? h0 + hr : 0)) * Dqk + pc * 8;
    cp_async16(smem_u32(sQ + hr * pitch + pc * 16), src, v);
  }
  const int nchunks = (a.k + kChunk - 1) / kChunk;
  auto issue_chunk = [&](int cidx, int buf) {
    if (threadIdx.x < kChunk) {
      const int slot = cidx * kChunk + threadIdx.x;
      int p = slot < a.k ? idx_row[slot] : -1;
      if (p < -1 || p >= len) {
        report_status(a.status, kStatusDeviceCheck, 0xA77Eu);
        p = -1;
      }
      sIdx[buf * kChunk + threadIdx.x] = p;
    }
    // the index loads above are read back after a barrier; here every thread
    // reads the slot's index itself to start its copies right away
    for (int e = threadIdx.x; e < kChunk * pieces; e += kAttnThreads) {
      const int rr = e / pieces, pc = e - rr * pieces;
      const int slot = cidx * kChunk + rr;
      int p = slot < a.k ? idx_row[slot] : -1;
      const bool v = p >= 0 && p < len;
      const uint16_t* src = lat + (int64_t)(v ? p : 0) * Dqk + pc * 8;
      cp_async16(smem_u32(sC + (buf * kChunk + rr) * pitch + pc * 16), src, v);
    }
    cp_async_commit();
  };
  issue_chunk(0, 0);

  float o[kOT][4];
#pragma unroll
  for (int j = 0; j < kOT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.0f, l_hi = 0.0f;   // rows g and g+8
  const uint32_t sQa = smem_u32(sQ);

  for (int cidx = 0; cidx < nchunks; ++cidx) {
    const int buf = cidx & 1;
    cp_async_wait<0>();
    __syncthreads();
    if (cidx + 1 < nchunks) issue_chunk(cidx + 1, buf ^ 1);
    const uint32_t sCa = smem_u32(sC + buf * kChunk * pitch);

    // ---- logits of keys 8w..8w+7 for the 16 heads
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int ks = 0; ks < Dqk / 16; ++ks) {
      uint32_t a0, a1, a2, a3, b0, b1;
      ldsm_x4(sQa + (lane & 15) * pitch + (ks * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
      const uint32_t l16 = lane & 15;
      ldsm_x2(sCa + (warp * 8 + (l16 & 7)) * pitch + (ks * 16 + (l16 >> 3) * 8) * 2, b0, b1);
      mma_16816(s, a0, a1, a2, a3, b0, b1);
    }
    float* S = sS + buf * kHeadsPerCta * kSPitch;
    {
      const int kc = warp * 8 + 2 * c4;
      const bool v0 = sIdx[buf * kChunk + kc] >= 0, v1 = sIdx[buf * kChunk + kc + 1] >= 0;
      S[g * kSPitch + kc] = v0 ? s[0] * a.scale_log2 : -INFINITY;
      S[g * kSPitch + kc + 1] = v1 ? s[1] * a.scale_log2 : -INFINITY;
      S[(g + 8) * kSPitch + kc] = v0 ? s[2] * a.scale_log2 : -INFINITY;
      S[(g + 8) * kSPitch + kc + 1] = v1 ? s[3] * a.scale_log2 : -INFINITY;
    }
    __syncthreads();

    // ---- online softmax for rows g, g+8 (quad c4 reads keys 8*c4..8*c4+7)
    float alpha_lo, alpha_hi;
    {
      float x_lo[8], x_hi[8];
      float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        x_lo[e] = S[g * kSPitch + c4 * 8 + e];
        x_hi[e] = S[(g + 8) * kSPitch + c4 * 8 + e];
        mx_lo = fmaxf(mx_lo, x_lo[e]);
        mx_hi = fmaxf(mx_hi, x_hi[e]);
      }
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
      const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
      const float mu_lo = mn_lo == -INFINITY ? 0.0f : mn_lo;
      const float mu_hi = mn_hi == -INFINITY ? 0.0f : mn_hi;
      alpha_lo = exp2f(m_lo - mu_lo);
      alpha_hi = exp2f(m_hi - mu_hi);
      float sum_lo = 0.f, sum_hi = 0.f;
      uint32_t p_lo[4], p_hi[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float p0 = exp2f(x_lo[e] - mu_lo), p1 = exp2f(x_lo[e + 1] - mu_lo);
        const float q0 = exp2f(x_hi[e] - mu_hi), q1 = exp2f(x_hi[e + 1] - mu_hi);
        sum_lo += p0 + p1;
        sum_hi += q0 + q1;
        p_lo[e / 2] = pack_bf16(p0, p1);
        p_hi[e / 2] = pack_bf16(q0, q1);
      }
      sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 1);
      sum_lo += __shfl_xor_sync(0xffffffffu, sum_lo, 2);
      sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 1);
      sum_hi += __shfl_xor_sync(0xffffffffu, sum_hi, 2);
      l_lo = l_lo * alpha_lo + sum_lo;
      l_hi = l_hi * alpha_hi + sum_hi;
      m_lo = mn_lo;
      m_hi = mn_hi;
      if (c4 == warp) {
        uint16_t* P = sP + buf * kHeadsPerCta * kPPitch;
        *reinterpret_cast<uint4*>(P + g * kPPitch + c4 * 8) = make_uint4(p_lo[0], p_lo[1], p_lo[2], p_lo[3]);
        *reinterpret_cast<uint4*>(P + (g + 8) * kPPitch + c4 * 8) = make_uint4(p_hi[0], p_hi[1], p_hi[2], p_hi[3]);
      }
    }
#pragma unroll
    for (int j = 0; j < kOT; ++j) {
      o[j][0] *= alpha_lo;
      o[j][1] *= alpha_lo;
      o[j][2] *= alpha_hi;
      o[j][3] *= alpha_hi;
    }
    __syncthreads();

    // ---- O[:, warp quarter] += P (16 x 32) . V (32 x DV/4)
    const uint32_t sPa = smem_u32(sP + buf * kHeadsPerCta * kPPitch);
#pragma unroll
    for (int ks = 0; ks < kChunk / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(sPa + (lane & 15) * (kPPitch * 2) + (ks * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
      const uint32_t mi = lane >> 3;
      const uint32_t key = ks * 16 + (mi & 1u) * 8 + (lane & 7u);
#pragma unroll
      for (int j = 0; j < kOT; j += 2) {
        const int v0 = (int)warp * (DV / 4) + j * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sCa + key * pitch + (v0 + (mi >> 1) * 8) * 2, b0, b1, b2, b3);
        mma_16816(o[j], a0, a1, a2, a3, b0, b1);
        mma_16816(o[j + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }

  // ---- normalise and store
  const float inv_lo = l_lo > 0.f ? 1.0f / l_lo : 0.0f;
  const float inv_hi = l_hi > 0.f ? 1.0f / l_hi : 0.0f;
  const int hlo = h0 + (int)g, hhi = h0 + (int)g + 8;
#pragma unroll
  for (int j = 0; j < kOT; ++j) {
    const int col = (int)warp * (DV / 4) + j * 8 + 2 * (int)c4;
    if (hlo < a.H)
      *reinterpret_cast<uint32_t*>(a.out + ((int64_t)row * a.H + hlo) * DV + col) =
          pack_bf16(o[j][0] * inv_lo, o[j][1] * inv_lo);
    if (hhi < a.H)
      *reinterpret_cast<uint32_t*>(a.out + ((int64_t)row * a.H + hhi) * DV + col) =
          pack_bf16(o[j][2] * inv_hi, o[j][3] * inv_hi);
  }
  if (a.lse && warp == 0 && c4 == 0) {
    const float ln2 = 0.6931471805599453f;
    if (hlo < a.H) a.lse[(int64_t)row * a.H + hlo] = l_lo > 0.f ? m_lo * ln2 + logf(l_lo) : -INFINITY;
    if (hhi < a.H) a.lse[(int64_t)row * a.H + hhi] = l_hi > 0.f ? m_hi * ln2 + logf(l_hi) : -INFINITY;
  }
}

static size_t attn_smem_bytes(int Dqk) {
  const size_t pitch = (size_t)Dqk * 2 + 16;
  return kHeadsPerCta * pitch + 2 * kChunk * pitch + 2 * kHeadsPerCta * kSPitch * 4 +
         2 * kHeadsPerCta * kPPitch * 2 + 2 * kChunk * 4;
}

template <int DV>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t stream) {
  const size_t smem = attn_smem_bytes(a.Dqk);
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.rows, (a.H + kHeadsPerCta - 1) / kHeadsPerCta);
  sparse_attn_kernel<DV><<<grid, kAttnThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  switch (a.Dv) {
    case 64: return launch_attn_t<64>(a, stream);
    case 128: return launch_attn_t<128>(a, stream);
    case 256: return launch_attn_t<256>(a, stream);
    case 512: return launch_attn_t<512>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
