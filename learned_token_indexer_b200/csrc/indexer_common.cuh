// indexer_common.cuh -- pieces shared by the indexer kernels (score scan and
// fused prefill score + top-k): the tensor-core orientation, shared-memory
// geometry, and the epilogue's ReLU / head-weight / head-sum of eq. (1)
// (page "2.2.1 · DSA 与索引器", §1.1, eq. (1)).
//
// Orientation: keys on the MMA's M dimension (128 TMEM lanes), the query
// tokens' heads on N.  One accumulator column block of HI columns holds
// D[s, j] = q[t, j] . k[s] for one token t and 128 keys s, so the thread that
// owns TMEM lane s reduces over the heads in registers with no cross-thread
// traffic:  I[t, s] = sum_j w[t, j] * max(D[s, j], 0).
#pragma once
#include "sm100.cuh"

namespace dsa {

constexpr int kTileKeys = 128;     // keys per tile (MMA M)
constexpr int kSwizzleBytes = 128; // TMA 128B swizzle span = one K block row

// Bytes of one K-major operand row per 128-byte K block.
template <bool FP8>
struct ElemTraits {
  static constexpr int kBytes = FP8 ? 1 : 2;
  static constexpr int kElemsPerBlock = kSwizzleBytes / kBytes;  // 64 bf16 / 128 e4m3
  static constexpr uint32_t kFormat = FP8 ? 0u : 1u;             // idesc a/b format
};

__host__ __device__ constexpr int num_kblocks(int dI, int elem_bytes) {
  return (dI * elem_bytes + kSwizzleBytes - 1) / kSwizzleBytes;
}
// Number of 32-byte MMA K steps that hold data (the rest of the block is
// TMA zero fill and is skipped).
__host__ __device__ constexpr int num_ksteps(int dI, int elem_bytes) { return (dI * elem_bytes + 31) / 32; }

// Issue one tile's MMAs: D[128 x N] = A[128 keys x dI] * B[N x dI]^T.
// a_base / b_base: shared addresses of K block 0 of each operand; K block kb
// of an operand with R rows starts R*128 bytes later.
template <bool FP8>
__device__ __forceinline__ void issue_tile_mma(uint32_t d_tmem, uint32_t a_base, uint32_t b_base, int b_rows,
                                               int ksteps, uint32_t idesc) {
  for (int ks = 0; ks < ksteps; ++ks) {
    const int kb = ks >> 2;             // 4 steps of 32 bytes per 128-byte block
    const uint32_t koff = (ks & 3) * 32;
    const uint64_t ad = smem_desc_sw128(a_base + kb * kTileKeys * kSwizzleBytes + koff);
    const uint64_t bd = smem_desc_sw128(b_base + kb * b_rows * kSwizzleBytes + koff);
    if constexpr (FP8)
      mma_fp8_ss(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
    else
      mma_bf16_ss(d_tmem, ad, bd, idesc, ks > 0 ? 1u : 0u);
  }
}

// Load HI accumulator columns (one token) of this thread's TMEM lane.
template <int HI>
__device__ __forceinline__ void tmem_load_heads(uint32_t taddr, uint32_t (&r)[HI]) {
  if constexpr (HI == 4) tmem_ld_32x32b_x4(taddr, r);
  else if constexpr (HI == 8) tmem_ld_32x32b_x8(taddr, r);
  else if constexpr (HI == 16) tmem_ld_32x32b_x16(taddr, r);
  else if constexpr (HI == 32) tmem_ld_32x32b_x32(taddr, r);
  else if constexpr (HI == 64) tmem_ld_32x32b_x64(taddr, r);
  else static_assert(HI == 4, "unsupported indexer head count");
}

// Eq. (1) for one (token, key): sum_j w_j * ReLU(D_j), fp32, heads in order.
template <int HI>
__device__ __forceinline__ float relu_weighted_head_sum(const uint32_t (&acc)[HI], const float* w_smem) {
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < HI; ++j) s = fmaf(w_smem[j], fmaxf(__uint_as_float(acc[j]), 0.0f), s);
  return s;
}

// Eq. (1) for TOK consecutive tokens of one accumulator (columns
// [j*HI, (j+1)*HI) hold token j's heads) and this thread's key.  TMEM is read
// in units of up to 32 columns, loading unit u+1 while unit u is reduced; each
// token keeps 4 independent partial sums so the FMA chain does not serialise.
// After the last load the accumulator is handed back (`acc_empty`, one arrive
// per warp) before the last unit is reduced.
template <int HI, int TOK>
__device__ __forceinline__ void group_head_sums(uint32_t taddr, const float* w_smem, float (&score)[TOK],
                                                uint64_t* acc_empty, uint32_t lane) {
  constexpr int UW = HI < 32 ? HI : 32;      // columns per unit
  constexpr int UPT = HI / UW;               // units per token
  constexpr int NU = TOK * UPT;
  float2 part[TOK][2];
#pragma unroll
  for (int j = 0; j < TOK; ++j) part[j][0] = part[j][1] = make_float2(0.0f, 0.0f);
  uint32_t buf[2][UW];
  auto load = [&](int u, uint32_t (&r)[UW]) {
    const uint32_t col = (uint32_t)((u / UPT) * HI + (u % UPT) * UW);
    if constexpr (UW == 4) tmem_ld_32x32b_x4(taddr + col, r);
    else if constexpr (UW == 8) tmem_ld_32x32b_x8(taddr + col, r);
    else if constexpr (UW == 16) tmem_ld_32x32b_x16(taddr + col, r);
    else tmem_ld_32x32b_x32(taddr + col, r);
  };
  load(0, buf[0]);
  tmem_wait_ld(buf[0]);
#pragma unroll
  for (int u = 0; u < NU; ++u) {
    if (u + 1 < NU) load(u + 1, buf[(u + 1) & 1]);
    const int j = u / UPT;
    const float4* w = reinterpret_cast<const float4*>(w_smem + j * HI + (u % UPT) * UW);
#pragma unroll
    for (int h = 0; h < UW; h += 4) {
      const float4 w4 = w[h >> 2];   // four heads' weights in one shared load
      const float2 x0 = make_float2(fmaxf(__uint_as_float(buf[u & 1][h]), 0.0f),
                                    fmaxf(__uint_as_float(buf[u & 1][h + 1]), 0.0f));
      const float2 x1 = make_float2(fmaxf(__uint_as_float(buf[u & 1][h + 2]), 0.0f),
                                    fmaxf(__uint_as_float(buf[u & 1][h + 3]), 0.0f));
      part[j][0] = ffma2(make_float2(w4.x, w4.y), x0, part[j][0]);
      part[j][1] = ffma2(make_float2(w4.z, w4.w), x1, part[j][1]);
    }
    if (u + 1 < NU) {
      tmem_wait_ld(buf[(u + 1) & 1]);
      if (u + 2 == NU) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
      }
    }
  }
  if (NU == 1) {
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(acc_empty);
  }
#pragma unroll
  for (int j = 0; j < TOK; ++j) score[j] = (part[j][0].x + part[j][1].x) + (part[j][0].y + part[j][1].y);
}

}  // namespace dsa
