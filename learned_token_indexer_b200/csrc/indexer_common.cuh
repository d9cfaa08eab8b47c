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

}  // namespace dsa
