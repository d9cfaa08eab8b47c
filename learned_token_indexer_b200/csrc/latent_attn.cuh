// latent_attn.cuh -- pieces shared by the tcgen05 attention kernels over
// 576-column latent rows (latent_attn_decode.cu, latent_attn_dense.cu):
// packing, the 128-byte swizzled operand layout and register rebalancing.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace dsa {
namespace lattn {

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// Offset of 16-byte chunk `ch` (0..7) of row `n` in a block of the 128-byte
// swizzled layout (8-row, 1024-byte atoms; the chunk index is XOR-ed with the
// row's position in its atom).
__device__ __forceinline__ uint32_t swz_off(uint32_t n, uint32_t ch) {
  return (n >> 3) * 1024u + (n & 7u) * 128u + ((ch ^ (n & 7u)) << 4);
}

template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

}  // namespace lattn
}  // namespace dsa
