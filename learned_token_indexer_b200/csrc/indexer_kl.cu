// indexer_kl.cu -- eq. (8) of page "2.2.1 · DSA 与索引器" (§1.2): in the sparse
// training stage the indexer is fitted by a KL divergence computed only on
// each token's selected set S_t,
//
//     KL_t = D_KL( p_{t,S_t} || Softmax(I_{t,S_t}) ),
//
// with the teacher's weights divided by their retained mass over S_t (the
// remark after eq. (8)) and the scores I of eq. (1) recomputed on S_t.  The
// kernel returns KL_t and, for a loss L with dL/dKL_t = grad_scale, the
// gradients of L with respect to the indexer inputs q^I, w and k^I (the
// indexer is trained on its own loss; its inputs are detached from the main
// model, §1.2).  With g_s = grad_scale (softmax(I)_s - p_s):
//     dw_j = sum_s g_s ReLU(d_sj)               d_sj = q_j . k_s
//     dq_j = sum_s g_s w_j [d_sj > 0] k_s       (ReLU'(0) taken as 0)
//     dk_s = sum_j g_s w_j [d_sj > 0] q_j       (summed over every row t
//                                                that selected s)
//
// One CTA (4 warps) per query row.  The row's queries stay in shared memory;
// the selected key rows are gathered 64 at a time with 16-byte cp.async into
// three stages of padded rows (zero-filled for unused slots), two chunks
// ahead of the one being computed.  Two passes over the selected keys:
//   pass 1: D = K_S Q^T on mma.sync (warp w owns keys 16w..16w+15 of a chunk,
//           all heads), I_s = sum_j w_j ReLU(D_sj) -> shared memory;
//   row:    softmax over S_t, teacher renormalisation, KL_t, g_s;
//   pass 2: D is recomputed; dw accumulates in registers; the bf16 matrix
//           G_sj = g_s w_j [D_sj > 0] is the A operand of dk = G Q (taken
//           straight from the D accumulators) and, through shared memory,
//           of dq = G^T K_S (warp w owns heads 16w..16w+15).  dk rows are
//           added to global memory with float4 atomics (lane pairs swap
//           halves of their accumulator fragments to form 4 columns).
// Chunks whose slots are all unused are skipped, so short rows (t < k) cost
// what they select.  The heads are padded to 64 with zero queries and zero
// weights (exact: their D, ReLU and G are 0).
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kChunk = 64;       // selected keys per chunk
constexpr int kHP = 64;          // heads, padded
constexpr int kThreads = 128;
constexpr int kStages = 3;       // key-chunk stages in flight (two prefetched)
constexpr int kMaxChunks = kMaxKLTopk / kChunk;

template <int DI>
struct KLGeom {
  static constexpr int kPitch = DI * 2 + 16;       // bytes per Q / K row: 8 rows hit 8 bank groups
  static constexpr int kKsteps = DI / 16;
  static constexpr int kNT = DI / 8;               // 8-wide d^I tiles
  static constexpr int kPieces = DI / 8;           // 16-byte pieces per row
  static constexpr int kStageBytes = kChunk * kPitch;
  static constexpr int kQBytes = kHP * kPitch;
  static constexpr int kGPitch = kHP * 2 + 16;     // G rows (64 heads, bf16)
  static constexpr int kGBytes = kChunk * kGPitch;
  // shared memory: Q | K stages | G | w | positions | dw partials | scratch | chunk list | I / g
  static constexpr int kOffK = kQBytes;
  static constexpr int kOffG = kOffK + kStages * kStageBytes;
  static constexpr int kOffW = kOffG + kGBytes;
  static constexpr int kOffPos = kOffW + kHP * 4;
  static constexpr int kOffDw = kOffPos + kStages * kChunk * 4;
  static constexpr int kOffRed = kOffDw + 4 * kHP * 4;
  static constexpr int kOffList = kOffRed + 16 * 4;
  static constexpr int kOffI = kOffList + (kMaxChunks + 4) * 4;
  static size_t smem_bytes(int k) { return (size_t)kOffI + (size_t)k * 4; }
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
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
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Sum / max over the CTA's 4 warps (every thread gets the result).
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  return r;
}
__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const float r = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  return r;
}

// D[16 keys x 64 heads] of warp `warp` for the chunk in `stage` (fp32, mma C layout:
// d[nt][0..1] = key g, heads 8nt+2c..; d[nt][2..3] = key g+8).
template <int DI>
__device__ __forceinline__ void key_head_dots(uint32_t stage, uint32_t sq, int warp, int lane, float (&d)[8][4]) {
  using G = KLGeom<DI>;
  const int mi = lane >> 3;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) d[nt][0] = d[nt][1] = d[nt][2] = d[nt][3] = 0.f;
#pragma unroll
  for (int kk = 0; kk < G::kKsteps; ++kk) {
    uint32_t af[4];
    ldsm_x4(stage + (16 * warp + (mi & 1) * 8 + (lane & 7)) * G::kPitch + (16 * kk + (mi >> 1) * 8) * 2, af);
#pragma unroll
    for (int nt = 0; nt < 8; nt += 2) {
      uint32_t bf[4];
      ldsm_x4(sq + (8 * (nt + (mi >> 1)) + (lane & 7)) * G::kPitch + (16 * kk + (mi & 1) * 8) * 2, bf);
      mma16816(d[nt], af, bf[0], bf[1]);
      mma16816(d[nt + 1], af, bf[2], bf[3]);
    }
  }
}

template <int DI>
__global__ void __launch_bounds__(kThreads, 2) indexer_kl_kernel(const KLArgs a) {
  using G = KLGeom<DI>;
  extern __shared__ __align__(128) uint8_t smem[];
  float* sW = reinterpret_cast<float*>(smem + G::kOffW);
  int* sPos = reinterpret_cast<int*>(smem + G::kOffPos);
  float* sDw = reinterpret_cast<float*>(smem + G::kOffDw);
  float* sRed = reinterpret_cast<float*>(smem + G::kOffRed);
  int* sList = reinterpret_cast<int*>(smem + G::kOffList);
  float* sI = reinterpret_cast<float*>(smem + G::kOffI);
  const uint32_t sq = smem_u32(smem);
  const uint32_t sk = smem_u32(smem + G::kOffK);
  const uint32_t sg = smem_u32(smem + G::kOffG);

  const int row = blockIdx.x;
  const int b = row / a.nq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3, mi = lane >> 3;
  const int HI = a.HI, K = a.k;
  const int nchunks = (K + kChunk - 1) / kChunk;
  const int32_t* idx_row = a.idx + (int64_t)row * K;
  const float* teacher_row = a.teacher + (int64_t)row * K;
  const uint16_t* kbase = a.kI + (int64_t)b * a.kv_len * DI;
  const bool backward = a.dq || a.dw || a.dk || a.grad_logits;

  // Queries (zero rows past H^I) and head weights (zero past H^I).
  for (int p = tid; p < kHP * G::kPieces; p += kThreads) {
    const int h = p / G::kPieces, pc = p % G::kPieces;
    const uint16_t* src = a.q + ((int64_t)row * HI + (h < HI ? h : 0)) * DI + pc * 8;
    cp_async16(sq + h * G::kPitch + pc * 16, src, h < HI ? 16u : 0u);
  }
  cp_async_commit();
  if (tid < kHP) sW[tid] = tid < HI ? a.w[(int64_t)row * HI + tid] : 0.f;
  for (int s = tid; s < K; s += kThreads) sI[s] = -INFINITY;
  // Which chunks hold a valid slot; report indices outside [-1, kv_len).
  for (int ch = warp; ch < nchunks; ch += 4) {
    bool any = false, bad = false;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int s = ch * kChunk + h * 32 + lane;
      if (s < K) {
        const int p = idx_row[s];
        any |= (p >= 0 && p < a.kv_len);
        bad |= (p < -1 || p >= a.kv_len);
      }
    }
    any = __any_sync(0xffffffffu, any);
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      sList[4 + ch] = any ? 1 : 0;
      if (bad) report_status(a.status, kStatusDeviceCheck, 0xA77Eu);
    }
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int ch = 0; ch < nchunks; ++ch)
      if (sList[4 + ch]) sList[4 + n++] = ch;   // compacts in place (n <= ch)
    sList[0] = n;
  }
  __syncthreads();
  const int nl = sList[0];
  const int* list = sList + 4;

  float wr[8][2];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    wr[nt][0] = sW[8 * nt + 2 * c];
    wr[nt][1] = sW[8 * nt + 2 * c + 1];
  }

  // Gather the selected key rows of chunk list[v % nl] into stage v % kStages.
  auto load_chunk = [&](int v) {
    const int ch = list[v % nl];
    const int st = v % kStages;
    const uint32_t dst0 = sk + st * G::kStageBytes;
    for (int p = tid; p < kChunk * G::kPieces; p += kThreads) {
      const int r = p / G::kPieces, pc = p % G::kPieces;
      const int s = ch * kChunk + r;
      const int pos = s < K ? idx_row[s] : -1;
      const bool ok = pos >= 0 && pos < a.kv_len;
      cp_async16(dst0 + r * G::kPitch + pc * 16, kbase + (int64_t)(ok ? pos : 0) * DI + pc * 8, ok ? 16u : 0u);
      if (pc == 0) sPos[st * kChunk + r] = ok ? pos : -1;
    }
  };

  float dwacc[8][2];
  float dqacc[G::kNT][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) dwacc[nt][0] = dwacc[nt][1] = 0.f;
#pragma unroll
  for (int nt = 0; nt < G::kNT; ++nt) dqacc[nt][0] = dqacc[nt][1] = dqacc[nt][2] = dqacc[nt][3] = 0.f;

  bool row_ok = nl > 0;
  float kl = 0.f;
  // Row step between the passes: softmax over S_t, teacher renormalisation,
  // KL_t (accumulated per thread in kl) and g_s (written over sI).  Returns
  // false when the teacher has no mass on S_t.
  auto row_softmax_kl = [&]() -> bool {
    float mx = -INFINITY;
    for (int s = tid; s < K; s += kThreads) mx = fmaxf(mx, sI[s]);
    mx = block_max(mx, sRed);
    float z = 0.f, mass = 0.f;
    for (int s = tid; s < K; s += kThreads) {
      const float x = sI[s];
      if (x != -INFINITY) {
        z += expf(x - mx);
        mass += teacher_row[s];
      }
    }
    z = block_sum(z, sRed);
    mass = block_sum(mass, sRed);
    if (!(mass > 0.f)) return false;
    const float log_z = logf(z), inv_mass = 1.f / mass;
    for (int s = tid; s < K; s += kThreads) {
      const float x = sI[s];
      float gs = 0.f;
      if (x != -INFINITY) {
        const float ph = teacher_row[s] * inv_mass;
        const float lq = (x - mx) - log_z;
        if (ph > 0.f) kl += ph * (logf(ph) - lq);
        gs = a.grad_scale * (expf(lq) - ph);
      }
      sI[s] = gs;
      if (a.grad_logits) a.grad_logits[(int64_t)row * K + s] = gs;
    }
    __syncthreads();
    return true;
  };

  const int V = backward ? 2 * nl : nl;
  if (V > 0) load_chunk(0);
  cp_async_commit();
  if (V > 1) load_chunk(1);
  cp_async_commit();
  for (int v = 0; v < V; ++v) {
    // Chunk v has landed once at most one newer group is pending; after the
    // barrier every thread is done with chunk v - 1, whose stage the load of
    // chunk v + 2 reuses.
    cp_async_wait<1>();
    __syncthreads();
    if (v + 2 < V) load_chunk(v + 2);
    cp_async_commit();
    const int st = v % kStages;
    const int ch = list[v % nl];
    const uint32_t stage = sk + st * G::kStageBytes;
    const int slot0 = ch * kChunk + 16 * warp + g, slot1 = slot0 + 8;

    if (v == nl && !(row_ok = row_softmax_kl())) break;

    float d[8][4];
    key_head_dots<DI>(stage, sq, warp, lane, d);

    if (v < nl) {
      // ---- pass 1: I_s = sum_j w_j ReLU(D_sj) ----
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s0 += wr[nt][0] * fmaxf(d[nt][0], 0.f) + wr[nt][1] * fmaxf(d[nt][1], 0.f);
        s1 += wr[nt][0] * fmaxf(d[nt][2], 0.f) + wr[nt][1] * fmaxf(d[nt][3], 0.f);
      }
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (c == 0) {
        if (slot0 < K && sPos[st * kChunk + 16 * warp + g] >= 0) sI[slot0] = s0 + 0.f;
        if (slot1 < K && sPos[st * kChunk + 16 * warp + g + 8] >= 0) sI[slot1] = s1 + 0.f;
      }
    } else {
      // ---- pass 2: dw, G, dk = G Q, dq = G^T K ----
      const float g0 = slot0 < K ? sI[slot0] : 0.f;
      const float g1 = slot1 < K ? sI[slot1] : 0.f;
      uint32_t ga[8][2];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        dwacc[nt][0] += g0 * fmaxf(d[nt][0], 0.f) + g1 * fmaxf(d[nt][2], 0.f);
        dwacc[nt][1] += g0 * fmaxf(d[nt][1], 0.f) + g1 * fmaxf(d[nt][3], 0.f);
        ga[nt][0] = pack_bf16(d[nt][0] > 0.f ? g0 * wr[nt][0] : 0.f, d[nt][1] > 0.f ? g0 * wr[nt][1] : 0.f);
        ga[nt][1] = pack_bf16(d[nt][2] > 0.f ? g1 * wr[nt][0] : 0.f, d[nt][3] > 0.f ? g1 * wr[nt][1] : 0.f);
        st_shared_u32(sg + (16 * warp + g) * G::kGPitch + (8 * nt + 2 * c) * 2, ga[nt][0]);
        st_shared_u32(sg + (16 * warp + g + 8) * G::kGPitch + (8 * nt + 2 * c) * 2, ga[nt][1]);
      }
      if (a.dk) {
        // Even lanes of a pair add 4 columns of key g, odd lanes 4 columns of key g + 8.
        const bool odd = c & 1;
        const int pos = sPos[st * kChunk + 16 * warp + g + (odd ? 8 : 0)];
        float* dkrow = a.dk + ((int64_t)b * a.kv_len + (pos >= 0 ? pos : 0)) * DI + 2 * (c & ~1);
#pragma unroll
        for (int half = 0; half < (G::kNT + 7) / 8; ++half) {
          constexpr int kW = G::kNT < 8 ? G::kNT : 8;
          float acc[kW][4];
#pragma unroll
          for (int j = 0; j < kW; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t af[4] = {ga[2 * kk][0], ga[2 * kk][1], ga[2 * kk + 1][0], ga[2 * kk + 1][1]};
#pragma unroll
            for (int j = 0; j < kW; j += 2) {
              uint32_t bf[4];
              ldsm_x4_t(sq + (16 * kk + (mi & 1) * 8 + (lane & 7)) * G::kPitch + 8 * (half * 8 + j + (mi >> 1)) * 2,
                        bf);
              mma16816(acc[j], af, bf[0], bf[1]);
              mma16816(acc[j + 1], af, bf[2], bf[3]);
            }
          }
#pragma unroll
          for (int j = 0; j < kW; ++j) {
            const float r0 = __shfl_xor_sync(0xffffffffu, odd ? acc[j][0] : acc[j][2], 1);
            const float r1 = __shfl_xor_sync(0xffffffffu, odd ? acc[j][1] : acc[j][3], 1);
            const float4 v4 = odd ? make_float4(r0, r1, acc[j][2], acc[j][3]) : make_float4(acc[j][0], acc[j][1], r0, r1);
            if (pos >= 0) atomicAdd(reinterpret_cast<float4*>(dkrow + 8 * (half * 8 + j)), v4);
          }
        }
      }
      __syncthreads();   // G complete
      if (a.dq) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint32_t af[4];
          ldsm_x4_t(sg + (16 * kk + (mi >> 1) * 8 + (lane & 7)) * G::kGPitch + (16 * warp + (mi & 1) * 8) * 2, af);
#pragma unroll
          for (int nt = 0; nt < G::kNT; nt += 2) {
            uint32_t bf[4];
            ldsm_x4_t(stage + (16 * kk + (mi & 1) * 8 + (lane & 7)) * G::kPitch + 8 * (nt + (mi >> 1)) * 2, bf);
            mma16816(dqacc[nt], af, bf[0], bf[1]);
            mma16816(dqacc[nt + 1], af, bf[2], bf[3]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();
  if (row_ok && !backward) row_ok = row_softmax_kl();

  // ---- outputs ----
  kl = block_sum(kl, sRed);
  if (tid == 0) a.kl[row] = row_ok ? kl : 0.f;
  if (!row_ok) {
    if (a.grad_logits)
      for (int s = tid; s < K; s += kThreads) a.grad_logits[(int64_t)row * K + s] = 0.f;
    if (a.dw)
      for (int h = tid; h < HI; h += kThreads) a.dw[(int64_t)row * HI + h] = 0.f;
    if (a.dq)
      for (int e = tid; e < HI * DI; e += kThreads) a.dq[(int64_t)row * HI * DI + e] = 0.f;
    return;
  }
  if (!backward) return;
  if (a.dq) {
#pragma unroll
    for (int nt = 0; nt < G::kNT; ++nt) {
      const int h0 = 16 * warp + g, h1 = h0 + 8, col = 8 * nt + 2 * c;
      if (h0 < HI)
        *reinterpret_cast<float2*>(a.dq + ((int64_t)row * HI + h0) * DI + col) = make_float2(dqacc[nt][0], dqacc[nt][1]);
      if (h1 < HI)
        *reinterpret_cast<float2*>(a.dq + ((int64_t)row * HI + h1) * DI + col) = make_float2(dqacc[nt][2], dqacc[nt][3]);
    }
  }
  if (a.dw) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x = dwacc[nt][e];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (g == 0) sDw[warp * kHP + 8 * nt + 2 * c + e] = x;
      }
    }
    __syncthreads();
    if (tid < HI)
      a.dw[(int64_t)row * HI + tid] = (sDw[tid] + sDw[kHP + tid]) + (sDw[2 * kHP + tid] + sDw[3 * kHP + tid]);
  }
}

}  // namespace

size_t indexer_kl_smem_bytes(int dI, int k) {
  switch (dI) {
    case 32: return KLGeom<32>::smem_bytes(k);
    case 64: return KLGeom<64>::smem_bytes(k);
    case 128: return KLGeom<128>::smem_bytes(k);
    default: return 0;
  }
}

cudaError_t launch_indexer_kl(int dI, const KLArgs& a, cudaStream_t stream) {
  const size_t smem = indexer_kl_smem_bytes(dI, a.k);
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<a.rows, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
  };
  switch (dI) {
    case 32: return go(indexer_kl_kernel<32>);
    case 64: return go(indexer_kl_kernel<64>);
    case 128: return go(indexer_kl_kernel<128>);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
