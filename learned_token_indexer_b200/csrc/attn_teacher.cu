// attn_teacher.cu -- the teacher of the sparse training stage (page "2.2.1 ·
// DSA 与索引器", §1.2, the remark after eq. (8), and eq. (16)): when the
// teacher comes from the current sparse main attention, token t's target on
// its selected set S_t is the heads' attention probabilities summed over the
// heads and L1-normalised along the positions,
//
//     p_{t,s} = sum_h a_h(s) / sum_{s' in S_t} sum_h a_h(s'),
//     a_h(s)  = exp(scale q_{t,h} . c_s - lse_{t,h}),
//
// where lse_{t,h} is the log-sum-exp of head h's logits over S_t that the
// sparse attention forward (eq. (3)) already returned.  This recomputes the
// attention scores of the selected set once, as a training step around DSA
// must (the forward never materialises them).
//
// One CTA (4 warps) per query row.  The row's head group (16 heads) lives in
// registers as mma.sync A fragments (rows = heads, columns = latent).  The
// selected slots are taken 32 at a time; warp w owns slots 8w..8w+7 of every
// chunk: it gathers their latent rows itself (one TMA bulk copy per row from
// lanes 0-7, completing on the warp's own mbarrier) into a two-deep ring of
// padded rows, forms their logits for all 16 heads, turns them into a_h(s)
// with the head's lse and sums over the heads with lane shuffles.  The warps
// never wait for one another until the row's end, where the per-slot sums
// (in shared memory) are L1-normalised.  Unused slots are not copied and
// their sums are never stored; columns past Dqk stay zero (the ring is
// zeroed once).  Heads past H have a zero query and contribute nothing.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {

namespace {

constexpr int kTChunk = 32;                    // selected rows per chunk (4 warps x 8)
constexpr int kTThreads = 128;
constexpr int kTMaxDqk = 576;
constexpr int kTKsteps = kTMaxDqk / 16;        // 36
constexpr int kTPitch = kTMaxDqk * 2 + 16;     // 1168 bytes: 8 rows hit 8 bank groups
constexpr int kTStageBytes = kTChunk * kTPitch;
constexpr int kTNH = 16;                       // heads per group (mma M)
constexpr int kTMaxChunks = kMaxTeacherTopk / kTChunk;
// shared memory: 2 stages | positions [2][32] | scratch | mbarriers [2 stages][4 warps] |
// abort flag | chunk list | per-slot sums
constexpr int kTOffPos = 2 * kTStageBytes;
constexpr int kTOffRed = kTOffPos + 2 * kTChunk * 4;
constexpr int kTOffBar = kTOffRed + 16 * 4;               // 8-byte aligned
constexpr int kTOffAbort = kTOffBar + 2 * 4 * 8;
constexpr int kTOffList = kTOffAbort + 16;
constexpr int kTOffP = kTOffList + (kTMaxChunks + 4) * 4;
static_assert(kTOffBar % 8 == 0, "mbarriers need 8-byte alignment");

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
               "{%0,%1,%2,%3};"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kTThreads, 2) attn_teacher_kernel(const TeacherArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  int* sPos = reinterpret_cast<int*>(smem + kTOffPos);
  float* sRed = reinterpret_cast<float*>(smem + kTOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTOffBar);   // [stage * 4 + warp]
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + kTOffAbort);
  int* sList = reinterpret_cast<int*>(smem + kTOffList);
  float* sP = reinterpret_cast<float*>(smem + kTOffP);
  const uint32_t sc = smem_u32(smem);

  const int row = blockIdx.x;
  const int b = row / a.nq;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c4 = lane & 3, mi = lane >> 3;
  const int K = a.k;
  const int nchunks = (K + kTChunk - 1) / kTChunk;
  const int kst = a.Dqk / 16;
  const uint32_t row_bytes = (uint32_t)a.Dqk * 2u;
  const int32_t* idx_row = a.idx + (int64_t)row * K;
  const uint16_t* lat = a.latent + (int64_t)b * a.kv_len * a.Dqk;

  // Zero the ring once: columns past Dqk are never written by the copies.
  for (int i = tid; i < 2 * kTStageBytes / 16; i += kTThreads)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int s = tid; s < K; s += kTThreads) sP[s] = 0.f;
  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(&bars[i], 1);
    *abort_flag = 0u;
    mbar_fence_init();
  }
  for (int ch = warp; ch < nchunks; ch += 4) {
    const int s = ch * kTChunk + lane;
    bool any = false, bad = false;
    if (s < K) {
      const int p = idx_row[s];
      any = p >= 0 && p < a.kv_len;
      bad = p < -1 || p >= a.kv_len;
    }
    any = __any_sync(0xffffffffu, any);
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      sList[4 + ch] = any ? 1 : 0;
      if (bad) report_status(a.status, kStatusDeviceCheck, 0xA77Eu);
    }
  }
  fence_proxy_async_smem();   // the zeros are ordered before the bulk copies
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int ch = 0; ch < nchunks; ++ch)
      if (sList[4 + ch]) sList[4 + n++] = ch;
    sList[0] = n;
  }
  __syncthreads();
  const int nl = sList[0];
  const int* list = sList + 4;
  const int hgs = (a.H + kTNH - 1) / kTNH;
  const int V = nl * hgs;                         // (head group, chunk) steps
  const WaitCtl ctl{abort_flag, a.timeout_ns, a.status};

  // Warp `warp` copies the latent rows of its slots 8w..8w+7 of step v's chunk
  // into ring slot v & 1 (lanes 0-7, one bulk copy per valid slot).
  auto issue = [&](int v) {
    const int ch = list[v % nl];
    const int st = v & 1;
    int pos = -1;
    if (lane < 8) {
      const int s = ch * kTChunk + 8 * warp + lane;
      pos = s < K ? idx_row[s] : -1;
      if (pos >= a.kv_len) pos = -1;
    }
    const uint32_t mine = __ballot_sync(0xffffffffu, pos >= 0);
    if (lane == 0) mbar_arrive_expect_tx(&bars[st * 4 + warp], (uint32_t)__popc(mine) * row_bytes);
    __syncwarp();
    if (pos >= 0)
      bulk_copy_g2s(sc + st * kTStageBytes + (8 * warp + lane) * kTPitch, lat + (int64_t)pos * a.Dqk, row_bytes,
                    &bars[st * 4 + warp]);
    if (lane < 8) sPos[st * kTChunk + 8 * warp + lane] = pos;
  };

  uint32_t qa[kTKsteps][4];
  float l2lse0 = 0.f, l2lse1 = 0.f;
  int cur_hg = -1;
  constexpr float kLog2e = 1.4426950408889634f;
  const float scale_log2 = a.scale * kLog2e;
  bool ok = true;
  int issued = 0;                                 // steps whose copies this warp has issued

  if (V > 0) {
    issue(0);
    issued = 1;
  }
  for (int v = 0; v < V && ok; ++v) {
    const int st = v & 1;
    // ring slot v & 1 was last read at step v - 1 (program order): refill it
    // with step v + 1 only after this step's wait, from the other slot
    if (v + 1 < V) {
      issue(v + 1);
      issued = v + 2;
    }
    if (!mbar_wait(&bars[st * 4 + warp], (uint32_t)((v >> 1) & 1), ctl, 0x3101u)) {
      ok = false;
      break;
    }
    const int hg = v / nl;
    if (hg != cur_hg) {
      // this group's queries (rows g, g + 8; zero past H and past Dqk) and lse
      cur_hg = hg;
      const int h0 = hg * kTNH + g, h1 = h0 + 8;
      const bool v0 = h0 < a.H, v1 = h1 < a.H;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)row * a.H + (v0 ? h0 : 0)) * a.Dqk);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)row * a.H + (v1 ? h1 : 0)) * a.Dqk);
#pragma unroll
      for (int ks = 0; ks < kTKsteps; ++ks) {
        const bool in = ks < kst;
        const int e = ks * 8 + c4;
        qa[ks][0] = (in && v0) ? __ldg(q0 + e) : 0u;
        qa[ks][1] = (in && v1) ? __ldg(q1 + e) : 0u;
        qa[ks][2] = (in && v0) ? __ldg(q0 + e + 4) : 0u;
        qa[ks][3] = (in && v1) ? __ldg(q1 + e + 4) : 0u;
      }
      // a head past H gets lse = +inf, so its probabilities are exactly 0
      l2lse0 = v0 ? a.lse[(int64_t)row * a.H + h0] * kLog2e : INFINITY;
      l2lse1 = v1 ? a.lse[(int64_t)row * a.H + h1] * kLog2e : INFINITY;
    }
    const int ch = list[v % nl];
    // logits of slots 8w..8w+7 for the 16 heads: even / odd k-steps in
    // separate accumulators, fragments requested two steps ahead
    const uint32_t row_addr = sc + st * kTStageBytes + (8 * warp + (lane & 7)) * kTPitch + mi * 16;
    float sacc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
    uint32_t bf[3][4];
    ldsm_x4(row_addr, bf[0]);
    ldsm_x4(row_addr + 64, bf[1]);
#pragma unroll
    for (int i = 0; i < kTKsteps / 2; ++i) {
      if (i + 2 < kTKsteps / 2) ldsm_x4(row_addr + (i + 2) * 64, bf[(i + 2) % 3]);
      mma16816(sacc[0], qa[2 * i], bf[i % 3][0], bf[i % 3][1]);
      mma16816(sacc[1], qa[2 * i + 1], bf[i % 3][2], bf[i % 3][3]);
    }
    // a_h(s) for heads g, g + 8 and slots 2c4, 2c4 + 1; sum over the heads
    const float s00 = sacc[0][0] + sacc[1][0], s01 = sacc[0][1] + sacc[1][1];
    const float s10 = sacc[0][2] + sacc[1][2], s11 = sacc[0][3] + sacc[1][3];
    float e0 = exp2f(s00 * scale_log2 - l2lse0) + exp2f(s10 * scale_log2 - l2lse1);
    float e1 = exp2f(s01 * scale_log2 - l2lse0) + exp2f(s11 * scale_log2 - l2lse1);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      e0 += __shfl_xor_sync(0xffffffffu, e0, o);
      e1 += __shfl_xor_sync(0xffffffffu, e1, o);
    }
    if (g == 0) {
      const int k0 = 8 * warp + 2 * c4;
      const int s0 = ch * kTChunk + k0;
      if (sPos[st * kTChunk + k0] >= 0) sP[s0] += e0;
      if (sPos[st * kTChunk + k0 + 1] >= 0) sP[s0 + 1] += e1;
    }
    __syncwarp();   // this slot's positions and rows are read before the slot is refilled
  }
  if (!ok || *abort_flag != 0u) {
    // stopped early: let this warp's copies in flight land before the CTA
    // exits (each wait bounded by the same timeout)
    for (int v = max(0, issued - 2); v < issued; ++v) {
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(&bars[(v & 1) * 4 + warp]), (uint32_t)((v >> 1) & 1)) &&
             globaltimer_ns() - t0 < a.timeout_ns) {
      }
    }
  }
  __syncthreads();
  // L1 normalisation over the row's selected positions
  float tot = 0.f;
  for (int s = tid; s < K; s += kTThreads) tot += sP[s];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) sRed[warp] = tot;
  __syncthreads();
  tot = (sRed[0] + sRed[1]) + (sRed[2] + sRed[3]);
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  float* out = a.p_out + (int64_t)row * K;
  for (int s = tid; s < K; s += kTThreads) out[s] = sP[s] * inv;
}

}  // namespace

size_t attn_teacher_smem_bytes(int k) { return (size_t)kTOffP + (size_t)k * 4; }

cudaError_t launch_attn_teacher(const TeacherArgs& a, cudaStream_t stream) {
  const size_t smem = attn_teacher_smem_bytes(a.k);
  // the attribute is an upper bound: set once for the largest k, so a later
  // call with a larger k than the first still launches
  cudaError_t e = setup_once_per_device([]() {
    return cudaFuncSetAttribute(attn_teacher_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)attn_teacher_smem_bytes(kMaxTeacherTopk));
  });
  if (e != cudaSuccess) return e;
  attn_teacher_kernel<<<a.rows, kTThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace dsa
