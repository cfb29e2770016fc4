// K4 + K5: sliding-window attention and the gated combine.
//
// "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5 (the third branch attends to the
// neighbouring tokens), §6 (each branch output is scaled by a gate from the current
// token and the three are added); "一文比较 Kimi 和 Deepseek 的两篇稀疏注意力机制论文",
// "Deepseek 的论文核心点" (NSA's window crosses block boundaries).
//
// One CTA = one KV head g and 8 consecutive tokens t0..t0+7; warp w owns token t0+w
// with the group's G <= 16 heads as the 16 MMA rows.  The union of the 8 windows,
// [t0-w+1, t0+7], streams through shared memory in 64-token tiles shared by all
// warps; each row masks to its own window [t-w+1, t].  Epilogue:
// out = bf16(acc + g_win * o_win), where acc already holds g_cmp*o_cmp + g_slc*o_slc.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 64;

template <int DK, int DV>
struct Smem {
  static constexpr size_t kK = 2ull * kTile * DK * 2;
  static constexpr size_t kV = 2ull * kTile * DV * 2;
  static constexpr size_t kTotal = kK + kV;
};

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
swa_combine_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ gates,
                   const float* __restrict__ acc, __nv_bfloat16* __restrict__ out, int T, int Hq, int Hkv, int G,
                   int window, float scale_log2) {
  using SM = Smem<DK, DV>;
  using SwzK = SwzTile<DK>;
  using SwzV = SwzTile<DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + SM::kK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, cq = lane & 3;
  const int t0 = blockIdx.x * kWarps, g = blockIdx.y, b = blockIdx.z;
  const int t = t0 + warp;
  const bool active = t < T;
  const bool rv0 = active && gl < G, rv1 = active && gl + 8 < G;
  const int t_last = min(t0 + kWarps - 1, T - 1);
  const int kv_lo = max(0, t0 - window + 1);
  const int ntiles = (t_last - kv_lo + kTile) / kTile;
  const int lo = active ? max(0, t - window + 1) : 1, hi = active ? t : 0;   // this row's window [lo, hi]

  uint32_t qf[DK / 16][4];
  {
    const __nv_bfloat16* q0 = q + (((size_t)b * T + (active ? t : 0)) * Hq + g * G + gl) * DK;
    const __nv_bfloat16* q1 = q0 + 8 * DK;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
      qf[ks][0] = rv0 ? ld_u32(q0 + ks * 16 + 2 * cq) : 0u;
      qf[ks][1] = rv1 ? ld_u32(q1 + ks * 16 + 2 * cq) : 0u;
      qf[ks][2] = rv0 ? ld_u32(q0 + ks * 16 + 8 + 2 * cq) : 0u;
      qf[ks][3] = rv1 ? ld_u32(q1 + ks * 16 + 8 + 2 * cq) : 0u;
    }
  }

  auto load_tile = [&](int it, int buf) {
    const int u0 = kv_lo + it * kTile;
    for (int e = tid; e < kTile * (DK / 8); e += kThreads) {
      const int r = e / (DK / 8), ch = e % (DK / 8);
      const int u = u0 + r;
      const bool ok = u <= t_last;
      const __nv_bfloat16* src = k + (((size_t)b * T + (ok ? u : t_last)) * Hkv + g) * DK + ch * 8;
      cp_async16(sK + (size_t)buf * kTile * DK + SwzK::offset(r, ch), src, ok);
    }
    for (int e = tid; e < kTile * (DV / 8); e += kThreads) {
      const int r = e / (DV / 8), ch = e % (DV / 8);
      const int u = u0 + r;
      const bool ok = u <= t_last;
      const __nv_bfloat16* src = v + (((size_t)b * T + (ok ? u : t_last)) * Hkv + g) * DV + ch * 8;
      cp_async16(sV + (size_t)buf * kTile * DV + SwzV::offset(r, ch), src, ok);
    }
  };

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[DV / 8][4];
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  load_tile(0, 0);
  cp_async_commit();
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) load_tile(it + 1, (it + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int buf = it & 1;
    const int u0 = kv_lo + it * kTile;
    if (u0 <= hi && u0 + kTile - 1 >= lo) {     // this tile meets the row's window
      float s[kTile / 8][4];
#pragma unroll
      for (int j = 0; j < kTile / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
      const __nv_bfloat16* kb = sK + (size_t)buf * kTile * DK;
#pragma unroll
      for (int ks = 0; ks < DK / 16; ++ks) {
#pragma unroll
        for (int np = 0; np < kTile / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
          const int ch = 2 * ks + ((lane >> 3) & 1);
          ldsm_x4(b0, b1, b2, b3, smem_u32(kb + SwzK::offset(row, ch)));
          mma16816(s[2 * np], qf[ks], b0, b1);
          mma16816(s[2 * np + 1], qf[ks], b2, b3);
        }
      }
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < kTile / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int u = u0 + j * 8 + 2 * cq + e;
          const bool ok = u >= lo && u <= hi;
          s[j][e] = ok ? s[j][e] * scale_log2 : -INFINITY;
          s[j][2 + e] = ok ? s[j][2 + e] * scale_log2 : -INFINITY;
          mx0 = fmaxf(mx0, s[j][e]);
          mx1 = fmaxf(mx1, s[j][2 + e]);
        }
      mx0 = warp_max4(mx0);
      mx1 = warp_max4(mx1);
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float base0 = n0 == -INFINITY ? 0.f : n0, base1 = n1 == -INFINITY ? 0.f : n1;
      const float c0 = exp2f(m0 - base0), c1 = exp2f(m1 - base1);
      float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
      for (int j = 0; j < kTile / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          s[j][e] = exp2f(s[j][e] - base0);
          s[j][2 + e] = exp2f(s[j][2 + e] - base1);
          sum0 += s[j][e];
          sum1 += s[j][2 + e];
        }
      l0 = l0 * c0 + warp_sum4(sum0);
      l1 = l1 * c1 + warp_sum4(sum1);
      m0 = n0;
      m1 = n1;
#pragma unroll
      for (int j = 0; j < DV / 8; ++j) {
        o[j][0] *= c0; o[j][1] *= c0; o[j][2] *= c1; o[j][3] *= c1;
      }
      const __nv_bfloat16* vb = sV + (size_t)buf * kTile * DV;
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        uint32_t a[4];
        a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int np = 0; np < DV / 16; ++np) {
          uint32_t b0, b1, b2, b3;
          const int row = kk * 16 + (lane & 15);
          const int ch = 2 * np + (lane >> 4);
          ldsm_x4_t(b0, b1, b2, b3, smem_u32(vb + SwzV::offset(row, ch)));
          mma16816(o[2 * np], a, b0, b1);
          mma16816(o[2 * np + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if (!active) return;

  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = gl + half * 8;
    if (r >= G) continue;
    const size_t row = ((size_t)b * T + t) * Hq + g * G + r;
    const float gw = __bfloat162float(gates[row * 3 + 2]) * (half ? inv1 : inv0);
    const float* src = acc + row * DV;
    __nv_bfloat16* dst = out + row * DV;
#pragma unroll
    for (int j = 0; j < DV / 8; ++j) {
      const float2 a = *reinterpret_cast<const float2*>(src + j * 8 + 2 * cq);
      *reinterpret_cast<uint32_t*>(dst + j * 8 + 2 * cq) =
          pack_bf16(a.x + gw * o[j][2 * half], a.y + gw * o[j][2 * half + 1]);
    }
  }
}

template <int DK, int DV>
cudaError_t launch(const FwdArgs& a, cudaStream_t st) {
  const size_t smem = Smem<DK, DV>::kTotal;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(swa_combine_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid((a.T + kWarps - 1) / kWarps, a.Hkv, a.B);
  swa_combine_kernel<DK, DV><<<grid, kThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.gates), a.acc,
      static_cast<__nv_bfloat16*>(a.out), a.T, a.Hq, a.Hkv, a.G, a.window, a.scale_log2);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_swa_combine(const FwdArgs& a, cudaStream_t st) {
  if (window_tc_supported(a)) return launch_window_tc(a, st);
  if (a.cu) return cudaErrorInvalidValue;   // variable-length batches run on the tensor-core kernels only
  if (a.dk == 64 && a.dv == 64) return launch<64, 64>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch<128, 128>(a, st);
  if (a.dk == 192 && a.dv == 128) return launch<192, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
