// K3: selected-block attention ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5: the
// top-k blocks are expanded to all their tokens for token-level attention; §10: the
// group's query heads share the loaded blocks and form the matrix dimension).
//
// One CTA = one (token t, KV head g).  The G <= 16 query heads of the group are the
// 16 rows of every m16n8k16 tile; the CTA streams the token's selected 64-token K/V
// blocks through a two-stage shared-memory ring (each block read once for all heads),
// and each of its 4 warps takes 16 of the 64 keys of every block with its own online
// softmax.  The four partial softmax states are merged at the end and
// acc += g_slc * o_slc is written back.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kBlk = 64;     // selection block (tokens)

template <int DK, int DV>
struct Smem {
  static constexpr size_t kK = 2ull * kBlk * DK * 2;
  static constexpr size_t kV = 2ull * kBlk * DV * 2;
  static constexpr size_t kMerge = (size_t)kWarps * 16 * DV * 4 + kWarps * 16 * 2 * 4;
  static constexpr size_t kTotal = (kK + kV) > kMerge ? (kK + kV) : kMerge;
};

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads)
slc_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ gates,
                const int32_t* __restrict__ idx, float* __restrict__ acc, int T, int Hq, int Hkv, int G,
                int top_k, float scale_log2) {
  using SM = Smem<DK, DV>;
  using SwzK = SwzTile<DK>;
  using SwzV = SwzTile<DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + SM::kK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, cq = lane & 3;
  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const bool rv0 = gl < G, rv1 = gl + 8 < G;
  const int32_t* sel = idx + (((size_t)b * Hkv + g) * T + t) * top_k;
  int nsel = 0;
  for (int j = 0; j < top_k; ++j) nsel += sel[j] >= 0;

  uint32_t qf[DK / 16][4];
  {
    const __nv_bfloat16* q0 = q + (((size_t)b * T + t) * Hq + g * G + gl) * DK;
    const __nv_bfloat16* q1 = q0 + 8 * DK;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
      qf[ks][0] = rv0 ? ld_u32(q0 + ks * 16 + 2 * cq) : 0u;
      qf[ks][1] = rv1 ? ld_u32(q1 + ks * 16 + 2 * cq) : 0u;
      qf[ks][2] = rv0 ? ld_u32(q0 + ks * 16 + 8 + 2 * cq) : 0u;
      qf[ks][3] = rv1 ? ld_u32(q1 + ks * 16 + 8 + 2 * cq) : 0u;
    }
  }

  auto block_of = [&](int jj) { return min(max(sel[jj], 0), t / kBlk); };   // stays causal and in range
  auto load_block = [&](int jj, int buf) {
    const int u0 = block_of(jj) * kBlk;
    for (int e = tid; e < kBlk * (DK / 8); e += kThreads) {
      const int r = e / (DK / 8), ch = e % (DK / 8);
      const int u = u0 + r;
      const bool ok = u <= t;   // tokens after t are masked anyway; never read past T
      const __nv_bfloat16* src = k + (((size_t)b * T + (ok ? u : t)) * Hkv + g) * DK + ch * 8;
      cp_async16(sK + (size_t)buf * kBlk * DK + SwzK::offset(r, ch), src, ok);
    }
    for (int e = tid; e < kBlk * (DV / 8); e += kThreads) {
      const int r = e / (DV / 8), ch = e % (DV / 8);
      const int u = u0 + r;
      const bool ok = u <= t;
      const __nv_bfloat16* src = v + (((size_t)b * T + (ok ? u : t)) * Hkv + g) * DV + ch * 8;
      cp_async16(sV + (size_t)buf * kBlk * DV + SwzV::offset(r, ch), src, ok);
    }
  };

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[DV / 8][4];
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  if (nsel > 0) {
    load_block(0, 0);
    cp_async_commit();
  }
  for (int jj = 0; jj < nsel; ++jj) {
    if (jj + 1 < nsel) load_block(jj + 1, (jj + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int buf = jj & 1;
    const int u0 = block_of(jj) * kBlk + warp * 16;   // this warp's 16 keys
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const __nv_bfloat16* kb = sK + (size_t)buf * kBlk * DK;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
      uint32_t b0, b1, b2, b3;
      const int row = warp * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int ch = 2 * ks + ((lane >> 3) & 1);
      ldsm_x4(b0, b1, b2, b3, smem_u32(kb + SwzK::offset(row, ch)));
      mma16816(s[0], qf[ks], b0, b1);
      mma16816(s[1], qf[ks], b2, b3);
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int u = u0 + j * 8 + 2 * cq + e;
        const bool ok = u <= t;
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
    for (int j = 0; j < 2; ++j)
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
    uint32_t a[4];
    a[0] = pack_bf16(s[0][0], s[0][1]);
    a[1] = pack_bf16(s[0][2], s[0][3]);
    a[2] = pack_bf16(s[1][0], s[1][1]);
    a[3] = pack_bf16(s[1][2], s[1][3]);
    const __nv_bfloat16* vb = sV + (size_t)buf * kBlk * DV;
#pragma unroll
    for (int np = 0; np < DV / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      const int row = warp * 16 + (lane & 15);
      const int ch = 2 * np + (lane >> 4);
      ldsm_x4_t(b0, b1, b2, b3, smem_u32(vb + SwzV::offset(row, ch)));
      mma16816(o[2 * np], a, b0, b1);
      mma16816(o[2 * np + 1], a, b2, b3);
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // merge the four warps' partial softmax states
  float* sO = reinterpret_cast<float*>(smem);                 // [warp][16][DV]
  float* sML = sO + kWarps * 16 * DV;                         // [warp][16][2]
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) {
    *reinterpret_cast<float2*>(sO + ((size_t)warp * 16 + gl) * DV + j * 8 + 2 * cq) = make_float2(o[j][0], o[j][1]);
    *reinterpret_cast<float2*>(sO + ((size_t)warp * 16 + gl + 8) * DV + j * 8 + 2 * cq) =
        make_float2(o[j][2], o[j][3]);
  }
  if (cq == 0) {
    sML[(warp * 16 + gl) * 2 + 0] = m0;
    sML[(warp * 16 + gl) * 2 + 1] = l0;
    sML[(warp * 16 + gl + 8) * 2 + 0] = m1;
    sML[(warp * 16 + gl + 8) * 2 + 1] = l1;
  }
  __syncthreads();
  for (int e = tid; e < G * DV; e += kThreads) {
    const int r = e / DV, c = e % DV;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sML[(w * 16 + r) * 2]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = exp2f(sML[(w * 16 + r) * 2] - M);
        L += f * sML[(w * 16 + r) * 2 + 1];
        O += f * sO[((size_t)w * 16 + r) * DV + c];
      }
    }
    const size_t row = ((size_t)b * T + t) * Hq + g * G + r;
    const float gs = __bfloat162float(gates[row * 3 + 1]);
    acc[row * DV + c] += L > 0.f ? gs * O / L : 0.f;
  }
}

template <int DK, int DV>
cudaError_t launch(const FwdArgs& a, cudaStream_t st) {
  const size_t smem = Smem<DK, DV>::kTotal;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(slc_attn_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid(a.T, a.Hkv, a.B);
  slc_attn_kernel<DK, DV><<<grid, kThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.gates), a.idx, a.acc, a.T,
      a.Hq, a.Hkv, a.G, a.top_k, a.scale_log2);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_slc_attn(const FwdArgs& a, cudaStream_t st) {
  if (slc_attn_tc_supported(a)) return launch_slc_attn_tc(a, st);
  if (slc_attn_tma_supported(a)) return launch_slc_attn_tma(a, st);
  if (a.cu) return cudaErrorInvalidValue;   // variable-length batches run on the tensor-core kernels only
  if (a.dk == 64 && a.dv == 64) return launch<64, 64>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch<128, 128>(a, st);
  if (a.dk == 192 && a.dv == 128) return launch<192, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
