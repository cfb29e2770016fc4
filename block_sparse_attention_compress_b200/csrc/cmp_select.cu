// K2: compressed attention + group-summed block scores + top-k selection.
//
// "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5 (the compressed branch attends
// over one key/value per block and its output enters the sum), §8 (the heads of a
// GQA group add their block scores and share one top-k); "一文比较 Kimi 和 Deepseek
// 的两篇稀疏注意力机制论文", "Deepseek 的论文核心点" (selection scores are taken
// from the compressed attention).
//
// One CTA = one KV head g and 8 consecutive tokens; warp w owns token t0+w and its
// G <= 16 query heads as the 16 rows of an m16n8k16 tile (heads stacked as M).
// The compressed keys/values of the group stream through shared memory in
// tiles of 64 blocks, twice:
//   pass A  S = Q Kc^T, online max / sum  ->  log-sum-exp per (t, h);
//   pass B  P = exp(S - lse) (already normalised), O += P Vc, and the column
//           sums of P over the group's heads, folded into 64-token selection
//           block scores (compressed block i spans tokens [16i, 16i+32), so
//           selection block j collects i = 4j-1 .. 4j+3).
// Then each warp picks its token's top-k blocks (forced blocks first, higher
// score first, ties to the lower index) and writes them ascending.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kTile = 64;        // compressed blocks per shared-memory tile
constexpr int kMaxSel = 1024;    // selection blocks per token (T <= 65536)
constexpr int kL = 32, kS = 16, kSel = 64;

template <int DK, int DV>
struct Smem {
  static constexpr size_t kK = 2ull * kTile * DK * 2;
  static constexpr size_t kV = 2ull * kTile * DV * 2;
  static constexpr size_t kScore = (size_t)kWarps * kMaxSel * 4;
  static constexpr size_t kCs = (size_t)kWarps * kTile * 4;
  static constexpr size_t kTotal = kK + kV + kScore + kCs;
};

__device__ __forceinline__ int n_visible(int t, int nc) { return t < kL - 1 ? 0 : min(nc, (t - kL + 1) / kS + 1); }

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
cmp_select_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kc,
                  const __nv_bfloat16* __restrict__ vc, const __nv_bfloat16* __restrict__ gates,
                  float* __restrict__ acc, int32_t* __restrict__ idx_out, int T, int Hq, int Hkv, int G, int nc,
                  int top_k, int force_first, int force_local, float scale_log2, float w_straddle) {
  using SM = Smem<DK, DV>;
  using SwzK = SwzTile<DK>;
  using SwzV = SwzTile<DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + SM::kK);
  float* sScore = reinterpret_cast<float*>(smem + SM::kK + SM::kV);
  float* sCs = sScore + kWarps * kMaxSel;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, cq = lane & 3;
  const int n_tok_tiles = (T + kWarps - 1) / kWarps;
  const int t0 = (n_tok_tiles - 1 - (int)blockIdx.x) * kWarps;   // longest rows first
  const int g = blockIdx.y, b = blockIdx.z;
  const int t = t0 + warp;
  const bool active = t < T;
  const int nvis = active ? n_visible(t, nc) : 0;
  const int ntiles = (n_visible(min(t0 + kWarps - 1, T - 1), nc) + kTile - 1) / kTile;
  const bool rv0 = active && gl < G, rv1 = active && gl + 8 < G;

  // Q fragments of this warp's 16 rows (heads g*G .. g*G+G-1 of token t).
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

  auto load_tile = [&](int it, int buf, bool with_v) {
    const int i0 = it * kTile;
    for (int e = tid; e < kTile * (DK / 8); e += kThreads) {
      const int r = e / (DK / 8), ch = e % (DK / 8);
      const int i = i0 + r;
      const bool ok = i < nc;
      const __nv_bfloat16* src = kc + (((size_t)b * nc + (ok ? i : 0)) * Hkv + g) * DK + ch * 8;
      cp_async16(sK + (size_t)buf * kTile * DK + SwzK::offset(r, ch), src, ok);
    }
    if (with_v) {
      for (int e = tid; e < kTile * (DV / 8); e += kThreads) {
        const int r = e / (DV / 8), ch = e % (DV / 8);
        const int i = i0 + r;
        const bool ok = i < nc;
        const __nv_bfloat16* src = vc + (((size_t)b * nc + (ok ? i : 0)) * Hkv + g) * DV + ch * 8;
        cp_async16(sV + (size_t)buf * kTile * DV + SwzV::offset(r, ch), src, ok);
      }
    }
  };

  // S = Q Kc^T for one tile (16 rows x 64 compressed blocks), scaled to log2 units.
  auto scores = [&](int buf, float (&s)[kTile / 8][4]) {
#pragma unroll
    for (int j = 0; j < kTile / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const __nv_bfloat16* base = sK + (size_t)buf * kTile * DK;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < kTile / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(b0, b1, b2, b3, smem_u32(base + SwzK::offset(row, ch)));
        mma16816(s[2 * np], qf[ks], b0, b1);
        mma16816(s[2 * np + 1], qf[ks], b2, b3);
      }
    }
#pragma unroll
    for (int j = 0; j < kTile / 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] *= scale_log2;
  };

  // ---------------- pass A: log-sum-exp per row ----------------
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  if (ntiles > 0) {
    load_tile(0, 0, false);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) load_tile(it + 1, (it + 1) & 1, false);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[kTile / 8][4];
    scores(it & 1, s);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < kTile / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = it * kTile + j * 8 + 2 * cq + e;
        if (i >= nvis) { s[j][e] = -INFINITY; s[j][2 + e] = -INFINITY; }
        mx0 = fmaxf(mx0, s[j][e]);
        mx1 = fmaxf(mx1, s[j][2 + e]);
      }
    }
    mx0 = warp_max4(mx0);
    mx1 = warp_max4(mx1);
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    if (n0 != -INFINITY) {
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < kTile / 8; ++j) sum += exp2f(s[j][0] - n0) + exp2f(s[j][1] - n0);
      l0 = l0 * exp2f(m0 - n0) + warp_sum4(sum);
      m0 = n0;
    }
    if (n1 != -INFINITY) {
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < kTile / 8; ++j) sum += exp2f(s[j][2] - n1) + exp2f(s[j][3] - n1);
      l1 = l1 * exp2f(m1 - n1) + warp_sum4(sum);
      m1 = n1;
    }
    __syncthreads();
  }
  const float lse0 = (rv0 && l0 > 0.f) ? m0 + __log2f(l0) : INFINITY;
  const float lse1 = (rv1 && l1 > 0.f) ? m1 + __log2f(l1) : INFINITY;

  // ---------------- pass B: P, O = P Vc, block scores ----------------
  const int nb = active ? t / kSel + 1 : 0;     // eligible selection blocks
  float* score = sScore + warp * kMaxSel;
  float* cs = sCs + warp * kTile;
  for (int j = lane; j < nb; j += 32) score[j] = 0.f;
  __syncwarp();

  float o[DV / 8][4];
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float carry = 0.f;   // column sum of compressed block 64*it - 1 (belongs to two selection blocks)

  if (ntiles > 0) {
    load_tile(0, 0, true);
    cp_async_commit();
  }
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) load_tile(it + 1, (it + 1) & 1, true);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int buf = it & 1;
    float s[kTile / 8][4];
    scores(buf, s);
#pragma unroll
    for (int j = 0; j < kTile / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = it * kTile + j * 8 + 2 * cq + e;
        const bool ok = i < nvis;
        s[j][e] = ok ? exp2f(s[j][e] - lse0) : 0.f;
        s[j][2 + e] = ok ? exp2f(s[j][2 + e] - lse1) : 0.f;
      }
    }
    // O += P Vc
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
    // group sum over the rows (heads): rows beyond G carry p = 0 (lse = +inf)
#pragma unroll
    for (int j = 0; j < kTile / 8; ++j) {
      float c0 = s[j][0] + s[j][2], c1 = s[j][1] + s[j][3];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        c0 += __shfl_xor_sync(0xffffffffu, c0, off);
        c1 += __shfl_xor_sync(0xffffffffu, c1, off);
      }
      if (lane < 4) {   // block 2*lane + 1 (mod 4) straddles two selection blocks when lane is odd
        cs[j * 8 + 2 * lane] = c0;
        cs[j * 8 + 2 * lane + 1] = (lane & 1) ? c1 * w_straddle : c1;
      }
    }
    __syncwarp();
    if (lane < kTile / 4) {
      const int j = it * (kTile / 4) + lane;
      if (j < nb) {
        const float prev = lane == 0 ? carry : cs[4 * lane - 1];
        score[j] = prev + cs[4 * lane] + cs[4 * lane + 1] + cs[4 * lane + 2] + cs[4 * lane + 3];
      }
    }
    carry = cs[kTile - 1];
    __syncwarp();
    __syncthreads();
  }
  cp_async_wait<0>();
  if (lane == 0 && ntiles * (kTile / 4) < nb) score[ntiles * (kTile / 4)] = carry;
  __syncwarp();

  if (!active) return;

  // ---------------- epilogue: acc = g_cmp * o_cmp ----------------
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = gl + half * 8;
    if (r >= G) continue;
    const int h = g * G + r;
    const size_t row = ((size_t)b * T + t) * Hq + h;
    const float gc = __bfloat162float(gates[row * 3 + 0]);
    float* dst = acc + row * DV;
#pragma unroll
    for (int j = 0; j < DV / 8; ++j) {
      float2 v = make_float2(gc * o[j][2 * half], gc * o[j][2 * half + 1]);
      *reinterpret_cast<float2*>(dst + j * 8 + 2 * cq) = v;
    }
  }

  // ---------------- top-k over the nb eligible blocks ----------------
  int32_t* dst = idx_out + (((size_t)b * Hkv + g) * T + t) * top_k;
  if (nb <= top_k) {
    for (int j = lane; j < top_k; j += 32) dst[j] = j < nb ? j : -1;
    return;
  }
  const int own = t / kSel;
  uint32_t taken = 0;   // bit m <-> block lane + 32*m
  int nforced = 0;
  if (force_first) { if (lane == 0) taken |= 1u; ++nforced; }
  if (force_local && !(force_first && own == 0)) {
    if (lane == (own & 31)) taken |= 1u << (own >> 5);
    ++nforced;
  }
  const int mmax = (nb + 31) >> 5;
  for (int r = nforced; r < top_k; ++r) {
    float bs = -FLT_MAX;
    int bj = 0x7fffffff;
    for (int m = 0; m < mmax; ++m) {
      const int j = lane + 32 * m;
      if (j < nb && !((taken >> m) & 1u)) {
        const float sc = score[j];
        if (sc > bs) { bs = sc; bj = j; }   // j increases with m: strict > keeps the lower index
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, off);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
      if (os > bs || (os == bs && oj < bj)) { bs = os; bj = oj; }
    }
    if (bj != 0x7fffffff && lane == (bj & 31)) taken |= 1u << (bj >> 5);
  }
  int pos = 0;
  for (int m = 0; m < mmax; ++m) {
    const bool sel = (taken >> m) & 1u;
    const uint32_t bal = __ballot_sync(0xffffffffu, sel);
    if (sel) dst[pos + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * m;
    pos += __popc(bal);
  }
  for (int j = pos + lane; j < top_k; j += 32) dst[j] = -1;
}

template <int DK, int DV>
cudaError_t launch(const FwdArgs& a, cudaStream_t st) {
  const size_t smem = Smem<DK, DV>::kTotal;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e = cudaFuncSetAttribute(cmp_select_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid((a.T + kWarps - 1) / kWarps, a.Hkv, a.B);
  cmp_select_kernel<DK, DV><<<grid, kThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.kc),
      static_cast<const __nv_bfloat16*>(a.vc), static_cast<const __nv_bfloat16*>(a.gates), a.acc, a.idx, a.T,
      a.Hq, a.Hkv, a.G, a.nc, a.top_k, a.force_first, a.force_local, a.scale_log2, a.w_straddle);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_cmp_select(const FwdArgs& a, cudaStream_t st) {
  if (cmp_select_tc_supported(a)) return launch_cmp_select_tc(a, st);
  if (a.cu) return cudaErrorInvalidValue;   // variable-length batches run on the tensor-core kernels only
  if (a.dk == 64 && a.dv == 64) return launch<64, 64>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch<128, 128>(a, st);
  if (a.dk == 192 && a.dv == 128) return launch<192, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
