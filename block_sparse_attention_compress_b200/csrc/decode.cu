// K6: one decode step ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §13: a decode step
// is bound by the KV bytes it reads; the group-shared choice reads each chosen block
// once for all of the group's heads).
//
// One CTA = one (sequence, KV group); its 8 warps hold the group's G <= 16 query heads
// as the 16 rows of m16n8k16 tiles.  Everything happens in one launch:
//   A  warp w streams compressed blocks [512w, 512w+512) through its own two-stage
//      shared-memory ring (16 blocks = 10 KB per stage): online softmax for o_cmp and,
//      per head, the running sums of exp(s - m) per 64-token selection block
//      (rescaled whenever that head's running max grows);
//   M  the warps' states are merged: per-head log-sum-exp, each warp's weight and the
//      group-summed normalised block scores; then warp 0 runs the top-k (forced blocks
//      first, ties to the lower index) while warps 1..7 sum o_cmp and stream the
//      window, which needs no selection, with their own softmax states;
//   B  the selected blocks (two per warp), with one more softmax state per warp;
//      each branch's states are merged by log-sum-exp weights;
//   C  out = g_cmp*o_cmp + g_slc*o_slc + g_win*o_win, rounded to bf16.
// Loads are 16-byte cp.async of whole K/V rows (each row 384 + 256 bytes): a group of eight
// lanes copies one 128-byte line of a row, so each copy instruction of a warp moves lines of
// four rows, and each lane looks its four rows up once per tile.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "rows_attn.cuh"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int kRange = 512;          // compressed blocks per warp
constexpr int kJ = kRange / 4 + 1;   // selection blocks touched by one warp's range
constexpr int kMaxSel = 1024;
constexpr int kL = 32, kS = 16, kSel = 64;

template <int DK, int DV>
struct Smem {
  static constexpr size_t kStage = (size_t)kRows * (DK + DV) * 2;               // one tile (K then V)
  static constexpr size_t kRing = (size_t)kWarps * 2 * kStage;                   // per-warp double buffer
  static constexpr size_t kPart = (size_t)kWarps * 16 * kJ * 4;                  // per-warp per-head block sums
  static constexpr size_t kPersist =
      ((size_t)(kWarps * 16 * 2 + kWarps * 16 + kMaxSel + 32 + 3 * 16 * DV) * 4 + 127) / 128 * 128;
  static constexpr size_t kMergeBytes = (size_t)kWarps * 16 * (DV + 8) * 4 + (size_t)kWarps * 16 * 3 * 4;
  static constexpr size_t kPhaseB = kPersist + (kRing > kMergeBytes ? kRing : kMergeBytes);
  static constexpr size_t kTotal = (kRing + kPart) > kPhaseB ? (kRing + kPart) : kPhaseB;
  static_assert(kTotal <= 232448, "decode shared memory");
  static_assert(kPersist + kMergeBytes <= kRing, "o_cmp merge must not touch the per-warp block sums");
};


template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
decode_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kcache,
              const __nv_bfloat16* __restrict__ vcache, const __nv_bfloat16* __restrict__ kccache,
              const __nv_bfloat16* __restrict__ vccache, const int32_t* __restrict__ seqlens,
              const __nv_bfloat16* __restrict__ gates, __nv_bfloat16* __restrict__ out, int32_t* __restrict__ idx_out,
              int Lmax, int Ncmax, int max_seqlen, int Hq, int Hkv, int G, int top_k, int window, int force_first,
              int force_local, float scale_log2, float w_straddle) {
  using SM = Smem<DK, DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gl = lane >> 2, cq = lane & 3;
  const int g = blockIdx.x, b = blockIdx.y;
  const int L = min(max(seqlens[b], 1), max_seqlen);
  const int t = L - 1;
  const int nvis = t < kL - 1 ? 0 : min(Ncmax, (t - kL + 1) / kS + 1);
  const bool rv0 = gl < G, rv1 = gl + 8 < G;

  Tile<DK, DV> ring0{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)warp * 2 * SM::kStage), nullptr};
  ring0.v = ring0.k + kRows * DK;
  Tile<DK, DV> ring1{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)warp * 2 * SM::kStage + SM::kStage), nullptr};
  ring1.v = ring1.k + kRows * DK;
  float* part = reinterpret_cast<float*>(smem + SM::kRing) + (size_t)warp * 16 * kJ;   // [16][kJ]

  uint32_t qf[DK / 16][4];
  {
    const __nv_bfloat16* q0 = q + ((size_t)b * Hq + g * G + gl) * DK;
    const __nv_bfloat16* q1 = q0 + 8 * DK;
#pragma unroll
    for (int ks = 0; ks < DK / 16; ++ks) {
      qf[ks][0] = rv0 ? ld_u32(q0 + ks * 16 + 2 * cq) : 0u;
      qf[ks][1] = rv1 ? ld_u32(q1 + ks * 16 + 2 * cq) : 0u;
      qf[ks][2] = rv0 ? ld_u32(q0 + ks * 16 + 8 + 2 * cq) : 0u;
      qf[ks][3] = rv1 ? ld_u32(q1 + ks * 16 + 8 + 2 * cq) : 0u;
    }
  }

  // ---------------- A: compressed blocks of this warp ----------------
  for (int e = lane; e < 16 * kJ; e += 32) part[e] = 0.f;
  __syncwarp();
  State<DV> st;
  st.init();
  const int i_lo = warp * kRange;
  const int n_a = max(0, min(nvis - i_lo, kRange));
  {
    auto rowk = [&](int r) { return kccache + (((size_t)b * Ncmax + i_lo + r) * Hkv + g) * DK; };
    auto rowv = [&](int r) { return vccache + (((size_t)b * Ncmax + i_lo + r) * Hkv + g) * DV; };
    const int ntiles = (n_a + kRows - 1) / kRows;
    if (ntiles > 0) {
      load_rows<DK, DV>(ring0, 0, n_a, rowk, rowv, lane);
      cp_async_commit();
    }
    for (int it = 0; it < ntiles; ++it) {
      if (it + 1 < ntiles) load_rows<DK, DV>((it + 1) & 1 ? ring1 : ring0, (it + 1) * kRows, n_a, rowk, rowv, lane);
      cp_async_commit();
      cp_async_wait<1>();
      __syncwarp();
      const Tile<DK, DV> cur = (it & 1) ? ring1 : ring0;
      float s[2][4];
      qk_tile<DK>(qf, cur.k, s, scale_log2, lane);
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (it * kRows + j * 8 + 2 * cq + e >= n_a) { s[j][e] = -INFINITY; s[j][2 + e] = -INFINITY; }
      float c0, c1;
      softmax_update<DV>(st, s, c0, c1);
      // rescale this head's block sums when its running max grew (rare after the first tiles)
      if (rv0 && c0 != 1.f)
        for (int jj = cq; jj < kJ; jj += 4) part[gl * kJ + jj] *= c0;
      if (rv1 && c1 != 1.f)
        for (int jj = cq; jj < kJ; jj += 4) part[(gl + 8) * kJ + jj] *= c1;
      __syncwarp();
      // block sums: local compressed index il = 16*it + 8*nt + 2*cq + e goes to selection
      // block il/4 and, when il % 4 == 3, also to il/4 + 1 (two passes keep lanes apart)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int jb = 4 * it + 2 * nt + (cq >> 1);
        // local index 2*cq + 1 (mod 4) straddles two selection blocks when cq is odd
        const float w1 = (cq & 1) ? w_straddle : 1.f;
        float a0 = s[nt][0] + w1 * s[nt][1], a1 = s[nt][2] + w1 * s[nt][3];
        a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
        a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
        if ((cq & 1) == 0) {
          if (rv0) part[gl * kJ + jb] += a0;
          if (rv1) part[(gl + 8) * kJ + jb] += a1;
        }
      }
      __syncwarp();
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int jb = 4 * it + 2 * nt + (cq >> 1) + 1;
        if (cq & 1) {
          if (rv0) part[gl * kJ + jb] += w_straddle * s[nt][1];
          if (rv1) part[(gl + 8) * kJ + jb] += w_straddle * s[nt][3];
        }
      }
      pv_tile<DV>(s, cur.v, st.o, lane);
      __syncwarp();
    }
    cp_async_wait<0>();
  }
  __syncthreads();

  // ---------------- M: merge, scores, top-k, o_cmp ----------------
  // Small persistent buffers sit at the bottom (over the dead phase-A rings); above them one
  // union region serves the cross-warp merges and, later, the stage rings.
  float* sML = reinterpret_cast<float*>(smem);                         // [8][16][2] m, l
  float* sCoef = sML + kWarps * 16 * 2;                                // [8][16]
  float* sScore = sCoef + kWarps * 16;                                 // [kMaxSel]
  int* sIdx = reinterpret_cast<int*>(sScore + kMaxSel);                // [32]
  float* sOcmp = reinterpret_cast<float*>(sIdx + 32);                  // [16][DV]
  float* sOslc = sOcmp + 16 * DV;                                      // [16][DV]
  float* sOwin = sOslc + 16 * DV;                                      // [16][DV]
  uint8_t* uni = smem + SM::kPersist;                                  // merge scratch / stage rings
  float* sMerge = reinterpret_cast<float*>(uni);
  store_o<DV>(sMerge, st, 1.f, 1.f, warp, lane);
  store_ml(sML, st.m0, st.l0, st.m1, st.l1, warp, lane);
  __syncthreads();
  if (tid < 16) merge_coefs(sML, sCoef, G, tid);   // per-head log-sum-exp -> each warp's weight
  __syncthreads();
  const int nb = t / kSel + 1;
  {
    const float* partAll = reinterpret_cast<const float*>(smem + SM::kRing);
    for (int J = tid; J < nb; J += kThreads) {
      const int w = J / (kRange / 4), jj = J - w * (kRange / 4);
      float sc = 0.f;
      for (int r = 0; r < G; ++r) {
        sc += sCoef[w * 16 + r] * partAll[((size_t)w * 16 + r) * kJ + jj];
        if (jj == 0 && w > 0) sc += sCoef[(w - 1) * 16 + r] * partAll[((size_t)(w - 1) * 16 + r) * kJ + kJ - 1];
      }
      sScore[J] = sc;
    }
  }
  __syncthreads();   // the block sums are dead from here on
  const int own = t / kSel;
  Tile<DK, DV> rb0{reinterpret_cast<__nv_bfloat16*>(uni + (size_t)warp * 2 * SM::kStage), nullptr};
  rb0.v = rb0.k + kRows * DK;
  Tile<DK, DV> rb1{reinterpret_cast<__nv_bfloat16*>(uni + (size_t)warp * 2 * SM::kStage + SM::kStage), nullptr};
  rb1.v = rb1.k + kRows * DK;
  st.init();
  if (warp == 0) {   // top-k over the nb eligible blocks, while the other warps stream the window
    if (nb <= top_k) {
      for (int j = lane; j < top_k; j += 32) sIdx[j] = j < nb ? j : -1;
    } else {
      uint32_t taken = 0;
      int nforced = 0;
      if (force_first) { if (lane == 0) taken |= 1u; ++nforced; }
      if (force_local && !(force_first && own == 0)) {
        if (lane == (own & 31)) taken |= 1u << (own >> 5);
        ++nforced;
      }
      const int mmax = (nb + 31) >> 5;
      // this lane's candidates j = lane + 32*mm as order-preserving integer keys (the
      // scores are sums of probabilities, >= 0); key 0 marks "no candidate"
      uint32_t key[32];
#pragma unroll
      for (int mm = 0; mm < 32; ++mm) {
        const int j = lane + 32 * mm;
        key[mm] = (mm < mmax && j < nb && !((taken >> mm) & 1u)) ? __float_as_uint(sScore[j]) + 1u : 0u;
      }
      uint32_t bk = 0;   // this lane's best key and its mm (the lowest mm among equal keys)
      int bm = 0;
      auto local_best = [&]() {
        bk = 0;
        bm = 0;
#pragma unroll
        for (int mm = 0; mm < 32; ++mm)
          if (key[mm] > bk) { bk = key[mm]; bm = mm; }
      };
      local_best();
      for (int rr = nforced; rr < top_k; ++rr) {
        const uint32_t vmax = __reduce_max_sync(0xffffffffu, bk);
        if (vmax == 0u) break;
        const uint32_t jmin = __reduce_min_sync(0xffffffffu, bk == vmax ? (uint32_t)(lane + 32 * bm) : 0xffffffffu);
        if (lane == (int)(jmin & 31u)) {
          const int mw = (int)(jmin >> 5);
          taken |= 1u << mw;
#pragma unroll
          for (int mm = 0; mm < 32; ++mm)
            if (mm == mw) key[mm] = 0u;
          local_best();
        }
      }
      int pos = 0;
      for (int m = 0; m < mmax; ++m) {
        const bool sel = (taken >> m) & 1u;
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        if (sel) sIdx[pos + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * m;
        pos += __popc(bal);
      }
      for (int j = pos + lane; j < top_k; j += 32) sIdx[j] = -1;
    }
    __syncwarp();
    if (idx_out)
      for (int j = lane; j < top_k; j += 32) idx_out[((size_t)b * Hkv + g) * top_k + j] = sIdx[j];
  } else {
    // o_cmp = sum over warps of weight x o, then the window, split over warps 1..7 in
    // 16-row tiles (its rings overlay the merge scratch, hence the barrier in between)
    merge_sum<DV>(sMerge, sCoef, sOcmp, G, 32, kThreads - 32);
    tc::named_sync(1, kThreads - 32);
    const int lo = max(0, t - window + 1);
    const int nwin = t - lo + 1;
    const int per = ((nwin + kRows - 1) / kRows + kWarps - 2) / (kWarps - 1) * kRows;
    const int r0 = min(nwin, (warp - 1) * per);
    const int n = min(nwin, r0 + per) - r0;
    auto rowk = [&](int r) { return kcache + (((size_t)b * Lmax + lo + r0 + r) * Hkv + g) * DK; };
    auto rowv = [&](int r) { return vcache + (((size_t)b * Lmax + lo + r0 + r) * Hkv + g) * DV; };
    attend_rows<DK, DV>(qf, st, rb0, rb1, n, rowk, rowv, [](int) { return true; }, scale_log2, lane);
  }
  merge_states<DV>(st, uni, sOwin, G, warp, lane);   // warp 0's state is empty

  // ---------------- B: the selected blocks ----------------
  {
    // warp w takes the chosen blocks at positions w and w + 8 (and more when top_k > 16)
    st.init();
    for (int p = warp; p < top_k; p += kWarps) {
      const int j = sIdx[p];
      if (j < 0) continue;
      const int jb = min(j, own);
      const int u0 = jb * kSel;
      const int n = min(kSel, t - u0 + 1);
      auto rowk = [&](int r) { return kcache + (((size_t)b * Lmax + u0 + r) * Hkv + g) * DK; };
      auto rowv = [&](int r) { return vcache + (((size_t)b * Lmax + u0 + r) * Hkv + g) * DV; };
      attend_rows<DK, DV>(qf, st, rb0, rb1, n, rowk, rowv, [](int) { return true; }, scale_log2, lane);
    }
    merge_states<DV>(st, uni, sOslc, G, warp, lane);
  }

  // ---------------- C: gated combine ----------------
  for (int e = tid; e < G * DV; e += kThreads) {
    const int r = e / DV, c = e % DV;
    const size_t row = (size_t)b * Hq + g * G + r;
    const float g0 = __bfloat162float(gates[row * 3]), g1 = __bfloat162float(gates[row * 3 + 1]),
                g2 = __bfloat162float(gates[row * 3 + 2]);
    out[row * DV + c] = __float2bfloat16_rn(g0 * sOcmp[e] + g1 * sOslc[e] + g2 * sOwin[e]);
  }
}

template <int DK, int DV>
cudaError_t launch(const DecodeArgs& a, cudaStream_t st) {
  const size_t smem = Smem<DK, DV>::kTotal;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(decode_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid(a.Hkv, a.B);
  decode_kernel<DK, DV><<<grid, kThreads, smem, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.kc),
      static_cast<const __nv_bfloat16*>(a.vc), a.seqlens, static_cast<const __nv_bfloat16*>(a.gates),
      static_cast<__nv_bfloat16*>(a.out), a.idx, a.Lmax, a.Ncmax, a.max_seqlen, a.Hq, a.Hkv, a.G, a.top_k, a.window,
      a.force_first, a.force_local, a.scale_log2, a.w_straddle);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st) {
  if (a.dk == 64 && a.dv == 64) return launch<64, 64>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch<128, 128>(a, st);
  if (a.dk == 192 && a.dv == 128) return launch<192, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
