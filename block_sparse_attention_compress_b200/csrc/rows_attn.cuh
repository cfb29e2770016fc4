// Warp-level attention over gathered K/V rows, shared by the decode kernel and the DSA
// token-sparse attention: 8 warps each stream rows (16 at a time, through a 2-stage per-warp
// cp.async ring) with an online softmax over the query heads as the 16 rows of m16n8k16
// MMAs, then the warps' states are merged by log-sum-exp weights.
#pragma once

#include "common.cuh"

namespace nsa {
namespace {
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;            // rows per stage tile

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

// Online-softmax state of one warp: rows gl and gl+8 (two heads per lane quad).
template <int DV>
struct State {
  float m0, m1, l0, l1;
  float o[DV / 8][4];
  __device__ void init() {
    m0 = m1 = -INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int j = 0; j < DV / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  }
};

template <int DK, int DV>
struct Tile {
  __nv_bfloat16* k;  // [kRows][DK] swizzled
  __nv_bfloat16* v;  // [kRows][DV] swizzled
};

// Issue the copies of rows [r0, r0+16) of a K/V source into a stage; rows >= n are zero-filled.
// Eight lanes cover one 128-byte line of a row, so each copy instruction moves four whole lines
// (rows lane / 8 + 4m); each lane looks its four rows up once and steps through their lines.
template <int DK, int DV, class RowK, class RowV>
__device__ __forceinline__ void load_rows(Tile<DK, DV> st, int r0, int n, RowK rowk, RowV rowv, int lane) {
  static_assert(DK % 64 == 0 && DV % 64 == 0, "rows are whole 128-byte lines");
  const int rq = lane >> 3, cl = lane & 7;
#pragma unroll
  for (int m = 0; m < kRows / 4; ++m) {
    const int r = rq + 4 * m;
    const bool ok = r0 + r < n;
    const __nv_bfloat16* pk = rowk(ok ? r0 + r : 0);
    const __nv_bfloat16* pv = rowv(ok ? r0 + r : 0);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x)
      cp_async16(st.k + SwzTile<DK>::offset(r, cl + 8 * x), pk + (cl + 8 * x) * 8, ok);
#pragma unroll
    for (int x = 0; x < DV / 64; ++x)
      cp_async16(st.v + SwzTile<DV>::offset(r, cl + 8 * x), pv + (cl + 8 * x) * 8, ok);
  }
}

// S = Q K^T for one 16-row tile (two n-tiles), already scaled to log2 units.
template <int DK>
__device__ __forceinline__ void qk_tile(const uint32_t (&qf)[DK / 16][4], const __nv_bfloat16* k, float (&s)[2][4],
                                        float scale_log2, int lane) {
#pragma unroll
  for (int j = 0; j < 2; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < DK / 16; ++ks) {
    uint32_t b0, b1, b2, b3;
    const int row = (lane & 7) + ((lane >> 4) << 3);
    const int ch = 2 * ks + ((lane >> 3) & 1);
    ldsm_x4(b0, b1, b2, b3, smem_u32(k + SwzTile<DK>::offset(row, ch)));
    mma16816(s[0], qf[ks], b0, b1);
    mma16816(s[1], qf[ks], b2, b3);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[j][e] *= scale_log2;
}

// O += P V for one 16-row tile; P given as probabilities in the C-fragment layout.
template <int DV>
__device__ __forceinline__ void pv_tile(const float (&p)[2][4], const __nv_bfloat16* v, float (&o)[DV / 8][4],
                                        int lane) {
  uint32_t a[4];
  a[0] = pack_bf16(p[0][0], p[0][1]);
  a[1] = pack_bf16(p[0][2], p[0][3]);
  a[2] = pack_bf16(p[1][0], p[1][1]);
  a[3] = pack_bf16(p[1][2], p[1][3]);
#pragma unroll
  for (int np = 0; np < DV / 16; ++np) {
    uint32_t b0, b1, b2, b3;
    const int row = lane & 15;
    const int ch = 2 * np + (lane >> 4);
    ldsm_x4_t(b0, b1, b2, b3, smem_u32(v + SwzTile<DV>::offset(row, ch)));
    mma16816(o[2 * np], a, b0, b1);
    mma16816(o[2 * np + 1], a, b2, b3);
  }
}

// Online-softmax update of `st` with the masked logits `s` (masked entries are -inf);
// on return `s` holds exp2(s - m_new).  Returns the per-row rescale factors.
template <int DV>
__device__ __forceinline__ void softmax_update(State<DV>& st, float (&s)[2][4], float& c0, float& c1) {
  float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
  float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
  mx0 = warp_max4(mx0);
  mx1 = warp_max4(mx1);
  const float n0 = fmaxf(st.m0, mx0), n1 = fmaxf(st.m1, mx1);
  const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
  c0 = exp2f(st.m0 - b0);
  c1 = exp2f(st.m1 - b1);
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    s[j][0] = exp2f(s[j][0] - b0); s[j][1] = exp2f(s[j][1] - b0);
    s[j][2] = exp2f(s[j][2] - b1); s[j][3] = exp2f(s[j][3] - b1);
    sum0 += s[j][0] + s[j][1];
    sum1 += s[j][2] + s[j][3];
  }
  st.l0 = st.l0 * c0 + warp_sum4(sum0);
  st.l1 = st.l1 * c1 + warp_sum4(sum1);
  st.m0 = n0;
  st.m1 = n1;
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) {
    st.o[j][0] *= c0; st.o[j][1] *= c0; st.o[j][2] *= c1; st.o[j][3] *= c1;
  }
}

// Stream rows [0, n) of a K/V source through the warp's ring with one softmax.
template <int DK, int DV, class RowK, class RowV, class Valid>
__device__ void attend_rows(const uint32_t (&qf)[DK / 16][4], State<DV>& st, Tile<DK, DV> ring0,
                            Tile<DK, DV> ring1, int n, RowK rowk, RowV rowv, Valid valid, float scale_log2,
                            int lane) {
  const int ntiles = (n + kRows - 1) / kRows;
  if (ntiles == 0) return;
  load_rows<DK, DV>(ring0, 0, n, rowk, rowv, lane);
  cp_async_commit();
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) load_rows<DK, DV>((it + 1) & 1 ? ring1 : ring0, (it + 1) * kRows, n, rowk, rowv, lane);
    cp_async_commit();
    cp_async_wait<1>();
    __syncwarp();
    const Tile<DK, DV> cur = (it & 1) ? ring1 : ring0;
    float s[2][4];
    qk_tile<DK>(qf, cur.k, s, scale_log2, lane);
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = it * kRows + j * 8 + 2 * (lane & 3) + e;
        if (!(r < n && valid(r))) { s[j][e] = -INFINITY; s[j][2 + e] = -INFINITY; }
      }
    float c0, c1;
    softmax_update<DV>(st, s, c0, c1);
    pv_tile<DV>(s, cur.v, st.o, lane);
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncwarp();
}

// Shared-memory scratch of the cross-warp merges: per warp 16 rows of DV floats, each row
// padded by 8 floats so that the float2 stores of a C fragment (8 rows x 4 column pairs per
// half-warp) fall on 32 distinct banks.
template <int DV>
struct MergeBuf {
  static constexpr int kStride = DV + 8;
  static constexpr size_t kBytes = (size_t)kWarps * 16 * kStride * 4;
  __device__ static float* row(float* base, int w, int r) { return base + (w * 16 + r) * kStride; }
};

// Store the warp's (scaled) accumulator rows into its slot of the merge scratch.
template <int DV>
__device__ __forceinline__ void store_o(float* sO, const State<DV>& st, float f0, float f1, int warp, int lane) {
  const int gl = lane >> 2, cq = lane & 3;
  float* r0 = MergeBuf<DV>::row(sO, warp, gl) + 2 * cq;
  float* r1 = MergeBuf<DV>::row(sO, warp, gl + 8) + 2 * cq;
#pragma unroll
  for (int j = 0; j < DV / 8; ++j) {
    *reinterpret_cast<float2*>(r0 + j * 8) = make_float2(st.o[j][0] * f0, st.o[j][1] * f0);
    *reinterpret_cast<float2*>(r1 + j * 8) = make_float2(st.o[j][2] * f1, st.o[j][3] * f1);
  }
}

__device__ __forceinline__ void store_ml(float* sML, float m0, float l0, float m1, float l1, int warp, int lane) {
  const int gl = lane >> 2;
  if ((lane & 3) == 0) {
    sML[(warp * 16 + gl) * 2] = m0;
    sML[(warp * 16 + gl) * 2 + 1] = l0;
    sML[(warp * 16 + gl + 8) * 2] = m1;
    sML[(warp * 16 + gl + 8) * 2 + 1] = l1;
  }
}

// For row r (tid < 16): coef[w][r] = 2^(m_w - lse) with lse the log2-sum-exp over the warps'
// (m, l); the normalised merged row is sum_w coef[w][r] * o_w.  Rows >= G or with no
// visible key get coefficient 0.
__device__ __forceinline__ void merge_coefs(const float* sML, float* sCoef, int G, int r) {
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sML[(w * 16 + r) * 2]);
  float Ls = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) Ls += exp2f(sML[(w * 16 + r) * 2] - M) * sML[(w * 16 + r) * 2 + 1];
  }
  const float lse = (r < G && Ls > 0.f) ? M + __log2f(Ls) : INFINITY;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) sCoef[w * 16 + r] = exp2f(sML[(w * 16 + r) * 2] - lse);
}

// dst[r][c] = sum_w coef[w][r] * sO[w][r][c] for r < G, over threads [t0, t0 + nthr).
template <int DV>
__device__ __forceinline__ void merge_sum(const float* sO, const float* sCoef, float* dst, int G, int t0, int nthr) {
  for (int e = threadIdx.x - t0; e < G * DV; e += nthr) {
    const int r = e / DV, c = e % DV;
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      acc += sCoef[w * 16 + r] * MergeBuf<DV>::row(const_cast<float*>(sO), w, r)[c];
    dst[r * DV + c] = acc;
  }
}

// Merge the 8 warps' states into normalised rows (r < G) of sOut [16][DV].  The scratch
// (MergeBuf bytes, then 16 x kWarps coefficients and 16 x kWarps x 2 (m, l)) overlays the
// stage rings, so the call starts with a barrier.
template <int DV>
__device__ void merge_states(const State<DV>& st, uint8_t* scratch, float* sOut, int G, int warp, int lane) {
  float* sO = reinterpret_cast<float*>(scratch);
  float* sCoef = reinterpret_cast<float*>(scratch + MergeBuf<DV>::kBytes);
  float* sML = sCoef + kWarps * 16;
  __syncthreads();   // every warp is done with its stage ring
  store_o<DV>(sO, st, 1.f, 1.f, warp, lane);
  store_ml(sML, st.m0, st.l0, st.m1, st.l1, warp, lane);
  __syncthreads();
  if (threadIdx.x < 16) merge_coefs(sML, sCoef, G, threadIdx.x);
  __syncthreads();
  merge_sum<DV>(sO, sCoef, sOut, G, 0, kThreads);
  __syncthreads();
}

}  // namespace
}  // namespace nsa
