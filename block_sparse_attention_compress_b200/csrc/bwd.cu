// Backward of the NSA forward: gradients of q, k, v, the gates and the phi weights from the
// gradient of the output ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §13: NSA is trained
// natively, forward and backward; the chosen blocks are a discrete choice with no gradient).
//
// bwd_attn_kernel, one CTA per (batch, token t, KV group), 8 warps, the group's G <= 16 heads as
// the 16 rows of m16n8k16 MMAs.  For each branch (compressed, selected, window), with its gate
// g and output o (all per head):
//   pass 1  o and the log-sum-exp of the branch, recomputed (online softmax over its rows);
//           dgate = dout . o and D = g * (dout . o);
//   pass 2  per 16-row tile: P = exp(S - lse), dP = g * (dout V^T), dS = P * (dP - D);
//           dQ += dS K (registers); dK_rows += dS^T Q and dV_rows += (g P)^T dout, added to
//           the fp32 gradient buffers of the rows (K/V rows, or Kc/Vc rows) with atomics.
//   dq = scale * dQ, summed over the warps in shared memory.
// phi's backward (per KV head, keys and values alike):
//   bwd_phi_dx_kernel  dX[u] += sum over the compressed blocks i covering token u of
//                      W[(u - s*i)*d : (u - s*i + 1)*d, :] . dXc[i];
//   bwd_phi_dw_kernel  dW[r*d + c, j] = sum over (b, h, i) of X[b, s*i + r, h, c] * dXc[b, i, h, j].
// phi as the two-layer MLP (hidden = bf16(GELU(pre)), pre = vec(block) @ W1 + b1, Xc = hidden @ W2),
// from dXc:
//   bwd_mlp_dw2_kernel   dW2[j, m] = sum over the rows (b, i, h) of hidden[j] * dXc[m];
//   bwd_mlp_dpre_kernel  dpre[j] = (sum_m dXc[m] W2[j, m]) * GELU'(pre[j]), written over pre;
//   bwd_mlp_db_kernel    db1[j] = sum over the rows of dpre[j];
//   then the linear kernels above with dpre for dXc and W1 for W give dW1 and dX.
// Each warp streams its tiles through two shared-memory stages (the next tile is requested
// before the current one is waited for); the row gradients are float4 atomics (one per lane
// and 8 columns of a row).
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "rows_attn.cuh"

namespace nsa {

namespace {
constexpr int kL = 32, kS = 16, kSel = 64;

template <int DK, int DV>
struct BwdSmem {
  static constexpr size_t kStage = (size_t)kRows * (DK + DV) * 2;            // one tile (K then V)
  static constexpr size_t kRings = (size_t)kWarps * 2 * kStage;              // two stages per warp
  static constexpr size_t kMerge = MergeBuf<DV>::kBytes + (size_t)kWarps * 16 * 3 * 4;
  static constexpr size_t kU = kRings > kMerge ? kRings : kMerge;            // rings / merge scratch
  static constexpr size_t kQ = kU;                                           // Q bf16 [16][DK]
  static constexpr size_t kDO = kQ + 16 * DK * 2;                            // dout bf16 [16][DV]
  static constexpr size_t kX = kDO + 16 * DV * 2;                            // per warp [16][16] bf16
  static constexpr size_t kO = kX + (size_t)kWarps * 16 * 16 * 2;            // o of the branch [16][DV] fp32
  static constexpr size_t kDQ = kO + 16 * DV * 4;                            // dq [16][DK] fp32
  static constexpr size_t kRow = kDQ + 16 * DK * 4;                          // lse, D, gate [16] each
  static constexpr size_t kIdx = kRow + 3 * 16 * 4;                          // the chosen blocks [<= 32]
  static constexpr size_t kTotal = kIdx + 32 * 4;
  static_assert(kTotal <= 232448, "backward shared memory");
};

// A = X^T for X [16 rows][16 cols] bf16 (row stride 16): the m16k16 fragment of the transpose.
__device__ __forceinline__ void load_at(const __nv_bfloat16* X, uint32_t (&a)[4], int lane) {
  const int mi = lane >> 3, ri = lane & 7;
  const int row = (mi >> 1) * 8 + ri, col = (mi & 1) * 8;
  ldsm_x4_t(a[0], a[1], a[2], a[3], smem_u32(X + row * 16 + col));
}

// out[16][N] += A (16 x 16) . B, B = [16 rows][N] bf16 in the SwzTile<N> layout.
template <int N>
__device__ __forceinline__ void mma_ab(const uint32_t (&a)[4], const __nv_bfloat16* B, float (&out)[N / 8][4],
                                       int lane) {
#pragma unroll
  for (int np = 0; np < N / 16; ++np) {
    uint32_t b0, b1, b2, b3;
    const int row = lane & 15;
    const int ch = 2 * np + (lane >> 4);
    ldsm_x4_t(b0, b1, b2, b3, smem_u32(B + SwzTile<N>::offset(row, ch)));
    mma16816(out[2 * np], a, b0, b1);
    mma16816(out[2 * np + 1], a, b2, b3);
  }
}

// Adds a 16-row x (8 NX)-column MMA accumulator to the row gradients, scaled by sc, with one
// float4 atomic per lane and 8 columns: lanes cq and cq ^ 1 swap half their pairs, so that the
// even lane holds columns 4 (cq / 2) .. + 3 of row gl and the odd lane the same columns of row
// gl + 8.  dst is the lane's row (row gl for an even cq, gl + 8 for an odd one), or null when
// that row is masked; every lane takes part in the shuffles.
template <int NX>
__device__ __forceinline__ void red_rows(const float (&acc)[NX][4], float* dst, float sc, int cq) {
  const bool odd = cq & 1;
  const int col = 4 * (cq >> 1);
#pragma unroll
  for (int x = 0; x < NX; ++x) {
    const float s0 = odd ? acc[x][0] : acc[x][2], s1 = odd ? acc[x][1] : acc[x][3];
    const float r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
    const float4 val = odd ? make_float4(sc * r0, sc * r1, sc * acc[x][2], sc * acc[x][3])
                           : make_float4(sc * acc[x][0], sc * acc[x][1], sc * r0, sc * r1);
    if (dst) atomicAdd(reinterpret_cast<float4*>(dst + x * 8 + col), val);
  }
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ kc,
                const __nv_bfloat16* __restrict__ vc, const __nv_bfloat16* __restrict__ gates,
                const __nv_bfloat16* __restrict__ dout, const int32_t* __restrict__ idx, float* __restrict__ dq,
                float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dkc, float* __restrict__ dvc,
                float* __restrict__ dgates, int T, int Hq, int Hkv, int G, int nc, int top_k, int window,
                float scale_log2, const int32_t* __restrict__ cu) {
  using SM = BwdSmem<DK, DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  // sequence b's rows of q, k, v, gates, dout and the gradients start at row `base` (packed
  // variable-length batch: cu[b]); its tokens past its length have no work
  const int base = seq_base(cu, b, T);
  if (t >= seq_len(cu, b, T)) return;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + SM::kQ);
  __nv_bfloat16* sDO = reinterpret_cast<__nv_bfloat16*>(smem + SM::kDO);
  __nv_bfloat16* sX = reinterpret_cast<__nv_bfloat16*>(smem + SM::kX) + warp * 256;
  float* sO = reinterpret_cast<float*>(smem + SM::kO);
  float* sDQ = reinterpret_cast<float*>(smem + SM::kDQ);
  float* sLse = reinterpret_cast<float*>(smem + SM::kRow);
  float* sD = sLse + 16;
  float* sG = sD + 16;
  int* sIdx = reinterpret_cast<int*>(smem + SM::kIdx);
  static_assert(kThreads == 256, "the dgate sums take 16 threads per head row");
  const size_t row0 = ((size_t)base + t) * Hq + g * G;   // the group's first head row of this token
  for (int e = tid; e < 16 * (DK / 8); e += kThreads) {
    const int r = e / (DK / 8), ch = e % (DK / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < G) val = *reinterpret_cast<const uint4*>(q + (row0 + r) * DK + ch * 8);
    *reinterpret_cast<uint4*>(sQ + SwzTile<DK>::offset(r, ch)) = val;
  }
  for (int e = tid; e < 16 * (DV / 8); e += kThreads) {
    const int r = e / (DV / 8), ch = e % (DV / 8);
    uint4 val = make_uint4(0, 0, 0, 0);
    if (r < G) val = *reinterpret_cast<const uint4*>(dout + (row0 + r) * DV + ch * 8);
    *reinterpret_cast<uint4*>(sDO + SwzTile<DV>::offset(r, ch)) = val;
  }
  for (int e = tid; e < 16 * DK; e += kThreads) sDQ[e] = 0.f;
  const int32_t* myidx = idx + (((size_t)b * Hkv + g) * T + t) * top_k;
  for (int e = tid; e < top_k; e += kThreads) sIdx[e] = myidx[e];
  __syncthreads();
  uint32_t qf[DK / 16][4], df[DV / 16][4];
#pragma unroll
  for (int ks = 0; ks < DK / 16; ++ks) {
    const int row = lane & 15, ch = 2 * ks + (lane >> 4);
    ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(sQ + SwzTile<DK>::offset(row, ch)));
  }
#pragma unroll
  for (int ks = 0; ks < DV / 16; ++ks) {
    const int row = lane & 15, ch = 2 * ks + (lane >> 4);
    ldsm_x4(df[ks][0], df[ks][1], df[ks][2], df[ks][3], smem_u32(sDO + SwzTile<DV>::offset(row, ch)));
  }
  float dqa[DK / 8][4];
#pragma unroll
  for (int j = 0; j < DK / 8; ++j) dqa[j][0] = dqa[j][1] = dqa[j][2] = dqa[j][3] = 0.f;
  Tile<DK, DV> t0{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)warp * 2 * SM::kStage), nullptr};
  t0.v = t0.k + kRows * DK;
  Tile<DK, DV> t1{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)(warp * 2 + 1) * SM::kStage), nullptr};
  t1.v = t1.k + kRows * DK;
  const int own = t / kSel;

  for (int br = 0; br < 3; ++br) {   // 0 compressed, 1 selected, 2 window
    // the branch's rows: global row of row r, or -1 when it is masked
    int n = 0, lo = 0;
    if (br == 0) n = t < kL - 1 ? 0 : min(nc, (t - kL + 1) / kS + 1);
    else if (br == 1) n = top_k * kSel;
    else { lo = max(0, t - window + 1); n = t - lo + 1; }
    auto row_of = [&](int r) -> int {
      if (br == 0) return r;
      if (br == 2) return lo + r;
      const int j = sIdx[r / kSel];
      if (j < 0) return -1;
      const int u = min(j, own) * kSel + r % kSel;
      return u <= t ? u : -1;
    };
    const __nv_bfloat16* kb = br == 0 ? kc + ((size_t)b * nc * Hkv + g) * DK : k + ((size_t)base * Hkv + g) * DK;
    const __nv_bfloat16* vb = br == 0 ? vc + ((size_t)b * nc * Hkv + g) * DV : v + ((size_t)base * Hkv + g) * DV;
    const int ntiles = (n + kRows - 1) / kRows;
    // Lane l loads row l & 15 of a tile (chunks of parity l >> 4) and holds that row's global
    // index, -1 when the row is masked or past n; the masks of the other rows come from it by
    // shuffles.  Each warp takes tiles warp, warp + 8, ... through its two stages: the next
    // one is requested before the current one is waited for.
    auto tile_row = [&](int it) {
      const int r = it * kRows + (lane & 15);
      return r < n ? row_of(r) : -1;
    };
    auto issue = [&](int it, int slot, int u) {
      if (it < ntiles) {
        const Tile<DK, DV> dst = slot ? t1 : t0;
        const int rr = lane & 15, half = lane >> 4;
        const __nv_bfloat16* sk = kb + (size_t)max(u, 0) * Hkv * DK;
        const __nv_bfloat16* sv = vb + (size_t)max(u, 0) * Hkv * DV;
#pragma unroll
        for (int c = 0; c < DK / 16; ++c)
          cp_async16(dst.k + SwzTile<DK>::offset(rr, 2 * c + half), sk + (2 * c + half) * 8, u >= 0);
#pragma unroll
        for (int c = 0; c < DV / 16; ++c)
          cp_async16(dst.v + SwzTile<DV>::offset(rr, 2 * c + half), sv + (2 * c + half) * 8, u >= 0);
      }
      cp_async_commit();
    };
    auto scores = [&](const __nv_bfloat16* tk, int u, float (&s)[2][4]) {   // masked S of the tile, log2 units
      qk_tile<DK>(qf, tk, s, scale_log2, lane);
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (__shfl_sync(0xffffffffu, u, j * 8 + 2 * cq + e) < 0) { s[j][e] = -INFINITY; s[j][2 + e] = -INFINITY; }
    };
    // ---- pass 1: o and log-sum-exp of the branch
    State<DV> st;
    st.init();
    int u_cur = tile_row(warp);
    issue(warp, 0, u_cur);
    for (int it = warp, slot = 0; it < ntiles; it += kWarps, slot ^= 1) {
      const int u_nxt = tile_row(it + kWarps);
      issue(it + kWarps, slot ^ 1, u_nxt);
      cp_async_wait<1>();
      __syncwarp();
      const Tile<DK, DV> cur = slot ? t1 : t0;
      float s[2][4];
      scores(cur.k, u_cur, s);
      float c0, c1;
      softmax_update<DV>(st, s, c0, c1);
      pv_tile<DV>(s, cur.v, st.o, lane);
      __syncwarp();
      u_cur = u_nxt;
    }
    cp_async_wait<0>();
    {
      float* mO = reinterpret_cast<float*>(smem);
      float* mCoef = reinterpret_cast<float*>(smem + MergeBuf<DV>::kBytes);
      float* mML = mCoef + kWarps * 16;
      __syncthreads();
      store_o<DV>(mO, st, 1.f, 1.f, warp, lane);
      store_ml(mML, st.m0, st.l0, st.m1, st.l1, warp, lane);
      __syncthreads();
      if (tid < 16) {   // per head: lse (log2 units) and each warp's weight
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mML[(w * 16 + tid) * 2]);
        float L = 0.f;
        if (M != -INFINITY)
          for (int w = 0; w < kWarps; ++w) L += exp2f(mML[(w * 16 + tid) * 2] - M) * mML[(w * 16 + tid) * 2 + 1];
        const float lse = (tid < G && L > 0.f) ? M + __log2f(L) : INFINITY;
        sLse[tid] = lse;
        for (int w = 0; w < kWarps; ++w) mCoef[w * 16 + tid] = exp2f(mML[(w * 16 + tid) * 2] - lse);
      }
      __syncthreads();
      merge_sum<DV>(mO, mCoef, sO, G, 0, kThreads);
      __syncthreads();
      {   // dgate = dout . o and D = g * dgate: 16 threads per head row, 8 columns at a time
        const int r = tid >> 4, part = tid & 15;
        float dg = 0.f;
        if (r < G)
          for (int ch = part; ch < DV / 8; ch += 16) {
            const __nv_bfloat16* d8 = sDO + SwzTile<DV>::offset(r, ch);
            const float* o8 = sO + r * DV + ch * 8;
#pragma unroll
            for (int i = 0; i < 8; ++i) dg += __bfloat162float(d8[i]) * o8[i];
          }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) dg += __shfl_xor_sync(0xffffffffu, dg, off);
        if (part == 0) {
          const float gb = r < G ? __bfloat162float(gates[(row0 + r) * 3 + br]) : 0.f;
          sD[r] = gb * dg;
          sG[r] = gb;
          if (r < G) dgates[(row0 + r) * 3 + br] = dg;
        }
      }
      __syncthreads();
    }
    const float g0 = sG[gl], g1 = sG[gl + 8];
    const float lse0 = sLse[gl], lse1 = sLse[gl + 8], D0 = sD[gl], D1 = sD[gl + 8];
    __syncthreads();   // the merge scratch becomes the tiles again
    // ---- pass 2: dS and the gradients
    u_cur = tile_row(warp);
    issue(warp, 0, u_cur);
    for (int it = warp, slot = 0; it < ntiles; it += kWarps, slot ^= 1) {
      const int u_nxt = tile_row(it + kWarps);
      issue(it + kWarps, slot ^ 1, u_nxt);
      cp_async_wait<1>();
      __syncwarp();
      const Tile<DK, DV> cur = slot ? t1 : t0;
      // this lane's row of the float4 gradient adds: gl for an even cq, gl + 8 for an odd one
      const int u_add = __shfl_sync(0xffffffffu, u_cur, gl + 8 * (cq & 1));
      float s[2][4], dp[2][4];
      scores(cur.k, u_cur, s);
      qk_tile<DV>(df, cur.v, dp, 1.f, lane);   // dout V^T
      float p[2][4], ds[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        p[j][0] = exp2f(s[j][0] - lse0); p[j][1] = exp2f(s[j][1] - lse0);
        p[j][2] = exp2f(s[j][2] - lse1); p[j][3] = exp2f(s[j][3] - lse1);
        ds[j][0] = p[j][0] * (g0 * dp[j][0] - D0); ds[j][1] = p[j][1] * (g0 * dp[j][1] - D0);
        ds[j][2] = p[j][2] * (g1 * dp[j][2] - D1); ds[j][3] = p[j][3] * (g1 * dp[j][3] - D1);
      }
      pv_tile<DK>(ds, cur.k, dqa, lane);   // dQ += dS K
      // dK rows += dS^T Q, then dV rows += (g P)^T dout, through the per-warp [16 heads][16 rows] tile
#pragma unroll
      for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int c = j * 8 + 2 * cq;
          const float x00 = pass ? g0 * p[j][0] : ds[j][0], x01 = pass ? g0 * p[j][1] : ds[j][1];
          const float x10 = pass ? g1 * p[j][2] : ds[j][2], x11 = pass ? g1 * p[j][3] : ds[j][3];
          *reinterpret_cast<uint32_t*>(sX + gl * 16 + c) = pack_bf16(x00, x01);
          *reinterpret_cast<uint32_t*>(sX + (gl + 8) * 16 + c) = pack_bf16(x10, x11);
        }
        __syncwarp();
        uint32_t a[4];
        load_at(sX, a, lane);
        __syncwarp();
        if (pass == 0) {
          float acc[DK / 8][4];
#pragma unroll
          for (int x = 0; x < DK / 8; ++x) acc[x][0] = acc[x][1] = acc[x][2] = acc[x][3] = 0.f;
          mma_ab<DK>(a, sQ, acc, lane);
          const int u = u_add;
          float* dst = u < 0 ? nullptr
                             : br == 0 ? dkc + (((size_t)b * nc + u) * Hkv + g) * DK
                                       : dk + (((size_t)base + u) * Hkv + g) * DK;
          red_rows<DK / 8>(acc, dst, scale_log2 * 0.69314718055994531f, cq);   // times the softmax scale
        } else {
          float acc[DV / 8][4];
#pragma unroll
          for (int x = 0; x < DV / 8; ++x) acc[x][0] = acc[x][1] = acc[x][2] = acc[x][3] = 0.f;
          mma_ab<DV>(a, sDO, acc, lane);
          const int u = u_add;
          float* dst = u < 0 ? nullptr
                             : br == 0 ? dvc + (((size_t)b * nc + u) * Hkv + g) * DV
                                       : dv + (((size_t)base + u) * Hkv + g) * DV;
          red_rows<DV / 8>(acc, dst, 1.f, cq);
        }
      }
      __syncwarp();
      u_cur = u_nxt;
    }
    cp_async_wait<0>();
    __syncthreads();   // before the next branch reuses the tiles and the merge scratch
  }
  // dq = scale * sum over the warps of dS K
#pragma unroll
  for (int x = 0; x < DK / 8; ++x) {
    atomicAdd(sDQ + gl * DK + x * 8 + 2 * cq, dqa[x][0]);
    atomicAdd(sDQ + gl * DK + x * 8 + 2 * cq + 1, dqa[x][1]);
    atomicAdd(sDQ + (gl + 8) * DK + x * 8 + 2 * cq, dqa[x][2]);
    atomicAdd(sDQ + (gl + 8) * DK + x * 8 + 2 * cq + 1, dqa[x][3]);
  }
  __syncthreads();
  const float sc = scale_log2 * 0.69314718055994531f;
  for (int e = tid; e < G * DK; e += kThreads) dq[row0 * DK + e] = sc * sDQ[e];
}

// dX[b, u, h, c] += sum over i with s*i <= u < s*i + l of sum_j W[(u - s*i)*D + c, j] dXc[b, i, h, j].
// One warp per (b, u, h): the lanes split j (each holds D/32 values of dXc[i]) and read the W
// rows contiguously; each output c is a warp sum.
template <int D>
__global__ void __launch_bounds__(256)
bwd_phi_dx_kernel(const __nv_bfloat16* __restrict__ w, const float* __restrict__ dxc, float* __restrict__ dx, int B,
                  int T, int H, int nc, const int32_t* __restrict__ cu) {
  const long gw = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= (long)B * T * H) return;
  const int h = (int)(gw % H), u = (int)((gw / H) % T), b = (int)(gw / ((long)H * T));
  if (u >= seq_len(cu, b, T)) return;
  float* dst = dx + (((size_t)seq_base(cu, b, T) + u) * H + h) * D;
  for (int i = max(0, (u - kL) / kS); i <= u / kS && i < nc; ++i) {
    const int r = u - kS * i;
    if (r < 0 || r >= kL) continue;
    const float* gi = dxc + (((size_t)b * nc + i) * H + h) * D;
    float gj[D / 32];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) gj[x] = gi[x * 32 + lane];
    for (int c = 0; c < D; ++c) {
      const __nv_bfloat16* wr = w + ((size_t)r * D + c) * D;
      float part = 0.f;
#pragma unroll
      for (int x = 0; x < D / 32; ++x) part += __bfloat162float(wr[x * 32 + lane]) * gj[x];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane == (c & 31)) dst[c] += part;   // spread the stores over the lanes
    }
  }
}

// dW[r*D + c, j] = sum over (b, h, i) of X[b, s*i + r, h, c] * dXc[b, i, h, j]: one thread per
// output element, a loop over every compressed block.
template <int D>
__global__ void __launch_bounds__(256)
bwd_phi_dw_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ dxc, float* __restrict__ dw, int B,
                  int T, int H, int nc, const int32_t* __restrict__ cu) {
  const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (size_t)kL * D * D) return;
  const int j = (int)(e % D), rc = (int)(e / D), r = rc / D, c = rc % D;
  float acc = 0.f;
  for (int b = 0; b < B; ++b) {
    const int base = seq_base(cu, b, T), len = seq_len(cu, b, T);
    const int nc_b = len < kL ? 0 : min(nc, (len - kL) / kS + 1);   // the sequence's own blocks
    for (int i = 0; i < nc_b; ++i)
      for (int h = 0; h < H; ++h)
        acc += __bfloat162float(x[(((size_t)base + kS * i + r) * H + h) * D + c]) *
               dxc[(((size_t)b * nc + i) * H + h) * D + j];
  }
  dw[e] = acc;
}

// d/dx of x * Phi(x): Phi(x) + x * phi(x), with Phi the normal CDF and phi its density
__device__ __forceinline__ float gelu_grad(float x) {
  return 0.5f * (1.f + erff(x * 0.70710678118654752f)) + x * 0.39894228040143268f * expf(-0.5f * x * x);
}

// One warp per row: the lanes split m; each j is a warp sum, kept by lane j % 32.
template <int D>
__global__ void __launch_bounds__(256)
bwd_mlp_dpre_kernel(const __nv_bfloat16* __restrict__ w2, const float* __restrict__ dxc, float* __restrict__ pre,
                    long rows) {
  const long gw = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= rows) return;
  float gm[D / 32];
#pragma unroll
  for (int x = 0; x < D / 32; ++x) gm[x] = dxc[gw * D + x * 32 + lane];
  float* pr = pre + gw * D;
  for (int j = 0; j < D; ++j) {
    const __nv_bfloat16* wr = w2 + (size_t)j * D;
    float part = 0.f;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) part += __bfloat162float(wr[x * 32 + lane]) * gm[x];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (lane == (j & 31)) pr[j] = part * gelu_grad(pr[j]);
  }
}

// One thread per output (j, m), a loop over the rows.
template <int D>
__global__ void __launch_bounds__(256)
bwd_mlp_dw2_kernel(const __nv_bfloat16* __restrict__ hidden, const float* __restrict__ dxc, float* __restrict__ dw2,
                   long rows) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= D * D) return;
  const int j = e / D, m = e % D;
  float acc = 0.f;
  for (long r = 0; r < rows; ++r) acc += __bfloat162float(hidden[r * D + j]) * dxc[r * D + m];
  dw2[e] = acc;
}

template <int D>
__global__ void __launch_bounds__(256)
bwd_mlp_db_kernel(const float* __restrict__ dpre, float* __restrict__ db, long rows) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= D) return;
  float acc = 0.f;
  for (long r = 0; r < rows; ++r) acc += dpre[r * D + j];
  db[j] = acc;
}

template <int D>
cudaError_t launch_mlp_tail(const void* w2, const void* hidden, const float* dxc, float* pre, float* dw2, float* db,
                            long rows, cudaStream_t st) {
  if (rows > 0) {
    bwd_mlp_dw2_kernel<D><<<(D * D + 255) / 256, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(hidden), dxc, dw2,
                                                                 rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    bwd_mlp_dpre_kernel<D><<<(unsigned)((rows * 32 + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w2),
                                                                                  dxc, pre, rows);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    cudaError_t e = cudaMemsetAsync(dw2, 0, (size_t)D * D * 4, st);
    if (e != cudaSuccess) return e;
  }
  bwd_mlp_db_kernel<D><<<1, 256, 0, st>>>(pre, db, rows);
  return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_attn(const BwdArgs& a, cudaStream_t st) {
  using SM = BwdSmem<DK, DV>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e =
        cudaFuncSetAttribute(bwd_attn_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kTotal);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  bwd_attn_kernel<DK, DV><<<dim3(a.T, a.Hkv, a.B), kThreads, SM::kTotal, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.kc),
      static_cast<const __nv_bfloat16*>(a.vc), static_cast<const __nv_bfloat16*>(a.gates),
      static_cast<const __nv_bfloat16*>(a.dout), a.idx, a.dq, a.gk, a.gv, a.gkc, a.gvc, a.dgates, a.T, a.Hq, a.Hkv,
      a.G, a.nc, a.top_k, a.window, a.scale_log2, a.cu);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_phi(const void* x, const void* w, const float* dxc, float* dx, float* dw, int B, int T, int H,
                       int nc, const int32_t* cu, cudaStream_t st) {
  if (nc == 0) return cudaSuccess;
  const long warps = (long)B * T * H;
  bwd_phi_dx_kernel<D><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(w), dxc, dx, B, T, H, nc, cu);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t n = (size_t)kL * D * D;
  bwd_phi_dw_kernel<D><<<(unsigned)((n + 255) / 256), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), dxc, dw, B,
                                                                    T, H, nc, cu);
  return cudaGetLastError();
}

cudaError_t phi_dispatch(int d, const void* x, const void* w, const float* dxc, float* dx, float* dw, int B, int T,
                         int H, int nc, const int32_t* cu, cudaStream_t st) {
  switch (d) {
    case 64: return launch_phi<64>(x, w, dxc, dx, dw, B, T, H, nc, cu, st);
    case 128: return launch_phi<128>(x, w, dxc, dx, dw, B, T, H, nc, cu, st);
    case 192: return launch_phi<192>(x, w, dxc, dx, dw, B, T, H, nc, cu, st);
    default: return cudaErrorInvalidValue;
  }
}
cudaError_t mlp_tail_dispatch(int d, const void* w2, const void* hidden, const float* dxc, float* pre, float* dw2,
                              float* db, long rows, cudaStream_t st) {
  switch (d) {
    case 64: return launch_mlp_tail<64>(w2, hidden, dxc, pre, dw2, db, rows, st);
    case 128: return launch_mlp_tail<128>(w2, hidden, dxc, pre, dw2, db, rows, st);
    case 192: return launch_mlp_tail<192>(w2, hidden, dxc, pre, dw2, db, rows, st);
    default: return cudaErrorInvalidValue;
  }
}
}  // namespace

cudaError_t launch_backward(const BwdArgs& a, cudaStream_t st) {
  cudaError_t e = cudaErrorInvalidValue;
  if (a.dk == 192 && a.dv == 128) e = launch_attn<192, 128>(a, st);
  else if (a.dk == 128 && a.dv == 128) e = launch_attn<128, 128>(a, st);
  else if (a.dk == 64 && a.dv == 64) e = launch_attn<64, 64>(a, st);
  if (e != cudaSuccess) return e;
  const float* dxk = a.gkc;
  const float* dxv = a.gvc;
  if (a.mlp) {   // through the MLP's second layer and GELU: dpre takes the place of dXc
    const long rows = (long)a.B * a.nc * a.Hkv;
    e = mlp_tail_dispatch(a.dk, a.w_k2, a.hid_k, a.gkc, a.pre_k, a.dw_k2, a.db_k, rows, st);
    if (e != cudaSuccess) return e;
    e = mlp_tail_dispatch(a.dv, a.w_v2, a.hid_v, a.gvc, a.pre_v, a.dw_v2, a.db_v, rows, st);
    if (e != cudaSuccess) return e;
    dxk = a.pre_k;
    dxv = a.pre_v;
  }
  e = phi_dispatch(a.dk, a.k, a.w_k, dxk, a.gk, a.dw_k, a.B, a.T, a.Hkv, a.nc, a.cu, st);
  if (e != cudaSuccess) return e;
  return phi_dispatch(a.dv, a.v, a.w_v, dxv, a.gv, a.dw_v, a.B, a.T, a.Hkv, a.nc, a.cu, st);
}

}  // namespace nsa
