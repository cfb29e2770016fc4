// DSA: token-wise sparse attention behind a lightning indexer (10100.com, "机器之心PRO · 会员通讯
// Week 45", "Which Attention is All You Need?", section "Linear v.s. Sparse", point 6: a light
// indexer scores every earlier token, the top-k tokens are kept, and full attention runs over them).
//
//   D1 indexer   score[t, s] = sum_j w[t, j] * ReLU(q_I[t, j] . k_I[s]) for s <= t, fp32, by warp
//                MMAs over 64 x 64 (query, key) tiles, one indexer head at a time.
//   D2 top-k     per query token: radix select of the k-th largest score (order-preserving
//                integer keys, four 8-bit passes), then one pass in index order that keeps the
//                larger scores and, among the equal ones, the lowest indices -- the list comes
//                out ascending.
//   D4 attention one CTA per (token, KV group): the 8 warps stream the chosen tokens' K/V rows
//                (gathered with cp.async) with an online softmax over the group's heads, then
//                merge their states.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "rows_attn.cuh"

namespace nsa {

namespace {
constexpr int kIdxTile = 64;   // queries and keys per indexer tile
constexpr int kIdxThreads = 128;

template <int DI>
__global__ void __launch_bounds__(kIdxThreads)
dsa_indexer_kernel(const __nv_bfloat16* __restrict__ qi, const __nv_bfloat16* __restrict__ ki,
                   const __nv_bfloat16* __restrict__ wi, float* __restrict__ scores, int T, int HI) {
  const int tq = blockIdx.x, ts = blockIdx.y, b = blockIdx.z;
  if (ts > tq) return;   // keys after every query of the tile
  __shared__ __align__(128) __nv_bfloat16 sQ[kIdxTile * DI];
  __shared__ __align__(128) __nv_bfloat16 sK[kIdxTile * DI];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  const int t0 = tq * kIdxTile, s0 = ts * kIdxTile;
  for (int e = tid; e < kIdxTile * (DI / 8); e += kIdxThreads) {
    const int r = e / (DI / 8), ch = e % (DI / 8);
    const bool ok = s0 + r < T;
    cp_async16(sK + SwzTile<DI>::offset(r, ch), ki + ((size_t)b * T + (ok ? s0 + r : 0)) * DI + ch * 8, ok);
  }
  const int ta = t0 + warp * 16 + gl, tb = ta + 8;   // this thread's two query rows
  float acc[kIdxTile / 8][4];
#pragma unroll
  for (int j = 0; j < kIdxTile / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
  for (int h = 0; h < HI; ++h) {
    __syncthreads();   // the previous head's query tile is no longer read
    for (int e = tid; e < kIdxTile * (DI / 8); e += kIdxThreads) {
      const int r = e / (DI / 8), ch = e % (DI / 8);
      const bool ok = t0 + r < T;
      cp_async16(sQ + SwzTile<DI>::offset(r, ch), qi + (((size_t)b * T + (ok ? t0 + r : 0)) * HI + h) * DI + ch * 8, ok);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    uint32_t qf[DI / 16][4];
#pragma unroll
    for (int ks = 0; ks < DI / 16; ++ks) {
      const int row = warp * 16 + (lane & 15);
      const int ch = 2 * ks + (lane >> 4);
      ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(sQ + SwzTile<DI>::offset(row, ch)));
    }
    const float wa = ta < T ? __bfloat162float(wi[((size_t)b * T + ta) * HI + h]) : 0.f;
    const float wb = tb < T ? __bfloat162float(wi[((size_t)b * T + tb) * HI + h]) : 0.f;
#pragma unroll
    for (int kt = 0; kt < kIdxTile / 16; ++kt) {
      float s[2][4];
      qk_tile<DI>(qf, sK + kt * 16 * DI, s, 1.f, lane);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        acc[2 * kt + x][0] += wa * fmaxf(s[x][0], 0.f);
        acc[2 * kt + x][1] += wa * fmaxf(s[x][1], 0.f);
        acc[2 * kt + x][2] += wb * fmaxf(s[x][2], 0.f);
        acc[2 * kt + x][3] += wb * fmaxf(s[x][3], 0.f);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kIdxTile / 8; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int s = s0 + j * 8 + 2 * cq + e;
      if (s < T && ta < T && s <= ta) scores[((size_t)b * T + ta) * T + s] = acc[j][e];
      if (s < T && tb < T && s <= tb) scores[((size_t)b * T + tb) * T + s] = acc[j][2 + e];
    }
}

// Order-preserving map of a float to an unsigned integer (larger float, larger key).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTopkThreads = 256;

// Block-wide exclusive prefix count of `flag` over the CTA's threads (in thread order) and
// the total; `sw` is shared scratch of kTopkThreads / 32 ints.
__device__ __forceinline__ int block_scan(bool flag, int* sw, int& total) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) sw[warp] = __popc(bal);
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kTopkThreads / 32; ++w) {
    const int c = sw[w];
    before += w < warp ? c : 0;
    total += c;
  }
  __syncthreads();   // sw is reused by the next scan
  return before + __popc(bal & ((1u << lane) - 1u));
}

__global__ void __launch_bounds__(kTopkThreads)
dsa_topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ sel, int T, int K) {
  const int t = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int n = t + 1;
  int32_t* dst = sel + ((size_t)b * T + t) * K;
  if (n <= K) {
    for (int i = tid; i < K; i += kTopkThreads) dst[i] = i < n ? i : -1;
    return;
  }
  const float* row = scores + ((size_t)b * T + t) * T;
  __shared__ int hist[256];
  __shared__ int s_digit, s_remaining;
  __shared__ int sw[kTopkThreads / 32];
  uint32_t prefix = 0, mask = 0;
  int remaining = K;   // how many of the keys matching prefix/mask are still to be taken
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    for (int s = tid; s < n; s += kTopkThreads) {
      const uint32_t u = ordered_key(row[s]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid == 0) {   // the digit of the remaining-th largest key among the matching ones
      int cum = 0, d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= remaining) break;
        cum += hist[d];
      }
      s_digit = d;
      s_remaining = remaining - cum;
    }
    __syncthreads();
    prefix |= (uint32_t)s_digit << shift;
    mask |= 255u << shift;
    remaining = s_remaining;
    __syncthreads();   // s_digit / s_remaining are rewritten in the next pass
  }
  // keys above the threshold, plus the `remaining` lowest-index keys equal to it
  const uint32_t thr = prefix;
  int eq_before = 0, out_before = 0;
  for (int base = 0; base < n; base += kTopkThreads) {
    const int s = base + tid;
    const uint32_t u = s < n ? ordered_key(row[s]) : 0u;
    const bool gt = s < n && u > thr, eq = s < n && u == thr;
    int eq_total;
    const int eq_rank = eq_before + block_scan(eq, sw, eq_total);
    const bool take = gt || (eq && eq_rank < remaining);
    int take_total;
    const int pos = out_before + block_scan(take, sw, take_total);
    if (take && pos < K) dst[pos] = s;
    eq_before += eq_total;
    out_before += take_total;
  }
}

template <int DK, int DV>
struct DsaSmem {
  static constexpr size_t kStage = (size_t)kRows * (DK + DV) * 2;
  static constexpr size_t kRing = (size_t)kWarps * 2 * kStage;
  static constexpr size_t kMerge = MergeBuf<DV>::kBytes + (size_t)kWarps * 16 * 3 * 4;
  static constexpr size_t kOut = (kRing > kMerge ? kRing : kMerge);   // sOut [16][DV] fp32 after it
  static constexpr size_t kTotal = kOut + (size_t)16 * DV * 4;
  static_assert(kTotal <= 232448, "dsa shared memory");
};

// One warp's online softmax over the chosen tokens rows[0, cnt) (each kept inside [0, t]), through
// its two-stage ring.  Lane l loads row l & 15 of a tile (the 16-byte chunks of parity l >> 4)
// and holds that row's token, -1 past cnt; the masks of the other rows come from it by shuffles.
// A tile's tokens are read two tiles ahead, so their loads overlap the math.
template <int DK, int DV>
__device__ void attend_tokens(const uint32_t (&qf)[DK / 16][4], State<DV>& st, Tile<DK, DV> ring0, Tile<DK, DV> ring1,
                              int cnt, const int32_t* rows, int t, const __nv_bfloat16* kb, const __nv_bfloat16* vb,
                              size_t kstride, size_t vstride, float scale_log2, int lane) {
  const int ntiles = (cnt + kRows - 1) / kRows;
  if (ntiles == 0) return;
  const int rr = lane & 15, half = lane >> 4, cq = lane & 3;
  auto token = [&](int it) {
    const int r = it * kRows + rr;
    return r < cnt ? min(max(rows[r], 0), t) : -1;
  };
  auto issue = [&](int it, int u) {
    if (it < ntiles) {
      const Tile<DK, DV> dst = (it & 1) ? ring1 : ring0;
      const __nv_bfloat16* sk = kb + (size_t)max(u, 0) * kstride;
      const __nv_bfloat16* sv = vb + (size_t)max(u, 0) * vstride;
#pragma unroll
      for (int c = 0; c < DK / 16; ++c)
        cp_async16(dst.k + SwzTile<DK>::offset(rr, 2 * c + half), sk + (2 * c + half) * 8, u >= 0);
#pragma unroll
      for (int c = 0; c < DV / 16; ++c)
        cp_async16(dst.v + SwzTile<DV>::offset(rr, 2 * c + half), sv + (2 * c + half) * 8, u >= 0);
    }
    cp_async_commit();
  };
  int u_cur = token(0), u_nxt = token(1);
  issue(0, u_cur);
  for (int it = 0; it < ntiles; ++it) {
    const int u_nn = token(it + 2);
    issue(it + 1, u_nxt);
    cp_async_wait<1>();
    __syncwarp();
    const Tile<DK, DV> cur = (it & 1) ? ring1 : ring0;
    float s[2][4];
    qk_tile<DK>(qf, cur.k, s, scale_log2, lane);
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (__shfl_sync(0xffffffffu, u_cur, j * 8 + 2 * cq + e) < 0) { s[j][e] = -INFINITY; s[j][2 + e] = -INFINITY; }
    float c0, c1;
    softmax_update<DV>(st, s, c0, c1);
    pv_tile<DV>(s, cur.v, st.o, lane);
    __syncwarp();
    u_cur = u_nxt;
    u_nxt = u_nn;
  }
  cp_async_wait<0>();
  __syncwarp();
}

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
dsa_attn_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ sel, __nv_bfloat16* __restrict__ out,
                int T, int Hq, int Hkv, int G, int K, float scale_log2) {
  using SM = DsaSmem<DK, DV>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  const bool rv0 = gl < G, rv1 = gl + 8 < G;
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
  const int n = min(t + 1, K);
  const int32_t* my = sel + ((size_t)b * T + t) * K;
  const int per = ((n + kRows - 1) / kRows + kWarps - 1) / kWarps * kRows;   // rows per warp, whole tiles
  const int r0 = min(n, warp * per), cnt = min(n, r0 + per) - r0;
  Tile<DK, DV> ring0{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)warp * 2 * SM::kStage), nullptr};
  ring0.v = ring0.k + kRows * DK;
  Tile<DK, DV> ring1{reinterpret_cast<__nv_bfloat16*>(smem + (size_t)warp * 2 * SM::kStage + SM::kStage), nullptr};
  ring1.v = ring1.k + kRows * DK;
  State<DV> st;
  st.init();
  attend_tokens<DK, DV>(qf, st, ring0, ring1, cnt, my + r0, t, k + ((size_t)b * T * Hkv + g) * DK,
                        v + ((size_t)b * T * Hkv + g) * DV, (size_t)Hkv * DK, (size_t)Hkv * DV, scale_log2, lane);
  float* sOut = reinterpret_cast<float*>(smem + SM::kOut);
  merge_states<DV>(st, smem, sOut, G, warp, lane);
  for (int e = tid; e < G * DV; e += kThreads) {
    const int r = e / DV, c = e % DV;
    out[(((size_t)b * T + t) * Hq + g * G + r) * DV + c] = __float2bfloat16_rn(sOut[e]);
  }
}

template <int DK, int DV>
cudaError_t launch_attn(const DsaArgs& a, cudaStream_t st) {
  using SM = DsaSmem<DK, DV>;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e =
        cudaFuncSetAttribute(dsa_attn_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kTotal);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  dsa_attn_kernel<DK, DV><<<dim3(a.T, a.Hkv, a.B), kThreads, SM::kTotal, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.sel, static_cast<__nv_bfloat16*>(a.out), a.T, a.Hq, a.Hkv, a.G,
      a.top_k, a.scale_log2);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_dsa_indexer(const DsaArgs& a, cudaStream_t st) {
  const int nt = (a.T + kIdxTile - 1) / kIdxTile;
  dim3 grid(nt, nt, a.B);
  const auto* qi = static_cast<const __nv_bfloat16*>(a.qi);
  const auto* ki = static_cast<const __nv_bfloat16*>(a.ki);
  const auto* wi = static_cast<const __nv_bfloat16*>(a.wi);
  if (a.di == 64) dsa_indexer_kernel<64><<<grid, kIdxThreads, 0, st>>>(qi, ki, wi, a.scores, a.T, a.hi);
  else if (a.di == 128) dsa_indexer_kernel<128><<<grid, kIdxThreads, 0, st>>>(qi, ki, wi, a.scores, a.T, a.hi);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const DsaArgs& a, cudaStream_t st) {
  dsa_topk_kernel<<<dim3(a.T, a.B), kTopkThreads, 0, st>>>(a.scores, a.sel, a.T, a.top_k);
  return cudaGetLastError();
}

cudaError_t launch_dsa_attn(const DsaArgs& a, cudaStream_t st) {
  if (a.dk == 192 && a.dv == 128) return launch_attn<192, 128>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch_attn<128, 128>(a, st);
  if (a.dk == 64 && a.dv == 64) return launch_attn<64, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
