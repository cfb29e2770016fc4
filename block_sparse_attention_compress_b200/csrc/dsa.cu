// DSA: token-wise sparse attention behind a lightning indexer (10100.com, "机器之心PRO · 会员通讯
// Week 45", "Which Attention is All You Need?", section "Linear v.s. Sparse", point 6: a light
// indexer scores every earlier token, the top-k tokens are kept, and full attention runs over them).
//
//   D1+D2 select  per 16 query tokens (one CTA, longest rows first), with no score matrix in
//                memory: the indexer score tiles score[t, s] = sum_j w[t, j] * ReLU(q_I[t, j] . k_I[s]),
//                s <= t (fp32, warp MMAs over 16 x 32 (query, key) tiles, one indexer head at a time)
//                are computed, and recomputed, as the selection needs them.  Four passes of an
//                8-bit radix select over order-preserving integer keys find each token's k-th
//                largest score (a 256-bin histogram per token in shared memory), a fifth pass
//                counts the keys above it and equal to it per quarter of the key range, and a
//                sixth writes the chosen tokens: those above, then the lowest-index ones equal to
//                it -- the list comes out ascending.  Every pass computes a tile with the same
//                instructions in the same order, so the scores agree bit for bit between passes.
//   D4 attention one CTA per (token, KV group): the 8 warps stream the chosen tokens' K/V rows
//                (gathered with cp.async) with an online softmax over the group's heads, then
//                merge their states.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "rows_attn.cuh"

namespace nsa {

namespace {
// Order-preserving map of a float to an unsigned integer (larger float, larger key).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelRows = 16;                    // query tokens per CTA (one MMA M)
constexpr int kSelWarps = 4;                    // each takes a contiguous quarter of the key tiles
constexpr int kSelThreads = 32 * kSelWarps;
constexpr int kSelKeys = 32;                    // keys per tile
constexpr int kBins = 256;
constexpr int kQResident = 32768;               // bytes of indexer queries kept in shared memory

template <int DI>
struct SelSmem {
  static constexpr size_t kKTile = (size_t)kSelKeys * DI * 2;
  static constexpr size_t kK = 0;                                          // [warp][2] key tiles
  static constexpr size_t kQ = kK + (size_t)kSelWarps * 2 * kKTile;        // [HI][16][DI] when resident
  static constexpr size_t kW = kQ + kQResident;                            // [HI][16] fp32 head weights
  static constexpr size_t kHist = kW + (size_t)64 * kSelRows * 4;          // [16][256]
  static constexpr size_t kState = kHist + (size_t)kSelRows * kBins * 4;   // prefix, mask, remaining [16]
  static constexpr size_t kCnt = kState + 3 * kSelRows * 4;                // [warp][16] (above, equal)
  static constexpr size_t kTotal = kCnt + (size_t)kSelWarps * kSelRows * 2 * 4;
  static_assert(kTotal <= 232448, "dsa select shared memory");
};

template <int DI>
__global__ void __launch_bounds__(kSelThreads)
dsa_select_kernel(const __nv_bfloat16* __restrict__ qi, const __nv_bfloat16* __restrict__ ki,
                  const __nv_bfloat16* __restrict__ wi, int32_t* __restrict__ sel, int T, int HI, int K) {
  using SM = SelSmem<DI>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int nq = (T + kSelRows - 1) / kSelRows;
  const int t0 = (nq - 1 - (int)blockIdx.x) * kSelRows, b = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + SM::kHist);
  uint32_t* s_prefix = reinterpret_cast<uint32_t*>(smem + SM::kState);
  uint32_t* s_mask = s_prefix + kSelRows;
  int* s_rem = reinterpret_cast<int*>(s_mask + kSelRows);
  int* s_cnt = reinterpret_cast<int*>(smem + SM::kCnt);
  float* sW = reinterpret_cast<float*>(smem + SM::kW);

  // tokens t0 .. t0+15; a token with t + 1 <= K takes every earlier token, the others select
  const int t_last = min(t0 + kSelRows - 1, T - 1);
  bool any_select = false;
  for (int r = 0; r < kSelRows; ++r) {
    const int t = t0 + r;
    if (t < T && t + 1 > K) any_select = true;
  }
  if (t0 + 1 <= K) {
    for (int e = tid; e < kSelRows * K; e += kSelThreads) {
      const int r = e / K, i = e % K, t = t0 + r;
      if (t < T && t + 1 <= K) sel[((size_t)b * T + t) * K + i] = i <= t ? i : -1;
    }
  }
  if (!any_select) return;

  const bool resident = (size_t)HI * kSelRows * DI * 2 <= (size_t)kQResident && HI <= 64;
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem + SM::kQ);
  if (resident) {
    for (int e = tid; e < HI * kSelRows * (DI / 8); e += kSelThreads) {
      const int h = e / (kSelRows * (DI / 8)), r = (e / (DI / 8)) % kSelRows, ch = e % (DI / 8);
      const bool ok = t0 + r < T;
      cp_async16(sQ + h * kSelRows * DI + SwzTile<DI>::offset(r, ch),
                 qi + (((size_t)b * T + (ok ? t0 + r : 0)) * HI + h) * DI + ch * 8, ok);
    }
    cp_async_commit();
  }
  for (int e = tid; e < HI * kSelRows; e += kSelThreads) {
    const int h = e / kSelRows, r = e % kSelRows;
    sW[e] = t0 + r < T ? __bfloat162float(wi[((size_t)b * T + t0 + r) * HI + h]) : 0.f;
  }
  if (tid < kSelRows) {
    s_prefix[tid] = 0u;
    s_mask[tid] = 0u;
    s_rem[tid] = K;
  }
  cp_async_wait<0>();
  __syncthreads();

  // this thread's two tokens (rows gl and gl + 8 of the MMA tile) and whether they select
  const int ta = t0 + gl, tb = ta + 8;
  const bool sa = ta < T && ta + 1 > K, sb = tb < T && tb + 1 > K;
  // this warp's key tiles: a contiguous quarter of 0 .. ntk-1
  const int ntk = t_last / kSelKeys + 1;
  const int kt_begin = warp * ntk / kSelWarps, kt_end = (warp + 1) * ntk / kSelWarps;
  __nv_bfloat16* sK0 = reinterpret_cast<__nv_bfloat16*>(smem + SM::kK + (size_t)warp * 2 * SM::kKTile);
  __nv_bfloat16* sK1 = sK0 + kSelKeys * DI;

  auto load_keys = [&](int kt, __nv_bfloat16* dst) {
    if (kt < kt_end) {
      const int s0 = kt * kSelKeys;
#pragma unroll
      for (int e = lane; e < kSelKeys * (DI / 8); e += 32) {
        const int r = e / (DI / 8), ch = e % (DI / 8);
        const bool ok = s0 + r < T;
        cp_async16(dst + SwzTile<DI>::offset(r, ch), ki + ((size_t)b * T + (ok ? s0 + r : 0)) * DI + ch * 8, ok);
      }
    }
    cp_async_commit();
  };
  // The score tile of key tile kt (keys kt*32 ..): acc[j][e] is token ta's score of key
  // kt*32 + 8j + 2cq + e, acc[j][2 + e] token tb's.  The same instructions in every pass.
  auto tile_scores = [&](const __nv_bfloat16* sKt, float (&acc)[kSelKeys / 8][4]) {
#pragma unroll
    for (int j = 0; j < kSelKeys / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    for (int h = 0; h < HI; ++h) {
      uint32_t qf[DI / 16][4];
      if (resident) {
#pragma unroll
        for (int ks = 0; ks < DI / 16; ++ks)
          ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3],
                  smem_u32(sQ + h * kSelRows * DI + SwzTile<DI>::offset(lane & 15, 2 * ks + (lane >> 4))));
      } else {
        const __nv_bfloat16* q0 = qi + (((size_t)b * T + min(ta, T - 1)) * HI + h) * DI;
        const __nv_bfloat16* q1 = qi + (((size_t)b * T + min(tb, T - 1)) * HI + h) * DI;
#pragma unroll
        for (int ks = 0; ks < DI / 16; ++ks) {
          qf[ks][0] = ld_u32(q0 + ks * 16 + 2 * cq);
          qf[ks][1] = ld_u32(q1 + ks * 16 + 2 * cq);
          qf[ks][2] = ld_u32(q0 + ks * 16 + 8 + 2 * cq);
          qf[ks][3] = ld_u32(q1 + ks * 16 + 8 + 2 * cq);
        }
      }
      const float wa = sW[h * kSelRows + gl], wb = sW[h * kSelRows + gl + 8];
#pragma unroll
      for (int kt = 0; kt < kSelKeys / 16; ++kt) {
        float s[2][4];
        qk_tile<DI>(qf, sKt + kt * 16 * DI, s, 1.f, lane);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          acc[2 * kt + x][0] += wa * fmaxf(s[x][0], 0.f);
          acc[2 * kt + x][1] += wa * fmaxf(s[x][1], 0.f);
          acc[2 * kt + x][2] += wb * fmaxf(s[x][2], 0.f);
          acc[2 * kt + x][3] += wb * fmaxf(s[x][3], 0.f);
        }
      }
    }
  };
  // one sweep of this warp's key tiles; visit(kt, acc) sees every tile in ascending order
  auto sweep = [&](auto&& visit) {
    load_keys(kt_begin, sK0);
    for (int kt = kt_begin; kt < kt_end; ++kt) {
      const int i = kt - kt_begin;
      load_keys(kt + 1, (i & 1) ? sK0 : sK1);
      cp_async_wait<1>();
      __syncwarp();
      float acc[kSelKeys / 8][4];
      tile_scores((i & 1) ? sK1 : sK0, acc);
      visit(kt, acc);
      __syncwarp();   // the buffer is refilled by the next iteration's load
    }
    cp_async_wait<0>();
  };

  // radix passes: the digit of the remaining-th largest key among those matching the prefix
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int e = tid; e < kSelRows * kBins; e += kSelThreads) hist[e] = 0u;
    __syncthreads();
    const uint32_t pa = s_prefix[gl], ma = s_mask[gl], pb = s_prefix[gl + 8], mb = s_mask[gl + 8];
    sweep([&](int kt, const float (&acc)[kSelKeys / 8][4]) {
#pragma unroll
      for (int j = 0; j < kSelKeys / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int s = kt * kSelKeys + j * 8 + 2 * cq + e;
          const uint32_t ua = ordered_key(acc[j][e]), ub = ordered_key(acc[j][2 + e]);
          if (sa && s <= ta && (ua & ma) == pa) atomicAdd(&hist[gl * kBins + ((ua >> shift) & 255u)], 1u);
          if (sb && s <= tb && (ub & mb) == pb) atomicAdd(&hist[(gl + 8) * kBins + ((ub >> shift) & 255u)], 1u);
        }
    });
    __syncthreads();
    if (tid < kSelRows) {
      const int t = t0 + tid;
      if (t < T && t + 1 > K) {
        const int remaining = s_rem[tid];
        int cum = 0, d = 255;
        for (; d > 0; --d) {
          const int c = (int)hist[tid * kBins + d];
          if (cum + c >= remaining) break;
          cum += c;
        }
        s_prefix[tid] |= (uint32_t)d << shift;
        s_mask[tid] |= 255u << shift;
        s_rem[tid] = remaining - cum;
      }
    }
    __syncthreads();
  }

  // count pass: per warp and token, the keys above the threshold and equal to it
  const uint32_t thr_a = s_prefix[gl], thr_b = s_prefix[gl + 8];
  const int rem_a = s_rem[gl], rem_b = s_rem[gl + 8];
  {
    int ga = 0, ea = 0, gb = 0, eb = 0;
    sweep([&](int kt, const float (&acc)[kSelKeys / 8][4]) {
#pragma unroll
      for (int j = 0; j < kSelKeys / 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int s = kt * kSelKeys + j * 8 + 2 * cq + e;
          const uint32_t ua = ordered_key(acc[j][e]), ub = ordered_key(acc[j][2 + e]);
          const bool va = sa && s <= ta, vb = sb && s <= tb;
          ga += va && ua > thr_a;
          ea += va && ua == thr_a;
          gb += vb && ub > thr_b;
          eb += vb && ub == thr_b;
        }
    });
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      ga += __shfl_xor_sync(0xffffffffu, ga, o);
      ea += __shfl_xor_sync(0xffffffffu, ea, o);
      gb += __shfl_xor_sync(0xffffffffu, gb, o);
      eb += __shfl_xor_sync(0xffffffffu, eb, o);
    }
    if (cq == 0) {
      s_cnt[(warp * kSelRows + gl) * 2] = ga;
      s_cnt[(warp * kSelRows + gl) * 2 + 1] = ea;
      s_cnt[(warp * kSelRows + gl + 8) * 2] = gb;
      s_cnt[(warp * kSelRows + gl + 8) * 2 + 1] = eb;
    }
  }
  __syncthreads();

  // emit pass: this warp's first output slot and equal-key rank for each of its two tokens
  int out_a = 0, eqs_a = 0, out_b = 0, eqs_b = 0;
  for (int w = 0; w < warp; ++w) {
    const int g_a = s_cnt[(w * kSelRows + gl) * 2], e_a = s_cnt[(w * kSelRows + gl) * 2 + 1];
    const int g_b = s_cnt[(w * kSelRows + gl + 8) * 2], e_b = s_cnt[(w * kSelRows + gl + 8) * 2 + 1];
    out_a += g_a + min(e_a, max(0, rem_a - eqs_a));
    out_b += g_b + min(e_b, max(0, rem_b - eqs_b));
    eqs_a += e_a;
    eqs_b += e_b;
  }
  int32_t* dst_a = sel + ((size_t)b * T + min(ta, T - 1)) * K;
  int32_t* dst_b = sel + ((size_t)b * T + min(tb, T - 1)) * K;
  // the quad's exclusive prefix of x in key order (lane cq holds keys 2cq, 2cq+1 of a chunk)
  auto quad_scan = [&](int x, int& total) {
    int inc = x;
    const int p1 = __shfl_up_sync(0xffffffffu, inc, 1, 4);
    if (cq >= 1) inc += p1;
    const int p2 = __shfl_up_sync(0xffffffffu, inc, 2, 4);
    if (cq >= 2) inc += p2;
    total = __shfl_sync(0xffffffffu, inc, 3, 4);
    return inc - x;
  };
  auto emit = [&](int s0, float v0, float v1, bool sel_row, int t, uint32_t thr, int rem, int& out, int& eqs,
                  int32_t* dst) {
    const uint32_t u0 = ordered_key(v0), u1 = ordered_key(v1);
    const bool ok0 = sel_row && s0 <= t, ok1 = sel_row && s0 + 1 <= t;
    const bool e0 = ok0 && u0 == thr, e1 = ok1 && u1 == thr;
    int eq_total;
    const int r0 = eqs + quad_scan((int)e0 + (int)e1, eq_total);
    const bool k0 = (ok0 && u0 > thr) || (e0 && r0 < rem);
    const bool k1 = (ok1 && u1 > thr) || (e1 && r0 + (int)e0 < rem);
    int take_total;
    const int p0 = out + quad_scan((int)k0 + (int)k1, take_total);
    if (k0 && p0 < K) dst[p0] = s0;
    if (k1 && p0 + (int)k0 < K) dst[p0 + (int)k0] = s0 + 1;
    out += take_total;
    eqs += eq_total;
  };
  sweep([&](int kt, const float (&acc)[kSelKeys / 8][4]) {
#pragma unroll
    for (int j = 0; j < kSelKeys / 8; ++j) {
      const int s0 = kt * kSelKeys + j * 8 + 2 * cq;
      emit(s0, acc[j][0], acc[j][1], sa, ta, thr_a, rem_a, out_a, eqs_a, dst_a);
      emit(s0, acc[j][2], acc[j][3], sb, tb, thr_b, rem_b, out_b, eqs_b, dst_b);
    }
  });
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
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e =
        cudaFuncSetAttribute(dsa_attn_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kTotal);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dsa_attn_kernel<DK, DV><<<dim3(a.T, a.Hkv, a.B), kThreads, SM::kTotal, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.sel, static_cast<__nv_bfloat16*>(a.out), a.T, a.Hq, a.Hkv, a.G,
      a.top_k, a.scale_log2);
  return cudaGetLastError();
}

template <int DI>
cudaError_t launch_select(const DsaArgs& a, cudaStream_t st) {
  using SM = SelSmem<DI>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e =
        cudaFuncSetAttribute(dsa_select_kernel<DI>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kTotal);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  const int nq = (a.T + kSelRows - 1) / kSelRows;
  dsa_select_kernel<DI><<<dim3(nq, a.B), kSelThreads, SM::kTotal, st>>>(
      static_cast<const __nv_bfloat16*>(a.qi), static_cast<const __nv_bfloat16*>(a.ki),
      static_cast<const __nv_bfloat16*>(a.wi), a.sel, a.T, a.hi, a.top_k);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_dsa_select(const DsaArgs& a, cudaStream_t st) {
  if (a.hi < 1 || a.hi > 64) return cudaErrorInvalidValue;
  if (a.di == 64) return launch_select<64>(a, st);
  if (a.di == 128) return launch_select<128>(a, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dsa_attn(const DsaArgs& a, cudaStream_t st) {
  if (a.dk == 192 && a.dv == 128) return launch_attn<192, 128>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch_attn<128, 128>(a, st);
  if (a.dk == 64 && a.dv == 64) return launch_attn<64, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
