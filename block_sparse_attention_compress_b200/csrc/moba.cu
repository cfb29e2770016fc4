// MoBA mode ("一文比较 Kimi 和 Deepseek 的两篇稀疏注意力机制论文", "Kimi 的论文核心点": every
// query attends to its own block with a causal staircase and to the past blocks whose
// mean-pooled key scores highest against it; "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文"
// §16-§17: mean pooling, no parameters, every head chooses for itself, 512-token blocks,
// top 3; the queries that chose one KV block are gathered so the block is read once).
//
// Five launches on the caller's stream:
//   M1 block means      kbar[b, j, h, :] = mean of the keys of block j, accumulated in fp32 and
//                       stored as two bf16 halves (hi = bf16(mean), lo = bf16(mean - hi)) so
//                       that the tensor-core dot product keeps about 16 mantissa bits;
//   M2 select           per 64-token tile and head: score_j = q . hi_j + q . lo_j for the past
//                       blocks (tiles of 64 blocks double buffered by cp.async), running top-k
//                       per row, idx = [past ascending.., own];
//                       counts the queries that chose each (b, h, j);
//   M3 lists            one CTA: exclusive scans of the counts (list offsets, 64-query chunks);
//                       then every choice is scattered into its (b, h, j) list as t*8 + slot;
//   M4 past attention   persistent CTAs walk the 64-query chunks: gather the chunk's queries,
//                       stream block j's 512 keys (no mask: every key is in the past), write
//                       per-query normalised o (bf16) and its log-sum-exp per slot;
//   M5 own + merge      per 64-token tile and head: causal attention inside the own block,
//                       then the partials of the past slots are merged in; out in bf16.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
constexpr int D = 128;            // head dim of this mode
constexpr int kQ = 64;            // queries per tile / chunk (4 warps x 16 rows)
constexpr int kThreads = 128;
constexpr int kKT = 64;           // keys per shared-memory tile
constexpr int kMaxK = 7;          // past blocks per query

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

__device__ __forceinline__ void load_q_frag(uint32_t (&qf)[D / 16][4], const __nv_bfloat16* q0, const __nv_bfloat16* q1,
                                            bool r0, bool r1, int cq) {
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
    qf[ks][0] = r0 ? ld_u32(q0 + ks * 16 + 2 * cq) : 0u;
    qf[ks][1] = r1 ? ld_u32(q1 + ks * 16 + 2 * cq) : 0u;
    qf[ks][2] = r0 ? ld_u32(q0 + ks * 16 + 8 + 2 * cq) : 0u;
    qf[ks][3] = r1 ? ld_u32(q1 + ks * 16 + 8 + 2 * cq) : 0u;
  }
}

// S (16 x 64) += Q K^T from a swizzled [64][D] bf16 tile.
__device__ __forceinline__ void qk64(const uint32_t (&qf)[D / 16][4], const __nv_bfloat16* k, float (&s)[8][4],
                                     int lane) {
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      uint32_t b0, b1, b2, b3;
      const int row = np * 16 + (lane & 7) + ((lane >> 4) << 3);
      const int ch = 2 * ks + ((lane >> 3) & 1);
      ldsm_x4(b0, b1, b2, b3, smem_u32(k + SwzTile<D>::offset(row, ch)));
      mma16816(s[2 * np], qf[ks], b0, b1);
      mma16816(s[2 * np + 1], qf[ks], b2, b3);
    }
}

// O (16 x D) += P V with P (16 x 64) in C-fragment layout.
__device__ __forceinline__ void pv64(const float (&p)[8][4], const __nv_bfloat16* v, float (&o)[D / 8][4], int lane) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int np = 0; np < D / 16; ++np) {
      uint32_t b0, b1, b2, b3;
      const int row = kk * 16 + (lane & 15);
      const int ch = 2 * np + (lane >> 4);
      ldsm_x4_t(b0, b1, b2, b3, smem_u32(v + SwzTile<D>::offset(row, ch)));
      mma16816(o[2 * np], a, b0, b1);
      mma16816(o[2 * np + 1], a, b2, b3);
    }
  }
}

// One online-softmax step for rows (gl, gl+8) with masked logits (-inf) already in log2 units.
__device__ __forceinline__ void online(float (&s)[8][4], float& m0, float& m1, float& l0, float& l1,
                                       float (&o)[D / 8][4]) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
    mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
  }
  mx0 = warp_max4(mx0);
  mx1 = warp_max4(mx1);
  const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
  const float b0 = n0 == -INFINITY ? 0.f : n0, b1 = n1 == -INFINITY ? 0.f : n1;
  const float c0 = exp2f(m0 - b0), c1 = exp2f(m1 - b1);
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    s[j][0] = exp2f(s[j][0] - b0); s[j][1] = exp2f(s[j][1] - b0);
    s[j][2] = exp2f(s[j][2] - b1); s[j][3] = exp2f(s[j][3] - b1);
    sum0 += s[j][0] + s[j][1];
    sum1 += s[j][2] + s[j][3];
  }
  l0 = l0 * c0 + warp_sum4(sum0);
  l1 = l1 * c1 + warp_sum4(sum1);
  m0 = n0;
  m1 = n1;
#pragma unroll
  for (int j = 0; j < D / 8; ++j) {
    o[j][0] *= c0; o[j][1] *= c0; o[j][2] *= c1; o[j][3] *= c1;
  }
}

// ------------------------------------------------------------------ M1
// kbar: [2][B][nblk][H][D] bf16, the hi halves then the lo halves.
__global__ void __launch_bounds__(D) moba_mean_kernel(const __nv_bfloat16* __restrict__ k,
                                                      __nv_bfloat16* __restrict__ kbar, int B, int T, int H, int bsz,
                                                      int nblk) {
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, c = threadIdx.x;
  const int u0 = j * bsz, u1 = min(T, u0 + bsz);
  float acc = 0.f;
  for (int u = u0; u < u1; ++u) acc += __bfloat162float(k[(((size_t)b * T + u) * H + h) * D + c]);
  const float mean = acc / (float)(u1 - u0);
  const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
  const size_t o = (((size_t)b * nblk + j) * H + h) * D + c;
  kbar[o] = hi;
  kbar[(size_t)B * nblk * H * D + o] = __float2bfloat16_rn(mean - __bfloat162float(hi));
}

// ------------------------------------------------------------------ M2
// Keeps the KK best (score desc, index asc) of the values offered to it, sorted best-first,
// entirely in registers: every slot index is a compile-time constant.  The KK-th best is kept
// apart as (tv, tj), so most offers cost one comparison.
template <int KK>
struct TopK {
  static constexpr int N = KK > 0 ? KK : 1;
  float v[N];
  int j[N];
  float tv;
  int tj;
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < N; ++i) { v[i] = -FLT_MAX; j[i] = 0x7fffffff; }
    tv = -FLT_MAX;
    tj = 0x7fffffff;
  }
  __device__ __forceinline__ static bool better(float a, int ja, float b, int jb) {
    return a > b || (a == b && ja < jb);
  }
  __device__ __forceinline__ void offer(float val, int idx) {
    if (!better(val, idx, tv, tj)) return;
    float cv = val;
    int cj = idx;
#pragma unroll
    for (int i = 0; i < N; ++i) {   // insertion by swapping down the sorted slots
      if (better(cv, cj, v[i], j[i])) {
        const float xv = v[i];
        const int xj = j[i];
        v[i] = cv;
        j[i] = cj;
        cv = xv;
        cj = xj;
      }
    }
    tv = v[N - 1];
    tj = j[N - 1];
  }
  __device__ __forceinline__ void pop() {   // drop the best slot
#pragma unroll
    for (int i = 0; i + 1 < N; ++i) { v[i] = v[i + 1]; j[i] = j[i + 1]; }
    v[N - 1] = -FLT_MAX;
    j[N - 1] = 0x7fffffff;
  }
};

// One instantiation per top_k (0 .. kMaxK), so that the per-thread candidate lists and the
// merged selections live in registers.  A CTA takes 256 queries of one head (16 warps of 16,
// each warp with its own block J), so that each tile of block means it streams through shared
// memory serves 256 queries, and three CTAs (48 warps) share an SM.
constexpr int kSelQ = 256, kSelThreads = 512;
template <int KK>
__global__ void __launch_bounds__(kSelThreads) moba_select_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kbar, int32_t* __restrict__ idx,
    int32_t* __restrict__ counts, int B, int T, int H, int bsz, int nblk) {
  constexpr int N = TopK<KK>::N;
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sHi = reinterpret_cast<__nv_bfloat16*>(smem);          // [2][kKT][D]
  __nv_bfloat16* sLo = sHi + 2 * kKT * D;                               // [2][kKT][D]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  const int t0 = blockIdx.x * kSelQ, h = blockIdx.y, b = blockIdx.z;
  const int J = (t0 + warp * 16) / bsz;        // this warp's own block (bsz % 64 == 0: one per 16 rows)
  const int Jc = min(t0 + kSelQ - 1, T - 1) / bsz;   // the CTA's largest: the blocks it streams
  const int ta = t0 + warp * 16 + gl, tb = ta + 8;
  const size_t lo_off = (size_t)B * nblk * H * D;
  const bool choose = KK > 0 && J > KK;        // else every past block is taken
  TopK<KK> k0, k1;
  k0.init();
  k1.init();
  if (KK > 0 && Jc > KK) {                     // the same decision for every warp of the CTA
    uint32_t qf[D / 16][4];
    load_q_frag(qf, q + (((size_t)b * T + min(ta, T - 1)) * H + h) * D,
                q + (((size_t)b * T + min(tb, T - 1)) * H + h) * D, ta < T, tb < T, cq);
    auto load = [&](int j0, int buf) {   // blocks j0 .. j0+63 (zeros past Jc)
      for (int e = tid; e < kKT * (D / 8); e += kSelThreads) {
        const int r = e / (D / 8), ch = e % (D / 8);
        const int j = j0 + r;
        const size_t src = (((size_t)b * nblk + min(j, Jc - 1)) * H + h) * D + ch * 8;
        cp_async16(sHi + buf * kKT * D + SwzTile<D>::offset(r, ch), kbar + src, j < Jc);
        cp_async16(sLo + buf * kKT * D + SwzTile<D>::offset(r, ch), kbar + lo_off + src, j < Jc);
      }
    };
    load(0, 0);
    cp_async_commit();
    for (int j0 = 0, it = 0; j0 < Jc; j0 += kKT, ++it) {
      if (j0 + kKT < Jc) load(j0 + kKT, (it + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      float s[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      qk64(qf, sHi + (it & 1) * kKT * D, s, lane);
      qk64(qf, sLo + (it & 1) * kKT * D, s, lane);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = j0 + nt * 8 + 2 * cq + e;
          if (choose && j < J) {
            k0.offer(s[nt][e], j);
            k1.offer(s[nt][2 + e], j);
          }
        }
      __syncthreads();   // this buffer is refilled two tiles later
    }
    cp_async_wait<0>();
  }
  // merge the quad's four lists: KK rounds of a quad-wide argmax over the lists' heads
  int sel0[N], sel1[N];
#pragma unroll
  for (int i = 0; i < N; ++i) sel0[i] = sel1[i] = i;
  if (choose) {
#pragma unroll
    for (int r = 0; r < N; ++r) {
      float bv0 = k0.v[0], bv1 = k1.v[0];
      int bj0 = k0.j[0], bj1 = k1.j[0];
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        const float ov0 = __shfl_xor_sync(0xffffffffu, bv0, off), ov1 = __shfl_xor_sync(0xffffffffu, bv1, off);
        const int oj0 = __shfl_xor_sync(0xffffffffu, bj0, off), oj1 = __shfl_xor_sync(0xffffffffu, bj1, off);
        if (TopK<KK>::better(ov0, oj0, bv0, bj0)) { bv0 = ov0; bj0 = oj0; }
        if (TopK<KK>::better(ov1, oj1, bv1, bj1)) { bv1 = ov1; bj1 = oj1; }
      }
      sel0[r] = bj0;
      sel1[r] = bj1;
      if (k0.j[0] == bj0) k0.pop();   // indices are unique across the quad's lanes
      if (k1.j[0] == bj1) k1.pop();
    }
    // ascending block order: odd-even transposition sort over the N slots
#pragma unroll
    for (int pass = 0; pass < N; ++pass)
#pragma unroll
      for (int i = pass & 1; i + 1 < N; i += 2) {
        if (sel0[i] > sel0[i + 1]) { const int x = sel0[i]; sel0[i] = sel0[i + 1]; sel0[i + 1] = x; }
        if (sel1[i] > sel1[i + 1]) { const int x = sel1[i]; sel1[i] = sel1[i + 1]; sel1[i + 1] = x; }
      }
  }
  // the picks are counted per block in shared memory (the tile buffers are free now, and the
  // CTA's blocks 0 .. Jc fit them: at most 16384 of 64 KB), then added to the global counts
  // once per block: the global adds of many queries on the same popular blocks were the
  // kernel's largest single cost
  int32_t* hist = reinterpret_cast<int32_t*>(smem);
  __syncthreads();
  for (int j = tid; j <= Jc; j += kSelThreads) hist[j] = 0;
  __syncthreads();
  if (cq == 0) {
    const int kk = min(KK, J);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int t = half ? tb : ta;
      if (t >= T) continue;
      int32_t* dst = idx + (((size_t)b * H + h) * T + t) * (KK + 1);
#pragma unroll
      for (int i = 0; i < KK; ++i) {
        if (i < kk) {
          const int sj = half ? sel1[i] : sel0[i];
          dst[i] = sj;
          atomicAdd(hist + sj, 1);
        } else {
          dst[i + 1] = -1;
        }
      }
      dst[kk] = J;
    }
  }
  __syncthreads();
  int32_t* cnt = counts + ((size_t)b * H + h) * nblk;
  for (int j = tid; j <= Jc; j += kSelThreads)
    if (hist[j] != 0) atomicAdd(cnt + j, hist[j]);
}

// ------------------------------------------------------------------ M3
// Exclusive scans over all (b, h, j): list offsets and 64-query chunk starts (one CTA).
__global__ void __launch_bounds__(1024) moba_scan_kernel(const int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets, int32_t* __restrict__ chunks,
                                                         int32_t* __restrict__ fill, int32_t* __restrict__ chunk_list,
                                                         int E, int cq) {
  __shared__ int32_t s0[1024], s1[1024];
  __shared__ int32_t carry0, carry1;
  if (threadIdx.x == 0) { carry0 = 0; carry1 = 0; }
  __syncthreads();
  for (int base = 0; base < E; base += 1024) {
    const int e = base + threadIdx.x;
    const int c = e < E ? counts[e] : 0;
    s0[threadIdx.x] = c;
    s1[threadIdx.x] = (c + cq - 1) / cq;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {   // Hillis-Steele inclusive scan
      const int a0 = threadIdx.x >= off ? s0[threadIdx.x - off] : 0;
      const int a1 = threadIdx.x >= off ? s1[threadIdx.x - off] : 0;
      __syncthreads();
      s0[threadIdx.x] += a0;
      s1[threadIdx.x] += a1;
      __syncthreads();
    }
    if (e < E) {
      offsets[e] = carry0 + s0[threadIdx.x] - c;
      chunks[e] = carry1 + s1[threadIdx.x] - (c + cq - 1) / cq;
      fill[e] = 0;
    }
    __syncthreads();
    if (threadIdx.x == 1023) { carry0 += s0[1023]; carry1 += s1[1023]; }
    __syncthreads();
  }
  if (threadIdx.x == 0) { offsets[E] = carry0; chunks[E] = carry1; }
  __syncthreads();
  // the list of every chunk, so that a chunk finds its list with one load
  for (int e = threadIdx.x; e < E; e += 1024)
    for (int c = chunks[e]; c < chunks[e + 1]; ++c) chunk_list[c] = e;
}

// One CTA per 256 consecutive queries of one (b, h): the picks are counted per block in shared
// memory, each block's range in its list is reserved with one global add per CTA, and every
// pick then goes to its slot (the order inside a list is free: each query's result depends only
// on its own row).
constexpr int kScatterQ = 256;
__global__ void __launch_bounds__(kScatterQ)
moba_scatter_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ offsets, int32_t* __restrict__ fill,
                    int32_t* __restrict__ list, int T, int H, int nblk, int top_k, int bsz) {
  extern __shared__ int32_t s_slot[];   // [block]: the CTA's count, then the first slot of its range
  const int bh = blockIdx.y, t0 = blockIdx.x * kScatterQ, t = t0 + threadIdx.x;
  const int jc = min(t0 + kScatterQ - 1, T - 1) / bsz;   // the picks are blocks below the own block: < jc
  for (int j = threadIdx.x; j < jc; j += kScatterQ) s_slot[j] = 0;
  __syncthreads();
  int pick[8], local[8];
  int n = 0;
  if (t < T) {
    const int32_t* row = idx + ((size_t)bh * T + t) * (top_k + 1);
    const int own = t / bsz;
    for (int s = 0; s < top_k; ++s) {
      const int j = row[s];
      if (j < 0 || j >= own) break;
      pick[n] = j;
      local[n] = atomicAdd(&s_slot[j], 1);
      ++n;
    }
  }
  __syncthreads();
  for (int j = threadIdx.x; j < jc; j += kScatterQ) {
    const int c = s_slot[j];
    const size_t e = (size_t)bh * nblk + j;
    s_slot[j] = c > 0 ? offsets[e] + atomicAdd(&fill[e], c) : 0;
  }
  __syncthreads();
  for (int s = 0; s < n; ++s) list[s_slot[pick[s]] + local[s]] = t * 8 + s;
}

// ------------------------------------------------------------------ M4
__global__ void __launch_bounds__(kThreads) moba_past_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets, const int32_t* __restrict__ chunks,
    const int32_t* __restrict__ list, __nv_bfloat16* __restrict__ part_o, float* __restrict__ part_lse, int T, int H,
    int nblk, int bsz, int top_k, int E, float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);             // [2][64][D]
  __nv_bfloat16* sV = sK + 2 * kKT * D;                                    // [2][64][D]
  __shared__ int32_t sList[kQ];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  const int total = chunks[E];
  for (int c = blockIdx.x; c < total; c += gridDim.x) {
    // (b, h, j) whose chunk range holds c: last e with chunks[e] <= c (binary search)
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (chunks[mid] <= c) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int bh = e / nblk, j = e % nblk, b = bh / H, h = bh % H;
    const int first = (c - chunks[e]) * kQ;
    const int nq = min(kQ, counts[e] - first);
    __syncthreads();
    if (tid < kQ) sList[tid] = tid < nq ? list[offsets[e] + first + tid] : -1;
    __syncthreads();
    const int ea = sList[warp * 16 + gl], eb = sList[warp * 16 + gl + 8];
    const int ta = ea >> 3, tb = eb >> 3;
    uint32_t qf[D / 16][4];
    load_q_frag(qf, q + (((size_t)b * T + (ea >= 0 ? ta : 0)) * H + h) * D,
                q + (((size_t)b * T + (eb >= 0 ? tb : 0)) * H + h) * D, ea >= 0, eb >= 0, cq);
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    const int u0 = j * bsz;
    const int ntiles = bsz / kKT;
    auto load = [&](int it, int buf) {
      for (int x = tid; x < kKT * (D / 8); x += kThreads) {
        const int r = x / (D / 8), ch = x % (D / 8);
        const size_t row = ((size_t)b * T + u0 + it * kKT + r) * H + h;
        cp_async16(sK + buf * kKT * D + SwzTile<D>::offset(r, ch), k + row * D + ch * 8, true);
        cp_async16(sV + buf * kKT * D + SwzTile<D>::offset(r, ch), v + row * D + ch * 8, true);
      }
    };
    load(0, 0);
    cp_async_commit();
    for (int it = 0; it < ntiles; ++it) {
      if (it + 1 < ntiles) load(it + 1, (it + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      float s[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
      qk64(qf, sK + (it & 1) * kKT * D, s, lane);
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int x = 0; x < 4; ++x) s[i][x] *= scale_log2;
      online(s, m0, m1, l0, l1, o);
      pv64(s, sV + (it & 1) * kKT * D, o, lane);
      __syncthreads();
    }
    cp_async_wait<0>();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int ent = half ? eb : ea;
      if (ent < 0) continue;
      const int t = ent >> 3, slot = ent & 7;
      const float l = half ? l1 : l0, m = half ? m1 : m0;
      const float inv = 1.f / l;
      const size_t base = (((size_t)b * T + t) * H + h) * top_k + slot;
      __nv_bfloat16* dst = part_o + base * D;
#pragma unroll
      for (int i = 0; i < D / 8; ++i)
        *reinterpret_cast<uint32_t*>(dst + i * 8 + 2 * cq) =
            pack_bf16(o[i][2 * half] * inv, o[i][2 * half + 1] * inv);
      if (cq == 0) part_lse[base] = m + __log2f(l);
    }
  }
}

// ------------------------------------------------------------------ M5
__global__ void __launch_bounds__(kThreads) moba_own_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ part_o, const float* __restrict__ part_lse,
    __nv_bfloat16* __restrict__ out, int T, int H, int bsz, int top_k, float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = sK + 2 * kKT * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gl = lane >> 2, cq = lane & 3;
  const int t0 = blockIdx.x * kQ, h = blockIdx.y, b = blockIdx.z;
  const int J = t0 / bsz, u0 = J * bsz;
  const int ta = t0 + warp * 16 + gl, tb = ta + 8;
  const int t_last = min(T - 1, t0 + kQ - 1);
  uint32_t qf[D / 16][4];
  load_q_frag(qf, q + (((size_t)b * T + min(ta, T - 1)) * H + h) * D, q + (((size_t)b * T + min(tb, T - 1)) * H + h) * D,
              ta < T, tb < T, cq);
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int ntiles = (t_last - u0) / kKT + 1;
  auto load = [&](int it, int buf) {
    for (int x = tid; x < kKT * (D / 8); x += kThreads) {
      const int r = x / (D / 8), ch = x % (D / 8);
      const int u = u0 + it * kKT + r;
      const bool ok = u <= t_last;
      const size_t row = ((size_t)b * T + (ok ? u : t_last)) * H + h;
      cp_async16(sK + buf * kKT * D + SwzTile<D>::offset(r, ch), k + row * D + ch * 8, ok);
      cp_async16(sV + buf * kKT * D + SwzTile<D>::offset(r, ch), v + row * D + ch * 8, ok);
    }
  };
  load(0, 0);
  cp_async_commit();
  for (int it = 0; it < ntiles; ++it) {
    if (it + 1 < ntiles) load(it + 1, (it + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
    qk64(qf, sK + (it & 1) * kKT * D, s, lane);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int u = u0 + it * kKT + nt * 8 + 2 * cq + e;
        s[nt][e] = u <= ta ? s[nt][e] * scale_log2 : -INFINITY;
        s[nt][2 + e] = u <= tb ? s[nt][2 + e] * scale_log2 : -INFINITY;
      }
    online(s, m0, m1, l0, l1, o);
    pv64(s, sV + (it & 1) * kKT * D, o, lane);
    __syncthreads();
  }
  cp_async_wait<0>();
  // merge the past slots (each a normalised o with its log-sum-exp) into the own-block state
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int t = half ? tb : ta;
    if (t >= T) continue;
    const int32_t* row = idx + (((size_t)b * H + h) * T + t) * (top_k + 1);
    float m = half ? m1 : m0, l = half ? l1 : l0;   // own block: m finite (t itself is always visible)
    float lse[kMaxK];
    int np = 0;
    for (int s = 0; s < top_k; ++s) {
      const int j = row[s];
      if (j < 0 || j >= J) break;
      lse[np++] = part_lse[(((size_t)b * T + t) * H + h) * top_k + s];
    }
    float M = m + __log2f(l);
    for (int s = 0; s < np; ++s) M = fmaxf(M, lse[s]);
    const float w_own = exp2f(m - M);        // multiplies the unnormalised own o (sum l)
    float wsum = l * w_own;
    float ws[kMaxK];
    for (int s = 0; s < np; ++s) { ws[s] = exp2f(lse[s] - M); wsum += ws[s]; }
    const float inv = 1.f / wsum;
    __nv_bfloat16* dst = out + (((size_t)b * T + t) * H + h) * D;
    const __nv_bfloat16* po = part_o + (((size_t)b * T + t) * H + h) * top_k * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      float x0 = o[i][2 * half] * w_own, x1 = o[i][2 * half + 1] * w_own;
      for (int s = 0; s < np; ++s) {
        const __nv_bfloat162 p2 = *reinterpret_cast<const __nv_bfloat162*>(po + s * D + i * 8 + 2 * cq);
        const float2 pf = __bfloat1622float2(p2);
        x0 += ws[s] * pf.x;
        x1 += ws[s] * pf.y;
      }
      *reinterpret_cast<uint32_t*>(dst + i * 8 + 2 * cq) = pack_bf16(x0 * inv, x1 * inv);
    }
  }
}

constexpr size_t kAttnSmem = 4ull * kKT * D * 2;   // K and V, double buffered: 64 KB
constexpr size_t kSelectSmem = 4ull * kKT * D * 2; // hi and lo block means, double buffered: 64 KB

}  // namespace

MobaLayout moba_layout(int B, int T, int H, int bsz, int top_k) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  MobaLayout L{};
  const size_t nblk = (T + bsz - 1) / bsz;
  const size_t E = (size_t)B * H * nblk;
  size_t off = 0;
  L.err = off; off = up(off + 4);   // status word of the bounded device waits
  L.kbar = off; off = up(off + (size_t)B * nblk * H * D * 4);   // hi and lo bf16 halves
  L.idx = off; off = up(off + (size_t)B * H * T * (top_k + 1) * 4);
  L.counts = off; off = up(off + E * 4);
  L.offsets = off; off = up(off + (E + 1) * 4);
  L.chunks = off; off = up(off + (E + 1) * 4);
  L.fill = off; off = up(off + E * 4);
  // chunk -> list, for the smallest chunk size used (64 queries)
  L.chunk_list = off; off = up(off + ((size_t)B * H * T * top_k / kQ + E + 1) * 4);
  L.list = off; off = up(off + (size_t)B * H * T * top_k * 4);
  L.part_lse = off; off = up(off + (size_t)B * T * H * top_k * 4);
  L.part_o = off; off = up(off + (size_t)B * T * H * top_k * D * 2);
  L.total = off;
  return L;
}

template <int KK>
static cudaError_t launch_select(const MobaArgs& a, const __nv_bfloat16* q, const __nv_bfloat16* kbar, int32_t* idx,
                                 int32_t* counts, int nblk, cudaStream_t st) {
  if ((size_t)nblk * 4 > kSelectSmem) return cudaErrorInvalidValue;   // the per-CTA pick counts
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e =
        cudaFuncSetAttribute(moba_select_kernel<KK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSelectSmem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  moba_select_kernel<KK><<<dim3((a.T + kSelQ - 1) / kSelQ, a.H, a.B), kSelThreads, kSelectSmem, st>>>(q, kbar, idx, counts, a.B,
                                                                                            a.T, a.H, a.bsz, nblk);
  return cudaGetLastError();
}

cudaError_t launch_moba(const MobaArgs& a, cudaStream_t st) {
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e = cudaFuncSetAttribute(moba_past_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moba_own_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAttnSmem);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  const int nblk = (a.T + a.bsz - 1) / a.bsz;
  const int E = a.B * a.H * nblk;
  const MobaLayout L = moba_layout(a.B, a.T, a.H, a.bsz, a.top_k);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  __nv_bfloat16* kbar = reinterpret_cast<__nv_bfloat16*>(ws + L.kbar);
  int32_t* idx = a.idx ? a.idx : reinterpret_cast<int32_t*>(ws + L.idx);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  int32_t* chunks = reinterpret_cast<int32_t*>(ws + L.chunks);
  int32_t* fill = reinterpret_cast<int32_t*>(ws + L.fill);
  int32_t* chunk_list = reinterpret_cast<int32_t*>(ws + L.chunk_list);
  int32_t* list = reinterpret_cast<int32_t*>(ws + L.list);
  float* part_lse = reinterpret_cast<float*>(ws + L.part_lse);
  __nv_bfloat16* part_o = reinterpret_cast<__nv_bfloat16*>(ws + L.part_o);
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(a.k);
  const __nv_bfloat16* v = static_cast<const __nv_bfloat16*>(a.v);
  const bool tc = moba_past_tc_supported(a);
  cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)E * 4, st);
  if (e != cudaSuccess) return e;
  if (a.mark) { e = a.mark(a.mark_ctx, st); if (e != cudaSuccess) return e; }
  moba_mean_kernel<<<dim3(nblk, a.H, a.B), D, 0, st>>>(k, kbar, a.B, a.T, a.H, a.bsz, nblk);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.mark) { e = a.mark(a.mark_ctx, st); if (e != cudaSuccess) return e; }
  if (moba_select_tc_supported(a, nblk)) {
    e = launch_moba_select_tc(a, kbar, idx, counts, nblk, st);
  } else switch (a.top_k) {
    case 0: e = launch_select<0>(a, q, kbar, idx, counts, nblk, st); break;
    case 1: e = launch_select<1>(a, q, kbar, idx, counts, nblk, st); break;
    case 2: e = launch_select<2>(a, q, kbar, idx, counts, nblk, st); break;
    case 3: e = launch_select<3>(a, q, kbar, idx, counts, nblk, st); break;
    case 4: e = launch_select<4>(a, q, kbar, idx, counts, nblk, st); break;
    case 5: e = launch_select<5>(a, q, kbar, idx, counts, nblk, st); break;
    case 6: e = launch_select<6>(a, q, kbar, idx, counts, nblk, st); break;
    case 7: e = launch_select<7>(a, q, kbar, idx, counts, nblk, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  if (a.mark) { e = a.mark(a.mark_ctx, st); if (e != cudaSuccess) return e; }
  const int cq = tc ? moba_past_tc_chunk() : kQ;   // queries per past-attention chunk
  moba_scan_kernel<<<1, 1024, 0, st>>>(counts, offsets, chunks, fill, chunk_list, E, cq);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const size_t smem = (size_t)nblk * 4;   // at most 16384 blocks: 64 KB
    static PerDevice scatter_attr;
    e = scatter_attr.once(
        [] { return cudaFuncSetAttribute(moba_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 65536); });
    if (e != cudaSuccess) return e;
    if (smem > 65536) return cudaErrorInvalidValue;
    moba_scatter_kernel<<<dim3((a.T + kScatterQ - 1) / kScatterQ, a.B * a.H), kScatterQ, smem, st>>>(
        idx, offsets, fill, list, a.T, a.H, nblk, a.top_k, a.bsz);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.mark) { e = a.mark(a.mark_ctx, st); if (e != cudaSuccess) return e; }
  const int sms = sm_count();
  if (a.top_k > 0 && tc) {
    // every list holds at most B*H*T*top_k entries in all: the chunk count is bounded by
    // that over the chunk size plus one partial chunk per list
    const size_t max_chunks = ((size_t)a.B * a.H * a.T * a.top_k + cq - 1) / cq + (size_t)E;
    e = launch_moba_past_tc(a, counts, offsets, chunks, chunk_list, list, part_o, part_lse, nblk, E, max_chunks, st);
    if (e != cudaSuccess) return e;
  } else if (a.top_k > 0) {
    moba_past_kernel<<<sms * 3, kThreads, kAttnSmem, st>>>(q, k, v, counts, offsets, chunks, list, part_o, part_lse,
                                                           a.T, a.H, nblk, a.bsz, a.top_k, E, a.scale_log2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.mark) { e = a.mark(a.mark_ctx, st); if (e != cudaSuccess) return e; }
  if (tc) {
    e = launch_moba_own_tc(a, idx, part_o, part_lse, st);
    if (e != cudaSuccess) return e;
  } else {
    moba_own_kernel<<<dim3((a.T + kQ - 1) / kQ, a.H, a.B), kThreads, kAttnSmem, st>>>(
        q, k, v, idx, part_o, part_lse, static_cast<__nv_bfloat16*>(a.out), a.T, a.H, a.bsz, a.top_k, a.scale_log2);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (a.mark) e = a.mark(a.mark_ctx, st);
  return e;
}

}  // namespace nsa
