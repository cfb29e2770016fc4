// MoBA block selection on the fifth-generation tensor cores ("一文比较 Kimi 和 Deepseek 的两篇
// 稀疏注意力机制论文", "Kimi 的论文核心点": each query scores the past blocks by the dot product
// with their mean key and keeps the top-k; the own block is always attended).
//
// One CTA per 128 consecutive queries of one (batch, head): the 128 queries are the M of the
// MMA (one TMEM lane each), the past blocks' means come in tiles of 64 (the N):
//   S = Q Kbar^T   (M = 128, N = 64, K = 128: the bf16 hi and lo halves of the fp32 means
//                   accumulate into the same fp32 tile, so S = q . (hi + lo))
// Warp 16 loads the queries and the mean tiles by TMA (two tiles in flight), one thread of
// warp 17 issues the MMAs into two TMEM buffers, and warps 0-15 offer the past blocks to
// register top-k lists (larger score first, then the lower block): warps w, w + 4, w + 8 and
// w + 12 read the same 32 query rows (TMEM lane quadrant w % 4), each 16 of a tile's 64
// blocks, and the four lists of a query are merged at the end.  The offers are the kernel's
// cost (with random scores nearly every offer inserts in some lane of the warp), so each
// query's chain is split in four.  The merge lists and then the per-block pick counts use the
// tile buffers, free by then; the counts are added to the global ones once per block.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int D = 128;
constexpr int kRows = 128;                        // queries per CTA
constexpr int kTileB = 64;                        // block means per tile
constexpr int kOfferWarps = 16, kTmaWarp = 16, kMmaWarp = 17, kThreads = 576;
constexpr int kSplit = kOfferWarps / 4;          // offer threads per query
constexpr int kCols = kTileB / kSplit;           // a tile's blocks per offer thread
constexpr uint32_t kQSlab = kRows * 128;          // 128 rows x 64 bf16 (128-byte swizzle): 16 KB
constexpr uint32_t kBSlab = kTileB * 128;         // 64 rows x 64 bf16: 8 KB
constexpr uint32_t kTileBytes = 4 * kBSlab;       // hi and lo, two 64-column slabs each: 32 KB
constexpr uint32_t kTmemCols = 128;               // two 64-column S buffers
constexpr int kMaxBlocks = 2 * (int)kTileBytes / 4;   // the pick counts reuse the two tile buffers

enum Err { kErrQ = 101, kErrFull, kErrEmpty, kErrSFull, kErrSEmpty };

struct SelSmem {
  static constexpr uint32_t kQ = 0;                          // 2 slabs
  static constexpr uint32_t kB = kQ + 2 * kQSlab;            // [2 tiles][hi s0, hi s1, lo s0, lo s1]
  static constexpr uint32_t kBar = kB + 2 * kTileBytes;
  static constexpr int kNumBars = 1 + 2 + 2 + 2 + 2;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};

// the KK best (score desc, then block asc) of the values offered, sorted best-first, in registers
template <int KK>
struct TopRow {
  static constexpr int N = KK > 0 ? KK : 1;
  float v[N];
  int j[N];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      v[i] = -FLT_MAX;
      j[i] = 0x7fffffff;
    }
  }
  __device__ __forceinline__ static bool better(float a, int ja, float b, int jb) {
    return a > b || (a == b && ja < jb);
  }
  __device__ __forceinline__ void offer(float val, int idx) {
    if (!better(val, idx, v[N - 1], j[N - 1])) return;
    float cv = val;
    int cj = idx;
#pragma unroll
    for (int i = 0; i < N; ++i)
      if (better(cv, cj, v[i], j[i])) {
        const float xv = v[i];
        const int xj = j[i];
        v[i] = cv;
        j[i] = cj;
        cv = xv;
        cj = xj;
      }
  }
};

template <int KK>
__global__ void __launch_bounds__(kThreads, 2)
moba_select_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kb,
                      int32_t* __restrict__ idx, int32_t* __restrict__ counts, int B, int T, int H, int bsz, int nblk,
                      int* __restrict__ err) {
  using SM = SelSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sB = smem + SM::kB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* bar_q = bars;
  uint64_t* full = bars + 1;      // [tile buffer] the means landed
  uint64_t* empty = full + 2;     // [tile buffer] the MMAs have read them
  uint64_t* s_full = empty + 2;   // [S buffer] the scores are in TMEM
  uint64_t* s_empty = s_full + 2; // [S buffer] the offer warps have read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kRows, h = blockIdx.y, b = blockIdx.z;
  const int Jc = min(t0 + kRows - 1, T - 1) / bsz;    // the largest own block of the CTA's queries
  const bool score = KK > 0 && Jc > KK;              // else every query takes all its past blocks
  const int ntile = score ? (Jc + kTileB - 1) / kTileB : 0;

  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(full + i, 1);
      tc::mbar_init(empty + i, 1);
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_empty + i, kOfferWarps);
    }
    tc::fence_barrier_init();
  }
  if (score && warp == kMmaWarp) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = score ? *tmem_slot : 0u;

  TopRow<KK> top;
  top.init();
  const int part = warp >> 2;                        // offer warps: which kCols of a tile's blocks
  const int r = 32 * (warp & 3) + lane;              // this thread's query (offer warps)
  const int t = t0 + r;
  const int J = t / bsz;                             // its own block: the past blocks are 0 .. J-1

  if (warp == kTmaWarp) {
    if (score && lane == 0) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_kb);
      tc::mbar_expect_tx(bar_q, 2 * kQSlab);
      for (int s = 0; s < 2; ++s) tc::tma_load_3d(sQ + s * kQSlab, &tm_q, bar_q, s * 64, h, b * T + t0);
      bool ok = true;
      for (int it = 0; it < ntile && ok; ++it) {
        const int buf = it & 1;
        ok = tc::mbar_wait(empty + buf, ((it >> 1) & 1) ^ 1, err, kErrEmpty);
        if (!ok) break;
        const int j0 = it * kTileB;
        uint8_t* dst = sB + buf * kTileBytes;
        tc::mbar_expect_tx(full + buf, kTileBytes);
        for (int s = 0; s < 2; ++s) {
          tc::tma_load_3d(dst + s * kBSlab, &tm_kb, full + buf, s * 64, h, b * nblk + j0);                  // hi
          tc::tma_load_3d(dst + (2 + s) * kBSlab, &tm_kb, full + buf, s * 64, h, (B + b) * nblk + j0);     // lo
        }
      }
      // the last loads land before the CTA's final barrier: the MMA thread waits for every one
    }
  } else if (warp == kMmaWarp) {
    if (score && tc::elect_one()) {
      const uint32_t idS = tc::idesc_bf16(kRows, kTileB, 0, 0);   // S = Q Kbar^T: both K-major
      bool ok = tc::mbar_wait(bar_q, 0u, err, kErrQ);
      for (int it = 0; it < ntile && ok; ++it) {
        const int buf = it & 1;
        ok = tc::mbar_wait(full + buf, (it >> 1) & 1, err, kErrFull) &&
             tc::mbar_wait(s_empty + buf, ((it >> 1) & 1) ^ 1, err, kErrSEmpty);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t d = tmem + kTileB * buf;
        const uint8_t* src = sB + buf * kTileBytes;
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)   // the hi half, then the lo half of the means
#pragma unroll
          for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t dq = tc::sdesc(sQ + s * kQSlab + ks * 32, 16, 1024);
              const uint64_t dk = tc::sdesc(src + (2 * hl + s) * kBSlab + ks * 32, 16, 1024);
              tc::mma_ss(d, dq, dk, idS, (hl | s | ks) != 0);
            }
        tc::mma_commit(empty + buf);
        tc::mma_commit(s_full + buf);
      }
    }
  } else {
    // ------------------------------------------------------------ offers (one query per thread)
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kCols * part;
    const bool mine = t < T && J > KK;
    bool ok = true;
    for (int it = 0; it < ntile; ++it) {
      const int buf = it & 1;
      ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(s_full + buf, (it >> 1) & 1, err, kErrSFull));
      if (!ok) break;
      tc::tc_fence_after();
      float v[kCols];
#pragma unroll
      for (int c = 0; c < kCols / 16; ++c)
        tc::tmem_ld16(lane_addr + kTileB * buf + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_empty + buf);
      if (mine) {
        const int j0 = it * kTileB + kCols * part;
#pragma unroll
        for (int c = 0; c < kCols; ++c)
          if (j0 + c < J) top.offer(v[c], j0 + c);
      }
    }
  }

  // every tile has been read (the MMAs before the last s_full, the offers before here): the
  // tile buffers take the other lists of each query, which join the first.  After a wait gave
  // up, tiles may still be landing: they are let land first.
  float* mv = reinterpret_cast<float*>(sB);                    // [part - 1][row][7]
  int* mj = reinterpret_cast<int*>(mv + (kSplit - 1) * kRows * 7);
  tc::settle_after_error(err);
  tc::tc_fence_before();
  __syncthreads();
  if (warp < kOfferWarps && part > 0) {
#pragma unroll
    for (int i = 0; i < TopRow<KK>::N; ++i) {
      mv[((part - 1) * kRows + r) * 7 + i] = top.v[i];
      mj[((part - 1) * kRows + r) * 7 + i] = top.j[i];
    }
  }
  __syncthreads();
  if (warp < 4) {
#pragma unroll
    for (int q = 0; q < kSplit - 1; ++q)
#pragma unroll
      for (int i = 0; i < TopRow<KK>::N; ++i) top.offer(mv[(q * kRows + r) * 7 + i], mj[(q * kRows + r) * 7 + i]);
  }
  // then the pick counts of blocks 0 .. Jc
  int32_t* hist = reinterpret_cast<int32_t*>(sB);
  __syncthreads();
  for (int j = tid; j <= Jc; j += kThreads) hist[j] = 0;
  __syncthreads();
  if (warp < 4 && t < T) {
    int sel[TopRow<KK>::N];
    const int kk = min(KK, J);
#pragma unroll
    for (int i = 0; i < TopRow<KK>::N; ++i) sel[i] = J > KK ? top.j[i] : i;
    // ascending block order: odd-even transposition sort over the slots
#pragma unroll
    for (int pass = 0; pass < TopRow<KK>::N; ++pass)
#pragma unroll
      for (int i = pass & 1; i + 1 < TopRow<KK>::N; i += 2)
        if (sel[i] > sel[i + 1]) {
          const int x = sel[i];
          sel[i] = sel[i + 1];
          sel[i + 1] = x;
        }
    int32_t* dst = idx + (((size_t)b * H + h) * T + t) * (KK + 1);
    // a list cut short by a wait that gave up still holds its initial entries: only past
    // blocks are written and counted (the counts and the lists built from them agree)
#pragma unroll
    for (int i = 0; i < KK; ++i) {
      if (i < kk) {
        const bool past = sel[i] >= 0 && sel[i] < J;
        dst[i] = past ? sel[i] : -1;
        if (past) atomicAdd(hist + sel[i], 1);
      } else {
        dst[i + 1] = -1;
      }
    }
    dst[kk] = J;
  }
  __syncthreads();
  int32_t* cnt = counts + ((size_t)b * H + h) * nblk;
  for (int j = tid; j <= Jc; j += kThreads)
    if (hist[j] != 0) atomicAdd(cnt + j, hist[j]);
  if (score && warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int KK>
cudaError_t launch_kk(const MobaArgs& a, const void* kbar, int32_t* idx, int32_t* counts, int nblk,
                      cudaStream_t st) {
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e = cudaFuncSetAttribute(moba_select_tc_kernel<KK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)SelSmem::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  CUtensorMap mq, mkb;
  const uint64_t dq[3] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.B * a.T};
  const uint64_t dkb[3] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)2 * a.B * nblk};
  const uint64_t s3[2] = {(uint64_t)D * 2, (uint64_t)a.H * D * 2};
  const uint32_t bq[3] = {64, 1, (uint32_t)kRows};
  const uint32_t bkb[3] = {64, 1, (uint32_t)kTileB};
  if (!make_tmap_bf16(&mq, a.q, 3, dq, s3, bq) || !make_tmap_bf16(&mkb, kbar, 3, dkb, s3, bkb))
    return cudaErrorInvalidValue;
  dim3 grid((a.T + kRows - 1) / kRows, a.H, a.B);
  moba_select_tc_kernel<KK><<<grid, kThreads, SelSmem::kAlloc, st>>>(mq, mkb, idx, counts, a.B, a.T, a.H, a.bsz,
                                                                     nblk, a.err);
  return cudaGetLastError();
}
}  // namespace

bool moba_select_tc_supported(const MobaArgs& a, int nblk) {
  return a.err != nullptr && a.top_k >= 0 && a.top_k <= 7 && nblk <= kMaxBlocks && a.bsz % kRows == 0;
}

cudaError_t launch_moba_select_tc(const MobaArgs& a, const void* kbar, int32_t* idx, int32_t* counts, int nblk,
                                  cudaStream_t st) {
  switch (a.top_k) {
    case 0: return launch_kk<0>(a, kbar, idx, counts, nblk, st);
    case 1: return launch_kk<1>(a, kbar, idx, counts, nblk, st);
    case 2: return launch_kk<2>(a, kbar, idx, counts, nblk, st);
    case 3: return launch_kk<3>(a, kbar, idx, counts, nblk, st);
    case 4: return launch_kk<4>(a, kbar, idx, counts, nblk, st);
    case 5: return launch_kk<5>(a, kbar, idx, counts, nblk, st);
    case 6: return launch_kk<6>(a, kbar, idx, counts, nblk, st);
    case 7: return launch_kk<7>(a, kbar, idx, counts, nblk, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nsa
