// K2 and K4 on the 5th-generation tensor cores.  K2: compressed attention + group-summed block
// scores + top-k ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5, §8; "一文比较 Kimi 和
// Deepseek 的两篇稀疏注意力机制论文", "Deepseek 的论文核心点": the selection scores come
// from the compressed attention and the group's heads add them before one top-k).
//
// One CTA = one KV group g and 8 consecutive tokens; its 128 query rows (token-major,
// 16 heads per token) are one tcgen05 M=128 tile held in shared memory.  The group's
// compressed keys/values stream through shared memory by TMA in tiles of 128 blocks.
//   pass A   S = Q Kc^T into TMEM (rows = (token, head)); each softmax thread owns a
//            row and keeps its running max and sum -> log-sum-exp per row.
//   pass B   S^T = Kc Q^T into TMEM (rows = compressed blocks, columns = (token, head)):
//            each softmax thread owns one compressed block, forms the normalised
//            probabilities of its 128 columns, adds each token's 16 heads in registers
//            (the group sum), folds them into 64-token selection-block scores, and
//            writes P^T (bf16) to shared memory; O^T = Vc^T P^T accumulates in TMEM
//            (rows = value dims), already normalised, so no rescaling is ever needed.
//   top-k    per token over the selection-block scores in shared memory.
//   epilogue acc[t, h, :] = g_cmp * o_cmp, read from O^T (each thread one value dim).
// Warp roles: 8 TMA producer, 9 MMA issuer (and TMEM owner), 0-7 softmax / epilogue in
// two groups of four (warp w owns TMEM lanes 32*(w%4)..+31; group w/4 takes one half of
// every tile's 128 columns: in the second pass that half is exactly four tokens).  Every wait is bounded (see tc.cuh); on a
// timeout the kernel records an error word, stops issuing work, and frees its TMEM.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int kSoftWarps = 8;                 // two groups of four softmax warps
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kTok = 8;            // tokens per CTA
constexpr int kRowsM = 128;        // query rows per CTA (8 tokens x 16 heads)
constexpr int kBlk = 128;          // compressed blocks per tile
constexpr int kKcSlots = 3;        // ring of 64-column Kc slices
constexpr int kMaxSel = 1024;
constexpr int kL = 32, kS = 16, kSel = 64;
constexpr uint32_t kSlice = kBlk * 128;          // one 64-column slice of a 128-row tile: 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

enum Err { kErrQ = 1, kErrKcFull, kErrKcEmpty, kErrVcFull, kErrVcEmpty, kErrSFull, kErrSEmpty, kErrPFull,
           kErrPEmpty, kErrOFull };

template <int DK, int DV>
struct Smem {
  static constexpr int kQSlices = DK / 64, kVSlices = DV / 64;
  static constexpr uint32_t kQ = 0;                                         // Q: kQSlices x 16 KB
  static constexpr uint32_t kKc = kQ + kQSlices * kSlice;                   // Kc ring: kKcSlots x 16 KB
  static constexpr uint32_t kVc = kKc + kKcSlots * kSlice;                  // Vc: 2 buffers x kVSlices x 16 KB
  static constexpr uint32_t kP = kVc + 2 * kVSlices * kSlice;               // P^T: 2 x 16 KB (N = 128 rows)
  static constexpr uint32_t kScore = kP + 2 * kSlice;                       // [8][1024] fp32
  static constexpr uint32_t kLse = kScore + kTok * kMaxSel * 4;             // [128] fp32
  static constexpr uint32_t kGate = kLse + kRowsM * 4;                      // [128] fp32
  static constexpr uint32_t kML = kP;                                       // [2][128][2] fp32, while P^T is unused
  static constexpr uint32_t kBar = kGate + kRowsM * 4;                      // mbarriers
  static constexpr int kNumBars = 1 + 2 * kKcSlots + 2 * 2 + 2 * 2 + 2 + 1;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;                         // room to align the base to 1 KB
  static_assert(kAlloc <= 232448, "shared memory");
};


__device__ __forceinline__ int n_visible(int t, int nc) { return t < kL - 1 ? 0 : min(nc, (t - kL + 1) / kS + 1); }

using tc::named_sync;
using tc::vote_all;

// kWin = false: compressed branch (keys = compressed blocks, scores + top-k, acc = g_cmp * o).
// kWin = true:  sliding window (keys = tokens [t0-w+1, t0+7], each row masked to its own
//               window, out = bf16(acc + g_win * o)).
template <int DK, int DV, bool kWin>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_vc, const __nv_bfloat16* __restrict__ gates,
               float* __restrict__ acc, int32_t* __restrict__ idx_out, __nv_bfloat16* __restrict__ out, int T, int Hq,
               int Hkv, int nc, int top_k, int force_first, int force_local, int window, float scale_log2,
               int* __restrict__ err) {
  using SM = Smem<DK, DV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sKc = smem + SM::kKc;
  uint8_t* sVc = smem + SM::kVc;
  uint8_t* sP = smem + SM::kP;
  float* sScore = reinterpret_cast<float*>(smem + SM::kScore);
  float* sLse = reinterpret_cast<float*>(smem + SM::kLse);
  float* sGate = reinterpret_cast<float*>(smem + SM::kGate);
  float* sML = reinterpret_cast<float*>(smem + SM::kML);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* bar_q = bars;
  uint64_t* kc_full = bars + 1;
  uint64_t* kc_empty = kc_full + kKcSlots;
  uint64_t* vc_full = kc_empty + kKcSlots;
  uint64_t* vc_empty = vc_full + 2;
  uint64_t* s_full = vc_empty + 2;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 1;
  uint64_t* o_full = p_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tok_tiles = (T + kTok - 1) / kTok;
  const int t0 = (n_tok_tiles - 1 - (int)blockIdx.x) * kTok;   // longest rows first
  const int g = blockIdx.y, b = blockIdx.z;
  const int t_last = min(t0 + kTok - 1, T - 1);
  // keys: compressed blocks 0.. (kWin = false) or tokens kv_lo.. (kWin = true)
  const int kv_lo = kWin ? max(0, t0 - window + 1) : 0;
  const int ntiles = kWin ? (t_last - kv_lo + kBlk) / kBlk : (n_visible(t_last, nc) + kBlk - 1) / kBlk;
  const int kv_rows = kWin ? T : nc;   // rows per batch in the key/value tensor maps

  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int i = 0; i < kKcSlots; ++i) { tc::mbar_init(kc_full + i, 1); tc::mbar_init(kc_empty + i, 1); }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(vc_full + i, 1);
      tc::mbar_init(vc_empty + i, 1);
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_empty + i, kSoftWarps);
    }
    tc::mbar_init(p_full, kSoftWarps);
    tc::mbar_init(p_empty, 1);
    tc::mbar_init(o_full, 1);
    tc::fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_kc);
      tc::prefetch_tmap(&tm_vc);
      tc::mbar_expect_tx(bar_q, SM::kQSlices * kSlice);
      for (int s = 0; s < SM::kQSlices; ++s) tc::tma_load_3d(sQ + s * kSlice, &tm_q, bar_q, s * 64, g * 16, b * T + t0);
      int fill = 0;   // Kc slice fills so far
      bool ok = true;
      for (int pass = 0; pass < 2 && ok; ++pass) {
        for (int n = 0; n < ntiles && ok; ++n) {
          const int row = b * kv_rows + kv_lo + n * kBlk;
          for (int s = 0; s < SM::kQSlices && ok; ++s, ++fill) {
            const int slot = fill % kKcSlots;
            ok = tc::mbar_wait(kc_empty + slot, ((fill / kKcSlots) & 1) ^ 1, err, kErrKcEmpty);
            if (!ok) break;
            tc::mbar_expect_tx(kc_full + slot, kSlice);
            tc::tma_load_3d(sKc + slot * kSlice, &tm_kc, kc_full + slot, s * 64, g, row);
          }
          if (pass == 1 && ok) {
            const int vb = n & 1;
            ok = tc::mbar_wait(vc_empty + vb, ((n >> 1) & 1) ^ 1, err, kErrVcEmpty);
            if (!ok) break;
            tc::mbar_expect_tx(vc_full + vb, SM::kVSlices * kSlice);
            for (int s = 0; s < SM::kVSlices; ++s)
              tc::tma_load_3d(sVc + (vb * SM::kVSlices + s) * kSlice, &tm_vc, vc_full + vb, s * 64, g, row);
          }
        }
      }
      // before leaving, let the copies still in flight land (bounded)
      for (int i = 0; i < kKcSlots && i < fill; ++i) {
        const int f = fill - 1 - i;
        tc::mbar_wait(kc_full + (f % kKcSlots), (f / kKcSlots) & 1, err, kErrKcFull);
      }
      for (int n = max(0, ntiles - 2); n < ntiles; ++n) tc::mbar_wait(vc_full + (n & 1), (n >> 1) & 1, err, kErrVcFull);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idA = tc::idesc_bf16(128, 128, 0, 0);     // S  = Q  Kc^T   (both K-major)
      const uint32_t idPV = tc::idesc_bf16(128, 128, 1, 1);    // O^T = Vc^T P^T (both MN-major)
      bool ok = tc::mbar_wait(bar_q, 0, err, kErrQ);
      tc::tc_fence_after();
      int use = 0;    // S buffer uses over both passes
      int fill = 0;   // Kc slices consumed
      auto issue_s = [&](int pass) -> bool {
        const int sb = use & 1;
        if (!tc::mbar_wait(s_empty + sb, ((use >> 1) & 1) ^ 1, err, kErrSEmpty)) return false;
        tc::tc_fence_after();
        const uint32_t d = tmem + (sb ? kColS1 : kColS0);
        for (int s = 0; s < SM::kQSlices; ++s, ++fill) {
          const int slot = fill % kKcSlots;
          if (!tc::mbar_wait(kc_full + slot, (fill / kKcSlots) & 1, err, kErrKcFull)) return false;
          tc::tc_fence_after();
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t dq = tc::sdesc(sQ + s * kSlice + ks * 32, 16, 1024);
            const uint64_t dk = tc::sdesc(sKc + slot * kSlice + ks * 32, 16, 1024);
            if (pass == 0) tc::mma_ss(d, dq, dk, idA, (s | ks) != 0);
            else tc::mma_ss(d, dk, dq, idA, (s | ks) != 0);
          }
          tc::mma_commit(kc_empty + slot);
        }
        tc::mma_commit(s_full + sb);
        ++use;
        return true;
      };
      for (int n = 0; n < ntiles && ok; ++n) ok = issue_s(0);
      if (ok && ntiles > 0) ok = issue_s(1);
      for (int n = 0; n < ntiles && ok; ++n) {
        if (n + 1 < ntiles) ok = issue_s(1);
        if (!ok) break;
        ok = tc::mbar_wait(p_full, n & 1, err, kErrPFull) && tc::mbar_wait(vc_full + (n & 1), (n >> 1) & 1, err, kErrVcFull);
        if (!ok) break;
        tc::tc_fence_after();
        const uint8_t* vb = sVc + (n & 1) * SM::kVSlices * kSlice;
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          const uint64_t da = tc::sdesc(vb + ks * 16 * 128, kSlice, 1024);
          const uint64_t db = tc::sdesc(sP + ks * 16 * 128, kSlice, 1024);
          tc::mma_ss(tmem + kColO, da, db, idPV, (n | ks) != 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(vc_empty + (n & 1));
      }
      if (ok && ntiles > 0) tc::mma_commit(o_full);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Two groups of four warps; group gr takes columns [64*gr, 64*gr+64) of every tile.
    // Warp quarter q = warp % 4 owns TMEM lanes 32q..32q+31; r is this thread's lane.
    const int gr = warp >> 2, q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int col0 = 64 * gr;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    bool ok = true;
    int use = 0;
    if (gr == 0) {   // gates of the 128 rows
      const int t = t0 + r / 16, h = g * 16 + (r % 16);
      sGate[r] = t < T ? __bfloat162float(gates[(((size_t)b * T + t) * Hq + h) * 3 + (kWin ? 2 : 0)]) : 0.f;
    }
    if (!kWin)
      for (int i = gr * 128 + r; i < kTok * kMaxSel; i += 256) sScore[i] = 0.f;

    // pass A: this thread's row r = (token r/16, head r%16), its half of every tile's columns
    {
      const int my_t = t0 + r / 16;
      const int my_lo = kWin ? max(0, my_t - window + 1) : 0;
      const int my_hi = my_t < T ? (kWin ? my_t + 1 : n_visible(my_t, nc)) : 0;
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < ntiles && ok; ++n, ++use) {
        const int sb = use & 1;
        ok = tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull);
        ok = __all_sync(0xffffffffu, ok);      // reconverge before the warp-wide TMEM loads
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t base = lane_addr + (sb ? kColS1 : kColS0) + col0;
        float v[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld16(base + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_empty + sb);
        // masked, scaled scores; only a tile that straddles this row's range needs the
        // per-element test.  Max and sum use eight independent chains each.
        const int i0 = kv_lo + n * kBlk + col0;
        if (i0 >= my_lo && i0 + 63 < my_hi) {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] *= scale_log2;
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) v[j] = (i0 + j >= my_lo && i0 + j < my_hi) ? v[j] * scale_log2 : -INFINITY;
        }
        float cmx[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) cmx[c] = fmaxf(fmaxf(v[c], v[c + 8]), fmaxf(v[c + 16], v[c + 24]));
#pragma unroll
        for (int c = 0; c < 8; ++c) cmx[c] = fmaxf(cmx[c], fmaxf(fmaxf(v[c + 32], v[c + 40]), fmaxf(v[c + 48], v[c + 56])));
        const float cm = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                               fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7])));
        const float mn = fmaxf(m, cm);
        if (mn != -INFINITY) {
          float ps[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) ps[c] = ex2(v[c] - mn);
#pragma unroll
          for (int j = 8; j < 64; ++j) ps[j & 7] += ex2(v[j] - mn);
          const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
          l = l * ex2(m - mn) + sum;
          m = mn;
        }
      }
      sML[(gr * 128 + r) * 2] = m;
      sML[(gr * 128 + r) * 2 + 1] = l;
    }
    ok = vote_all(3, kSoftWarps * 32, ok);
    if (gr == 0) {
      const float m0 = sML[r * 2], l0 = sML[r * 2 + 1], m1 = sML[(128 + r) * 2], l1 = sML[(128 + r) * 2 + 1];
      const float M = fmaxf(m0, m1);
      const float L = M == -INFINITY ? 0.f : l0 * ex2(m0 - M) + l1 * ex2(m1 - M);
      sLse[r] = (t0 + r / 16 < T && L > 0.f) ? M + __log2f(L) : INFINITY;
    }
    named_sync(3, kSoftWarps * 32);

    // pass B: this thread's key r of every tile; columns = tokens 4*gr .. 4*gr+3, 16 heads each
    int lo_tok[4], hi_tok[4], nb_tok[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = t0 + 4 * gr + k;
      const bool in = t < T;
      lo_tok[k] = kWin ? max(0, t - window + 1) : 0;
      hi_tok[k] = in ? (kWin ? t + 1 : n_visible(t, nc)) : 0;
      nb_tok[k] = in ? t / kSel + 1 : 0;
    }
    uint8_t* prow = sP + gr * kSlice + r * 128;   // row r of N-block gr of P^T
    // Selection-block scores: block j = i/4 collects i = 4j-1 .. 4j+3.  Each group of four
    // lanes adds its own four blocks plus the lane just below it into the block's entry.
    // Lane 31's block (i % 4 == 3) also belongs to the first selection block of the next
    // warp (or of the next tile); that carry is added two tiles later, after waiting for
    // the P^T phase that every softmax warp releases only after its own score writes, so
    // no barrier is needed inside the loop.  Each entry receives at most two additions.
    float carry_a[4] = {0.f, 0.f, 0.f, 0.f}, carry_b[4] = {0.f, 0.f, 0.f, 0.f};   // tiles n-1, n-2
    auto add_carry = [&](const float (&c)[4], int tile) {
      const int jt = tile * (kBlk / 4) + q4 * 8 + 8;
      if (lane == 31) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (jt < nb_tok[k]) sScore[(4 * gr + k) * kMaxSel + jt] += c[k];
      }
    };
    for (int n = 0; n < ntiles; ++n, ++use) {
      const int sb = use & 1;
      // no barrier inside this loop: a warp that gives up leaves at once and the others
      // give up at their next wait (they see the error word); all meet after the loop
      ok = tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t base = lane_addr + (sb ? kColS1 : kColS0) + col0;
      float v[64];
#pragma unroll
      for (int c = 0; c < 4; ++c) tc::tmem_ld16(base + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
      tc::tmem_wait_ld();
      const int i = kv_lo + n * kBlk + r;        // this thread's key (compressed block or token)
      float tok_sum[4];
      uint32_t pk[32];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const bool vis = i >= lo_tok[k] && i < hi_tok[k];
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float p0 = vis ? ex2(v[16 * k + j] * scale_log2 - sLse[col0 + 16 * k + j]) : 0.f;
          const float p1 = vis ? ex2(v[16 * k + j + 1] * scale_log2 - sLse[col0 + 16 * k + j + 1]) : 0.f;
          s += p0 + p1;
          __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
          pk[8 * k + j / 2] = *reinterpret_cast<uint32_t*>(&h2);
        }
        tok_sum[k] = s;
      }
      if (!kWin) {
        const int j0 = n * (kBlk / 4) + q4 * 8;    // first selection block of this warp
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float vv = tok_sum[k];
          float g4 = vv + __shfl_xor_sync(0xffffffffu, vv, 1);
          g4 += __shfl_xor_sync(0xffffffffu, g4, 2);
          const float prev = __shfl_up_sync(0xffffffffu, vv, 1);
          const int j = j0 + (lane >> 2);
          if ((lane & 3) == 0 && j < nb_tok[k]) sScore[(4 * gr + k) * kMaxSel + j] += g4 + (lane > 0 ? prev : 0.f);
        }
      }
      // P^T(n) may overwrite the buffer once PV(n-1) has read it
      if (n > 0) ok = tc::mbar_wait(p_empty, (n - 1) & 1, err, kErrPEmpty);
      if (!kWin && n > 0 && ok) {
        // P^T(n-1) was released by every softmax warp after its score writes of tiles
        // <= n-1; this warp has not released P^T(n) yet, so the phase is unambiguous
        ok = tc::mbar_wait(p_full, (n - 1) & 1, err, kErrPFull);
        if (n > 1) add_carry(carry_b, n - 2);
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        carry_b[k] = carry_a[k];
        carry_a[k] = tok_sum[k];
      }
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      tc::tc_fence_before();
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(s_empty + sb);
        tc::mbar_arrive(p_full);
      }
    }
    ok = vote_all(3, kSoftWarps * 32, ok);
    if (!kWin && ok) {    // the carries of the last two tiles
      if (ntiles > 1) add_carry(carry_b, ntiles - 2);
      if (ntiles > 0) add_carry(carry_a, ntiles - 1);
    }
    named_sync(3, kSoftWarps * 32);

    // top-k: warp w takes token w
    if (!kWin && ok) {
      const int k = warp;
      const int t = t0 + k;
      if (t < T) {
        const float* score = sScore + k * kMaxSel;
        const int nb = t / kSel + 1;
        int32_t* dst = idx_out + (((size_t)b * Hkv + g) * T + t) * top_k;
        if (nb <= top_k) {
          for (int j = lane; j < top_k; j += 32) dst[j] = j < nb ? j : -1;
        } else {
          const int own = t / kSel;
          uint32_t taken = 0;
          int nforced = 0;
          if (force_first) { if (lane == 0) taken |= 1u; ++nforced; }
          if (force_local && !(force_first && own == 0)) {
            if (lane == (own & 31)) taken |= 1u << (own >> 5);
            ++nforced;
          }
          const int mmax = (nb + 31) >> 5;
          // this lane's candidates j = lane + 32*mm as order-preserving integer keys: the
          // scores are sums of probabilities (>= 0), so their bit patterns order like the
          // values; key 0 marks "no candidate"
          uint32_t key[32];
#pragma unroll
          for (int mm = 0; mm < 32; ++mm) {
            const int j = lane + 32 * mm;
            key[mm] = (mm < mmax && j < nb && !((taken >> mm) & 1u)) ? __float_as_uint(score[j]) + 1u : 0u;
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
            // the lowest block index among the lanes holding the maximum
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
          for (int mm = 0; mm < mmax; ++mm) {
            const bool sel = (taken >> mm) & 1u;
            const uint32_t bal = __ballot_sync(0xffffffffu, sel);
            if (sel) dst[pos + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * mm;
            pos += __popc(bal);
          }
          for (int j = pos + lane; j < top_k; j += 32) dst[j] = -1;
        }
      }
    }

    // epilogue: lane r = value dim r of O^T; this group's 64 columns = tokens 4*gr .. 4*gr+3
    float prevacc[kWin ? 64 : 1];
    if (kWin) {
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int t = t0 + 4 * gr + c / 16;
        const size_t row = ((size_t)b * T + min(t, T - 1)) * Hq + g * 16 + (c % 16);
        prevacc[c] = (t < T && r < DV) ? acc[row * DV + r] : 0.f;
      }
    }
    if (ok && ntiles > 0) ok = tc::mbar_wait(o_full, 0, err, kErrOFull);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc::tc_fence_after();
      float v[64];
      if (ntiles > 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) tc::tmem_ld16(lane_addr + kColO + col0 + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) v[c] = 0.f;
      }
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int t = t0 + 4 * gr + c / 16;
        if (t < T && r < DV) {
          const size_t row = ((size_t)b * T + t) * Hq + g * 16 + (c % 16);
          const float gv = sGate[col0 + c] * v[c];
          if (kWin) out[row * DV + r] = __float2bfloat16_rn(prevacc[c] + gv);
          else acc[row * DV + r] = gv;
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DK, int DV, bool kWin>
cudaError_t launch_tc(const FwdArgs& a, cudaStream_t st) {
  using SM = Smem<DK, DV>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DK, DV, kWin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM::kAlloc);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const int rows = kWin ? a.T : a.nc;
  const void* kp = kWin ? a.k : a.kc;
  const void* vp = kWin ? a.v : a.vc;
  CUtensorMap mq, mk, mv;
  const uint64_t dq[3] = {(uint64_t)DK, (uint64_t)a.Hq, (uint64_t)a.B * a.T};
  const uint64_t sq[2] = {(uint64_t)DK * 2, (uint64_t)a.Hq * DK * 2};
  const uint32_t bq[3] = {64, 16, kTok};
  const uint64_t dk3[3] = {(uint64_t)DK, (uint64_t)a.Hkv, (uint64_t)a.B * rows};
  const uint64_t sk3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hkv * DK * 2};
  const uint64_t dv3[3] = {(uint64_t)DV, (uint64_t)a.Hkv, (uint64_t)a.B * rows};
  const uint64_t sv3[2] = {(uint64_t)DV * 2, (uint64_t)a.Hkv * DV * 2};
  const uint32_t bkv[3] = {64, 1, kBlk};
  if (!make_tmap_bf16(&mq, a.q, 3, dq, sq, bq)) return cudaErrorInvalidValue;
  if (rows > 0) {
    if (!make_tmap_bf16(&mk, kp, 3, dk3, sk3, bkv) || !make_tmap_bf16(&mv, vp, 3, dv3, sv3, bkv))
      return cudaErrorInvalidValue;
  } else {
    mk = mq;   // never dereferenced: no tile is loaded when there is no key
    mv = mq;
  }
  dim3 grid((a.T + kTok - 1) / kTok, a.Hkv, a.B);
  attn_tc_kernel<DK, DV, kWin><<<grid, kThreads, SM::kAlloc, st>>>(
      mq, mk, mv, static_cast<const __nv_bfloat16*>(a.gates), a.acc, a.idx, static_cast<__nv_bfloat16*>(a.out), a.T,
      a.Hq, a.Hkv, a.nc, a.top_k, a.force_first, a.force_local, a.window, a.scale_log2, a.err);
  return cudaGetLastError();
}
}  // namespace

bool cmp_select_tc_supported(const FwdArgs& a) {
  return a.G == 16 && a.dv == 128 && (a.dk == 128 || a.dk == 192) && a.T <= kMaxSel * kSel && a.err != nullptr;
}

cudaError_t launch_cmp_select_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192) return launch_tc<192, 128, false>(a, st);
  return launch_tc<128, 128, false>(a, st);
}

bool swa_tc_supported(const FwdArgs& a) { return cmp_select_tc_supported(a); }

cudaError_t launch_swa_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192) return launch_tc<192, 128, true>(a, st);
  return launch_tc<128, 128, true>(a, st);
}

}  // namespace nsa
