// MoBA past-block attention on the fifth-generation tensor cores ("一文比较 Kimi 和 Deepseek
// 的两篇稀疏注意力机制论文", "Kimi 的论文核心点"; "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文"
// §16-§17: the queries that chose one KV block are gathered, so that the block is read once
// for all of them and the attention over it is a dense product).
//
// Persistent: one CTA per SM walks the chunks, a chunk = up to 128 gathered queries of one
// (batch, head, past block j) list (one TMEM lane per query), against the block's keys in
// 128-key tiles:
//   S = Q K^T        (M = 128 queries, N = 128 keys; two TMEM buffers)
//   O += P V         (M = 128, N = 128; P in SMEM as the K-major A operand)
// Every key of a past block precedes every query that chose it, so nothing is masked.
// Warp roles as in the window kernel: a producer warp (it gathers each chunk's query rows
// with cp.async once the previous chunk's S MMAs are done with them, and streams K slices
// into a 3-slot ring and V tiles double buffered by TMA; both run across chunk boundaries),
// a single-thread MMA issuer that puts S(n+1) ahead of the P.V of tile n,
// and 8 softmax warps: warps w and w+4 share TMEM lanes 32(w%4).. (the same queries) and
// take the key halves [0, 64) and [64, 128) of every tile.  A row's softmax reference moves
// only when a score exceeds it by more than 2^8; the two threads of a row agree on it through
// one barrier of the warp pair per tile, and rescale their halves of O in TMEM when it moves.
// Epilogue per query of the chunk: part_o = bf16(O / l) and part_lse = m + log2(l), merged
// later with the own block.
#include <algorithm>
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int D = 128;                            // head dim of this mode
constexpr int kSoftWarps = 8;
constexpr int kTmaWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kRowsM = 128;                       // queries per chunk
constexpr int kBlk = 128;                         // keys per tile
constexpr int kKSlots = 3;
constexpr uint32_t kSlice = kBlk * 128;           // 128 rows x 64 columns: 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;        // S buffer b at 128b; O at 256
constexpr float kSlack = 8.f;
constexpr int kMaxPast = 8;                       // past-block slots per query (top_k <= 8)

enum Err { kErrQ = 61, kErrKFull, kErrKEmpty, kErrVFull, kErrVEmpty, kErrSFull, kErrSEmpty, kErrPFull, kErrPEmpty,
           kErrOFull, kErrQEmpty, kErrOEmpty };

struct Smem {
  static constexpr uint32_t kQ = 0;                                         // 2 x 64-column slices
  static constexpr uint32_t kK = kQ + 2 * kSlice;                           // ring of 64-column K slices
  static constexpr uint32_t kV = kK + kKSlots * kSlice;                     // 2 tiles x 2 slices
  static constexpr uint32_t kP = kV + 2 * 2 * kSlice;                       // P: [2 key halves][128 rows][128 B]
  static constexpr uint32_t kPair = kP + 2 * kSlice;                        // [2][128] fp32 + [2][128] flags
  static constexpr uint32_t kBar = kPair + 2 * kRowsM * 4 + 2 * kRowsM * 4;
  static constexpr int kNumBars = 1 + 2 * kKSlots + 2 * 2 + 2 * 2 + 2 + 1 + 2;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory");
};

__global__ void __launch_bounds__(kThreads, 1)
moba_past_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ counts,
                    const int32_t* __restrict__ offsets, const int32_t* __restrict__ chunks,
                    const int32_t* __restrict__ chunk_list, const int32_t* __restrict__ list,
                    __nv_bfloat16* __restrict__ part_o, float* __restrict__ part_lse, int T, int H, int nblk, int bsz,
                    int top_k, int E, float scale_log2, int* __restrict__ err) {
  using SM = Smem;
  const int total = chunks[E];
  if ((int)blockIdx.x >= total) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sP = smem + SM::kP;
  float* sPairMax = reinterpret_cast<float*>(smem + SM::kPair);            // [half][row]
  int* sPairFlag = reinterpret_cast<int*>(sPairMax + 2 * kRowsM);           // [half][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kKSlots;
  uint64_t* v_full = k_empty + kKSlots;
  uint64_t* v_empty = v_full + 2;
  uint64_t* s_full = v_empty + 2;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 1;
  uint64_t* o_full = p_empty + 1;
  uint64_t* q_empty = o_full + 1;   // the S MMAs of a chunk have read its queries
  uint64_t* o_empty = q_empty + 1;  // the softmax warps have read a chunk's O
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = bsz / kBlk;
  struct Chunk { int e, b, h, j, first, nq; };
  auto chunk_of = [&](int c) {
    Chunk x;
    x.e = chunk_list[c];   // the (b, h, j) list this chunk belongs to
    const int bh = x.e / nblk;
    x.j = x.e % nblk;
    x.b = bh / H;
    x.h = bh % H;
    x.first = (c - chunks[x.e]) * kRowsM;
    x.nq = min(kRowsM, counts[x.e] - x.first);
    return x;
  };

  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int i = 0; i < kKSlots; ++i) {
      tc::mbar_init(k_full + i, 1);
      tc::mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(v_full + i, 1);
      tc::mbar_init(v_empty + i, 1);
      tc::mbar_init(s_full + i, 1);
      tc::mbar_init(s_empty + i, kSoftWarps);
    }
    tc::mbar_init(p_full, kSoftWarps);
    tc::mbar_init(p_empty, 1);
    tc::mbar_init(o_full, 1);
    tc::mbar_init(q_empty, 1);
    tc::mbar_init(o_empty, kSoftWarps);
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
    // ------------------------------------------------------------ producer
    // Per chunk: gather its query rows (each lane four rows, cp.async into the K-major,
    // 128-byte-swizzled operand; zeros past the chunk's end) once the previous chunk's S
    // MMAs are done with the buffer, then stream the block's K/V tiles (lane 0, TMA).
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
    }
    int fill = 0, vcnt = 0, k = 0;
    bool ok = true;
    for (int c = blockIdx.x; c < total && ok; c += gridDim.x, ++k) {
      const Chunk x = chunk_of(c);
      if (k > 0) ok = __all_sync(0xffffffffu, tc::mbar_wait(q_empty, (k - 1) & 1, err, kErrQEmpty));
      if (!ok) break;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane + 32 * i;
        const int ent = r < x.nq ? list[offsets[x.e] + x.first + r] : -1;
        const __nv_bfloat16* src = q + (((size_t)x.b * T + (ent >= 0 ? (ent >> 3) : 0)) * H + x.h) * D;
#pragma unroll
        for (int ch = 0; ch < 16; ++ch)
          cp_async16(sQ + (ch >> 3) * kSlice + r * 128 + (((ch & 7) ^ (r & 7)) << 4), src + 8 * ch, ent >= 0);
      }
      cp_async_commit();
      cp_async_wait<0>();
      tc::fence_async_smem();   // the MMAs read these rows through the async proxy
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar_q);
      for (int n = 0; n < ntiles && ok; ++n) {
        const int row = x.b * T + x.j * bsz + n * kBlk;
        for (int s = 0; s < 2 && ok; ++s, ++fill) {
          const int slot = fill % kKSlots;
          ok = __all_sync(0xffffffffu, tc::mbar_wait(k_empty + slot, ((fill / kKSlots) & 1) ^ 1, err, kErrKEmpty));
          if (ok && lane == 0) {
            tc::mbar_expect_tx(k_full + slot, kSlice);
            tc::tma_load_3d(sK + slot * kSlice, &tm_k, k_full + slot, s * 64, x.h, row);
          }
        }
        if (!ok) break;
        const int vb = vcnt & 1;
        ok = __all_sync(0xffffffffu, tc::mbar_wait(v_empty + vb, ((vcnt >> 1) & 1) ^ 1, err, kErrVEmpty));
        if (ok && lane == 0) {
          tc::mbar_expect_tx(v_full + vb, 2 * kSlice);
          for (int s = 0; s < 2; ++s) tc::tma_load_3d(sV + (vb * 2 + s) * kSlice, &tm_v, v_full + vb, s * 64, x.h, row);
        }
        ++vcnt;
      }
    }
    if (lane == 0) {   // let the copies in flight land (bounded)
      for (int i = 0; i < kKSlots && i < fill; ++i) {
        const int f = fill - 1 - i;
        tc::mbar_drain(k_full + (f % kKSlots), (f / kKSlots) & 1);
      }
      for (int n = max(0, vcnt - 2); n < vcnt; ++n) tc::mbar_drain(v_full + (n & 1), (n >> 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);      // S = Q K^T  (both K-major)
      const uint32_t idPV = tc::idesc_bf16(128, D, 0, 1);       // O = P V    (P K-major, V MN-major)
      int fill = 0, use = 0, pc = 0, k = 0;
      bool ok = true;
      auto issue_s = [&]() -> bool {
        const int sb = use & 1;
        if (!tc::mbar_wait(s_empty + sb, ((use >> 1) & 1) ^ 1, err, kErrSEmpty)) return false;
        tc::tc_fence_after();
        for (int s = 0; s < 2; ++s, ++fill) {
          const int slot = fill % kKSlots;
          if (!tc::mbar_wait(k_full + slot, (fill / kKSlots) & 1, err, kErrKFull)) return false;
          tc::tc_fence_after();
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t dq = tc::sdesc(sQ + s * kSlice + ks * 32, 16, 1024);
            const uint64_t dk = tc::sdesc(sK + slot * kSlice + ks * 32, 16, 1024);
            tc::mma_ss(tmem + kColS + 128 * sb, dq, dk, idS, (s | ks) != 0);
          }
          tc::mma_commit(k_empty + slot);
        }
        tc::mma_commit(s_full + sb);
        ++use;
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        if (!tc::mbar_wait(p_full, pc & 1, err, kErrPFull) ||
            !tc::mbar_wait(v_full + (pc & 1), (pc >> 1) & 1, err, kErrVFull))
          return false;
        tc::tc_fence_after();
        const uint8_t* vb = sV + (pc & 1) * 2 * kSlice;
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          const uint64_t da = tc::sdesc(sP + (ks >> 2) * kSlice + (ks & 3) * 32, 16, 1024);
          const uint64_t db = tc::sdesc(vb + ks * 16 * 128, kSlice, 1024);
          tc::mma_ss(tmem + kColO, da, db, idPV, (n | ks) != 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(v_empty + (pc & 1));
        ++pc;
        return true;
      };
      for (int c = blockIdx.x; c < total && ok; c += gridDim.x, ++k) {
        ok = tc::mbar_wait(bar_q, k & 1, err, kErrQ);
        if (!ok) break;
        tc::tc_fence_after();
        ok = issue_s();
        if (ok && ntiles == 1) tc::mma_commit(q_empty);
        // O is overwritten (and o_full committed) only after the previous chunk's epilogue read it
        if (ok && k > 0) ok = tc::mbar_wait(o_empty, (k - 1) & 1, err, kErrOEmpty);
        for (int n = 0; n < ntiles && ok; ++n) {
          if (n + 1 < ntiles) {
            ok = issue_s();
            if (ok && n + 2 == ntiles) tc::mma_commit(q_empty);   // the chunk's last S reads Q
          }
          if (ok) ok = issue_pv(n);
        }
        if (ok) tc::mma_commit(o_full);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int gr = warp >> 2, q4 = warp & 3;       // key half, TMEM lane quadrant
    const int r = 32 * q4 + lane;                  // this thread's query row
    const int pbar = 1 + q4;                       // barrier of the warp pair sharing these rows
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    bool ok = true;
    int use = 0, pc = 0, k = 0;
    for (int c = blockIdx.x; c < total; c += gridDim.x, ++k) {
      const Chunk x = chunk_of(c);
      // this row's list entry, read now for the epilogue (it is in L2: the producer read it)
      const int ent = r < x.nq ? list[offsets[x.e] + x.first + r] : -1;
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < ntiles; ++n, ++use, ++pc) {
        const int sb = use & 1;
        ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull));
        float v[64];
        if (ok) {
          tc::tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            tc::tmem_ld16(lane_addr + kColS + 128 * sb + 64 * gr + 16 * cc, *reinterpret_cast<float(*)[16]>(v + 16 * cc));
          tc::tmem_wait_ld();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(s_empty + sb);
        }
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) v[jj] *= scale_log2;
        float cmx[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) cmx[cc] = fmaxf(fmaxf(v[cc], v[cc + 8]), fmaxf(v[cc + 16], v[cc + 24]));
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          cmx[cc] = fmaxf(cmx[cc], fmaxf(fmaxf(v[cc + 32], v[cc + 40]), fmaxf(v[cc + 48], v[cc + 56])));
        const float lmax = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                                 fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7])));
        // the two threads of a row agree on its reference; a failed wait also takes the
        // exchange, so that both warps of the pair leave together
        if (tc::vote_any(pbar, 64, !ok || lmax > m + kSlack)) {
          sPairMax[gr * kRowsM + r] = lmax;
          sPairFlag[gr * kRowsM + r] = ok;
          tc::named_sync(pbar, 64);
          const bool pair_ok = __all_sync(0xffffffffu, sPairFlag[r] && sPairFlag[kRowsM + r]);
          if (!pair_ok) {
            ok = false;
            break;
          }
          const float mn = fmaxf(m, fmaxf(sPairMax[r], sPairMax[kRowsM + r]));
          const float cf = mn == -INFINITY ? 1.f : ex2(m - mn);
          l *= cf;
          if (__any_sync(0xffffffffu, cf != 1.f) && n > 0) {
            // rescale this thread's half of the row's O once the previous P.V has finished
            ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (pc - 1) & 1, err, kErrPEmpty));
            if (ok) {
              tc::tc_fence_after();
#pragma unroll
              for (int qq = 0; qq < D / 2 / 16; ++qq) {
                float o[16];
                const uint32_t addr = lane_addr + kColO + (D / 2) * gr + 16 * qq;
                tc::tmem_ld16(addr, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] *= cf;
                tc::tmem_st16(addr, o);
              }
              tc::tmem_wait_st();
              tc::tc_fence_before();
            }
          }
          m = mn;
          tc::named_sync(pbar, 64);   // both halves have read the exchange before it is reused
        }
        const float base = m == -INFINITY ? 0.f : m;
        uint32_t pk[32];
        float ps[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) ps[cc] = 0.f;
#pragma unroll
        for (int jj = 0; jj < 64; jj += 2) {
          const float p0 = ex2(v[jj] - base), p1 = ex2(v[jj + 1] - base);
          ps[(jj >> 1) & 7] += p0 + p1;
          pk[jj / 2] = pack_bf16(p0, p1);
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        // P(pc) overwrites the buffer once P.V(pc-1) has read it
        if (pc > 0) ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(p_empty, (pc - 1) & 1, err, kErrPEmpty));
        uint8_t* prow = sP + gr * kSlice + r * 128;     // row r, keys of this half: K-major, 128-byte swizzle
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(p_full);
      }
      // epilogue: the row sum over both halves, then part_o = bf16(O / l), part_lse = m + log2(l)
      sPairMax[gr * kRowsM + r] = l;
      sPairFlag[gr * kRowsM + r] = ok;
      tc::named_sync(pbar, 64);
      const bool pair_ok = sPairFlag[r] && sPairFlag[kRowsM + r];
      const float L = sPairMax[r] + sPairMax[kRowsM + r];
      tc::named_sync(pbar, 64);   // both halves have read the sums before the next chunk reuses them
      ok = tc::vote_all(5, 32 * kSoftWarps, pair_ok && tc::mbar_wait(o_full, k & 1, err, kErrOFull));
      if (!ok) break;
      tc::tc_fence_after();
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const size_t base = ent >= 0 ? (((size_t)x.b * T + (ent >> 3)) * H + x.h) * top_k + (ent & 7) : 0;
      __nv_bfloat16* orow = part_o + base * D + (D / 2) * gr;
      float o[D / 2];
#pragma unroll
      for (int qq = 0; qq < D / 2 / 16; ++qq)
        tc::tmem_ld16(lane_addr + kColO + (D / 2) * gr + 16 * qq, *reinterpret_cast<float(*)[16]>(o + 16 * qq));
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty);
      if (ent >= 0) {
#pragma unroll
        for (int qq = 0; qq < D / 2 / 16; ++qq) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = pack_bf16(o[16 * qq + 2 * i] * inv, o[16 * qq + 2 * i + 1] * inv);
          *reinterpret_cast<uint4*>(orow + 16 * qq) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(orow + 16 * qq + 8) = make_uint4(w[4], w[5], w[6], w[7]);
        }
        if (gr == 0) part_lse[base] = m + __log2f(L);
      }
    }
  }

  tc::settle_after_error(err);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace

namespace {
// Own block + merge on tcgen05 ("逐篇讲解…" §16: every query also attends, causally, to the
// block it sits in).  One CTA = 128 consecutive queries of one head (TMEM lane = query),
// keys from the own block's start to the CTA's last query in 128-key tiles, masked to u <= t;
// the same TMA / MMA / softmax roles and lazy reference as the past-block kernel.  Epilogue:
// the own-block state (O unnormalised against the reference m, row sum l) merged with the
// query's past-block partials by their log-sum-exps; out in bf16.  Each softmax thread asks
// L2 for its half rows of those partials when it starts, so that the merge does not wait for
// DRAM.
__global__ void __launch_bounds__(kThreads, 1)
moba_own_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const int32_t* __restrict__ idx,
                   const __nv_bfloat16* __restrict__ part_o, const float* __restrict__ part_lse,
                   __nv_bfloat16* __restrict__ out, int T, int H, int bsz, int top_k, float scale_log2,
                   int* __restrict__ err) {
  using SM = Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sP = smem + SM::kP;
  float* sPairMax = reinterpret_cast<float*>(smem + SM::kPair);            // [half][row]
  int* sPairFlag = reinterpret_cast<int*>(sPairMax + 2 * kRowsM);           // [half][row]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kKSlots;
  uint64_t* v_full = k_empty + kKSlots;
  uint64_t* v_empty = v_full + 2;
  uint64_t* s_full = v_empty + 2;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* p_empty = p_full + 1;
  uint64_t* o_full = p_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * kRowsM, h = blockIdx.y, b = blockIdx.z;
  const int J = t0 / bsz, u0 = J * bsz;            // the own block (bsz % 128 == 0)
  const int t_last = min(T - 1, t0 + kRowsM - 1);
  const int ntiles = (t_last - u0) / kBlk + 1;

  if (tid == 0) {
    tc::mbar_init(bar_q, 1);
    for (int i = 0; i < kKSlots; ++i) {
      tc::mbar_init(k_full + i, 1);
      tc::mbar_init(k_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(v_full + i, 1);
      tc::mbar_init(v_empty + i, 1);
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
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      tc::mbar_expect_tx(bar_q, 2 * kSlice);
      for (int s = 0; s < 2; ++s) tc::tma_load_3d(sQ + s * kSlice, &tm_q, bar_q, s * 64, h, b * T + t0);
      int fill = 0;
      bool ok = true;
      for (int n = 0; n < ntiles && ok; ++n) {
        const int row = b * T + u0 + n * kBlk;
        for (int s = 0; s < 2 && ok; ++s, ++fill) {
          const int slot = fill % kKSlots;
          ok = tc::mbar_wait(k_empty + slot, ((fill / kKSlots) & 1) ^ 1, err, kErrKEmpty);
          if (!ok) break;
          tc::mbar_expect_tx(k_full + slot, kSlice);
          tc::tma_load_3d(sK + slot * kSlice, &tm_k, k_full + slot, s * 64, h, row);
        }
        if (!ok) break;
        const int vb = n & 1;
        ok = tc::mbar_wait(v_empty + vb, ((n >> 1) & 1) ^ 1, err, kErrVEmpty);
        if (!ok) break;
        tc::mbar_expect_tx(v_full + vb, 2 * kSlice);
        for (int s = 0; s < 2; ++s) tc::tma_load_3d(sV + (vb * 2 + s) * kSlice, &tm_v, v_full + vb, s * 64, h, row);
      }
      for (int i = 0; i < kKSlots && i < fill; ++i) {   // let the copies in flight land (bounded)
        const int f = fill - 1 - i;
        tc::mbar_drain(k_full + (f % kKSlots), (f / kKSlots) & 1);
      }
      for (int n = max(0, ntiles - 2); n < ntiles; ++n) tc::mbar_drain(v_full + (n & 1), (n >> 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);
      const uint32_t idPV = tc::idesc_bf16(128, D, 0, 1);
      bool ok = tc::mbar_wait(bar_q, 0, err, kErrQ);
      tc::tc_fence_after();
      int fill = 0;
      auto issue_s = [&](int n) -> bool {
        const int sb = n & 1;
        if (!tc::mbar_wait(s_empty + sb, ((n >> 1) & 1) ^ 1, err, kErrSEmpty)) return false;
        tc::tc_fence_after();
        for (int s = 0; s < 2; ++s, ++fill) {
          const int slot = fill % kKSlots;
          if (!tc::mbar_wait(k_full + slot, (fill / kKSlots) & 1, err, kErrKFull)) return false;
          tc::tc_fence_after();
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t dq = tc::sdesc(sQ + s * kSlice + ks * 32, 16, 1024);
            const uint64_t dk = tc::sdesc(sK + slot * kSlice + ks * 32, 16, 1024);
            tc::mma_ss(tmem + kColS + 128 * sb, dq, dk, idS, (s | ks) != 0);
          }
          tc::mma_commit(k_empty + slot);
        }
        tc::mma_commit(s_full + sb);
        return true;
      };
      auto issue_pv = [&](int n) -> bool {
        if (!tc::mbar_wait(p_full, n & 1, err, kErrPFull) ||
            !tc::mbar_wait(v_full + (n & 1), (n >> 1) & 1, err, kErrVFull))
          return false;
        tc::tc_fence_after();
        const uint8_t* vb = sV + (n & 1) * 2 * kSlice;
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          const uint64_t da = tc::sdesc(sP + (ks >> 2) * kSlice + (ks & 3) * 32, 16, 1024);
          const uint64_t db = tc::sdesc(vb + ks * 16 * 128, kSlice, 1024);
          tc::mma_ss(tmem + kColO, da, db, idPV, (n | ks) != 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(v_empty + (n & 1));
        return true;
      };
      if (ok && ntiles > 0) ok = issue_s(0);
      for (int n = 0; n < ntiles && ok; ++n) {
        if (n + 1 < ntiles) ok = issue_s(n + 1);
        if (ok) ok = issue_pv(n);
      }
      if (ok && ntiles > 0) tc::mma_commit(o_full);
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    const int gr = warp >> 2, q4 = warp & 3;       // key half, TMEM lane quadrant
    const int r = 32 * q4 + lane;                  // this thread's query: token t0 + r
    const int pbar = 1 + q4;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    const int t = t0 + r;
    const bool row_ok = t < T;
    const int my_hi = row_ok ? t : -1;             // keys [u0, my_hi]
    // the past-block partials this query merges in: their slots and log-sum-exps, read now
    const int32_t* irow = idx + (((size_t)b * H + h) * T + (row_ok ? t : 0)) * (top_k + 1);
    float plse[kMaxPast];
    int np = 0;
#pragma unroll
    for (int sl = 0; sl < kMaxPast; ++sl) {
      const int jj = (row_ok && sl < top_k) ? irow[sl] : -1;
      const bool in = jj >= 0 && jj < J && sl == np;
      plse[sl] = in ? part_lse[(((size_t)b * T + t) * H + h) * top_k + sl] : -INFINITY;
      np += in ? 1 : 0;
    }
    {   // this thread's half rows of those partials (one 128-byte line each) on their way to L2
        // while the own block's tiles run: the epilogue reads them after its O is complete
      const __nv_bfloat16* po = part_o + (((size_t)b * T + (row_ok ? t : 0)) * H + h) * top_k * D + (D / 2) * gr;
#pragma unroll
      for (int sl = 0; sl < kMaxPast; ++sl)
        if (sl < np) prefetch_l2(po + sl * D);
    }
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int sb = n & 1;
      ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(s_full + sb, (n >> 1) & 1, err, kErrSFull));
      float v[64];
      if (ok) {
        tc::tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          tc::tmem_ld16(lane_addr + kColS + 128 * sb + 64 * gr + 16 * cc, *reinterpret_cast<float(*)[16]>(v + 16 * cc));
        tc::tmem_wait_ld();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(s_empty + sb);
      }
      const int i0 = u0 + n * kBlk + 64 * gr;     // first key of this thread's half
      if (i0 + 63 <= my_hi) {
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) v[jj] *= scale_log2;
      } else {
#pragma unroll
        for (int jj = 0; jj < 64; ++jj) v[jj] = i0 + jj <= my_hi ? v[jj] * scale_log2 : -INFINITY;
      }
      float cmx[8];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) cmx[cc] = fmaxf(fmaxf(v[cc], v[cc + 8]), fmaxf(v[cc + 16], v[cc + 24]));
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        cmx[cc] = fmaxf(cmx[cc], fmaxf(fmaxf(v[cc + 32], v[cc + 40]), fmaxf(v[cc + 48], v[cc + 56])));
      const float lmax = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                               fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7])));
      if (tc::vote_any(pbar, 64, !ok || lmax > m + kSlack)) {
        sPairMax[gr * kRowsM + r] = lmax;
        sPairFlag[gr * kRowsM + r] = ok;
        tc::named_sync(pbar, 64);
        const bool pair_ok = __all_sync(0xffffffffu, sPairFlag[r] && sPairFlag[kRowsM + r]);
        if (!pair_ok) {
          ok = false;
          break;
        }
        const float mn = fmaxf(m, fmaxf(sPairMax[r], sPairMax[kRowsM + r]));
        const float cf = mn == -INFINITY ? 1.f : ex2(m - mn);
        l *= cf;
        if (__any_sync(0xffffffffu, cf != 1.f) && n > 0) {
          ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (n - 1) & 1, err, kErrPEmpty));
          if (ok) {
            tc::tc_fence_after();
#pragma unroll
            for (int qq = 0; qq < D / 2 / 16; ++qq) {
              float o[16];
              const uint32_t addr = lane_addr + kColO + (D / 2) * gr + 16 * qq;
              tc::tmem_ld16(addr, o);
              tc::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] *= cf;
              tc::tmem_st16(addr, o);
            }
            tc::tmem_wait_st();
            tc::tc_fence_before();
          }
        }
        m = mn;
        tc::named_sync(pbar, 64);
      }
      const float base = m == -INFINITY ? 0.f : m;
      uint32_t pk[32];
      float ps[8];
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) ps[cc] = 0.f;
#pragma unroll
      for (int jj = 0; jj < 64; jj += 2) {
        const float p0 = ex2(v[jj] - base), p1 = ex2(v[jj + 1] - base);
        ps[(jj >> 1) & 7] += p0 + p1;
        pk[jj / 2] = pack_bf16(p0, p1);
      }
      l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      if (n > 0) ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(p_empty, (n - 1) & 1, err, kErrPEmpty));
      uint8_t* prow = sP + gr * kSlice + r * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
      tc::fence_async_smem();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(p_full);
    }
    // epilogue: the own block's (m, L, O) merged with the past partials
    sPairMax[gr * kRowsM + r] = l;
    sPairFlag[gr * kRowsM + r] = ok;
    tc::named_sync(pbar, 64);
    const bool pair_ok = sPairFlag[r] && sPairFlag[kRowsM + r];
    const float L = sPairMax[r] + sPairMax[kRowsM + r];
    ok = __all_sync(0xffffffffu, pair_ok && (ntiles == 0 || tc::mbar_wait(o_full, 0, err, kErrOFull)));
    if (ok) {
      tc::tc_fence_after();
      float M = m + __log2f(L);                      // the own block's log-sum-exp (L >= 1: key t is visible)
#pragma unroll
      for (int sl = 0; sl < kMaxPast; ++sl) M = fmaxf(M, plse[sl]);
      const float w_own = ex2(m - M);               // multiplies the unnormalised O (row sum L)
      float wsum = L * w_own;
      float ws[kMaxPast];
#pragma unroll
      for (int sl = 0; sl < kMaxPast; ++sl) {
        ws[sl] = sl < np ? ex2(plse[sl] - M) : 0.f;
        wsum += ws[sl];
      }
      const float inv = row_ok && wsum > 0.f ? 1.f / wsum : 0.f;
      const size_t qrow = ((size_t)b * T + (row_ok ? t : 0)) * H + h;
      const __nv_bfloat16* po = part_o + qrow * top_k * D + (D / 2) * gr;
      __nv_bfloat16* orow = out + qrow * D + (D / 2) * gr;
#pragma unroll
      for (int qq = 0; qq < D / 2 / 16; ++qq) {
        float o[16];
        tc::tmem_ld16(lane_addr + kColO + (D / 2) * gr + 16 * qq, o);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] *= w_own;
#pragma unroll
        for (int sl = 0; sl < kMaxPast; ++sl) {
          if (sl < np) {
            const uint4* src = reinterpret_cast<const uint4*>(po + sl * D + 16 * qq);
            const uint4 a0 = src[0], a1 = src[1];
            const uint32_t wv[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
              o[2 * i] += ws[sl] * f.x;
              o[2 * i + 1] += ws[sl] * f.y;
            }
          }
        }
        if (row_ok) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w[i] = pack_bf16(o[2 * i] * inv, o[2 * i + 1] * inv);
          *reinterpret_cast<uint4*>(orow + 16 * qq) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(orow + 16 * qq + 8) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    }
  }

  tc::settle_after_error(err);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace

cudaError_t launch_moba_own_tc(const MobaArgs& a, const int32_t* idx, const __nv_bfloat16* part_o,
                               const float* part_lse, cudaStream_t st) {
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(moba_own_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  CUtensorMap mq, mk, mv;
  const uint64_t d3[3] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.B * a.T};
  const uint64_t s3[2] = {(uint64_t)D * 2, (uint64_t)a.H * D * 2};
  const uint32_t box[3] = {64, 1, (uint32_t)kBlk};
  if (!make_tmap_bf16(&mq, a.q, 3, d3, s3, box) || !make_tmap_bf16(&mk, a.k, 3, d3, s3, box) ||
      !make_tmap_bf16(&mv, a.v, 3, d3, s3, box))
    return cudaErrorInvalidValue;
  dim3 grid((a.T + kRowsM - 1) / kRowsM, a.H, a.B);
  moba_own_tc_kernel<<<grid, kThreads, Smem::kAlloc, st>>>(mq, mk, mv, idx, part_o, part_lse,
                                                            static_cast<__nv_bfloat16*>(a.out), a.T, a.H, a.bsz,
                                                            a.top_k, a.scale_log2, a.err);
  return cudaGetLastError();
}

bool moba_past_tc_supported(const MobaArgs& a) {
  return a.err != nullptr && a.bsz % kBlk == 0 && a.top_k > 0 && a.top_k <= 8;
}

int moba_past_tc_chunk() { return kRowsM; }

cudaError_t launch_moba_past_tc(const MobaArgs& a, const int32_t* counts, const int32_t* offsets,
                                const int32_t* chunks, const int32_t* chunk_list, const int32_t* list,
                                __nv_bfloat16* part_o, float* part_lse, int nblk, int E, size_t max_chunks,
                                cudaStream_t st) {
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(moba_past_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Smem::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  if (max_chunks == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  const uint64_t d3[3] = {(uint64_t)D, (uint64_t)a.H, (uint64_t)a.B * a.T};
  const uint64_t s3[2] = {(uint64_t)D * 2, (uint64_t)a.H * D * 2};
  const uint32_t box[3] = {64, 1, (uint32_t)kBlk};
  if (!make_tmap_bf16(&mk, a.k, 3, d3, s3, box) || !make_tmap_bf16(&mv, a.v, 3, d3, s3, box))
    return cudaErrorInvalidValue;
  const int sms = sm_count();
  const unsigned grid = (unsigned)std::min<size_t>(max_chunks, (size_t)sms);
  moba_past_tc_kernel<<<grid, kThreads, Smem::kAlloc, st>>>(
      mk, mv, static_cast<const __nv_bfloat16*>(a.q), counts, offsets, chunks, chunk_list, list, part_o, part_lse, a.T,
      a.H, nblk,
      a.bsz, a.top_k, E, a.scale_log2, a.err);
  return cudaGetLastError();
}

}  // namespace nsa
