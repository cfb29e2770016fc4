// K4 + K5 on the fifth-generation tensor cores, in one pass: the sliding-window branch
// and the gated combine ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5: the third
// branch attends to the neighbouring tokens; §6: each branch output is scaled by a gate
// from the current token and the three are added).
//
// Persistent: one CTA per SM walks the items, an item = 8 consecutive tokens x the group's
// 16 heads = 128 query rows (one TMEM lane each), over the union of their windows,
// [t0 - w + 1, t0 + 7], in tiles of 128 tokens:
//   S = Q K^T        (M = 128 rows, N = 128 keys; two TMEM buffers)
//   O += P V         (M = 128 rows, N = d_v; P in SMEM as the K-major A operand)
// Warp roles: a TMA producer (each item's Q once the previous item's S MMAs have read the
// buffer, K slices into a 3-slot ring, V tiles double buffered; the rings run across items),
// a single-thread MMA issuer that puts S(n+1) ahead of the P.V of tile n and accumulates
// alternate items into two O buffers in TMEM (so an item's tiles overlap the previous
// item's epilogue), 8 softmax warps: warp w and warp w+4 share TMEM lanes 32(w%4).. (the
// same rows) and take the tile's key columns [0, 64) and [64, 128); and 4 epilogue warps
// (one per TMEM lane quadrant) that write an item's rows while the softmax warps run the
// next item's tiles.
//
// Softmax in one pass: a row's reference m moves only when a score exceeds it by more
// than 2^8 (so p <= 2^8).  The two threads of a row agree on it through one barrier of
// the warp pair per tile; when it moves, each rescales its half of the row's O in TMEM
// once the previous P.V has finished.  Epilogue: out = bf16(acc + g_win * O / l).
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int kSoftWarps = 8;
constexpr int kTmaWarp = 8, kMmaWarp = 9, kEpiWarp0 = 10;   // epilogue: warps 10-13
constexpr int kThreads = 448;
constexpr int kTok = 8;
constexpr int kRowsM = 128;
constexpr int kBlk = 128;                         // keys per tile
constexpr int kKSlots = 3;
constexpr uint32_t kSlice = kBlk * 128;           // 128 rows x 64 columns: 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;        // S buffer b at 128b; O buffer b at 256 + 128b
constexpr float kSlack = 8.f;

enum Err { kErrQ = 41, kErrKFull, kErrKEmpty, kErrVFull, kErrVEmpty, kErrSFull, kErrSEmpty, kErrPFull, kErrPEmpty,
           kErrOFull, kErrOEmpty, kErrQEmpty, kErrLFull, kErrLEmpty };

template <int DK, int DV>
struct Smem {
  static constexpr int kQSlices = DK / 64, kVSlices = DV / 64;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kQSlices * kSlice;                    // ring of 64-column K slices
  static constexpr uint32_t kV = kK + kKSlots * kSlice;                     // 2 tiles x kVSlices slices
  static constexpr uint32_t kP = kV + 2 * kVSlices * kSlice;                // P: [2 key halves][128 rows][128 B]
  static constexpr uint32_t kPair = kP + 2 * kSlice;                        // [2][128] fp32 + [2][128] flags
  static constexpr uint32_t kL = kPair + 2 * kRowsM * 4 + 2 * kRowsM * 4;   // row sums: [item parity][128]
  static constexpr uint32_t kBar = kL + 2 * kRowsM * 4;
  static constexpr int kNumBars = 1 + 2 * kKSlots + 2 * 2 + 2 * 2 + 2 + 2 + 2 + 1 + 2 + 2;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory");
};

// VARLEN: a packed batch of sequences of different lengths (cu); its own instantiation, so
// that the equal-length one keeps its plain row arithmetic.
template <int DK, int DV, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
window_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ gates,
                 const float* __restrict__ acc, __nv_bfloat16* __restrict__ out, int B, int T, int Hq, int Hkv,
                 int window, float scale_log2, const int32_t* __restrict__ cu_in, int* __restrict__ err) {
  using SM = Smem<DK, DV>;
  const int32_t* cu = VARLEN ? cu_in : nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sP = smem + SM::kP;
  float* sPairMax = reinterpret_cast<float*>(smem + SM::kPair);            // [half][row]
  int* sPairFlag = reinterpret_cast<int*>(sPairMax + 2 * kRowsM);           // [half][row]
  float* sL = reinterpret_cast<float*>(smem + SM::kL);                      // [item parity][row]
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
  uint64_t* o_full = p_empty + 1;    // [2] an item's O (buffer k & 1) is complete
  uint64_t* o_empty = o_full + 2;    // [2] the epilogue warps have read it
  uint64_t* q_empty = o_empty + 2;   // the S MMAs of an item have read its Q
  uint64_t* l_full = q_empty + 1;    // [2] an item's row sums are in sL
  uint64_t* l_empty = l_full + 2;    // [2] the epilogue warps have read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tok_tiles = (T + kTok - 1) / kTok;
  const int n_items = n_tok_tiles * Hkv * B;
  // item -> (token tile, group, batch), the latest tokens first (all items but the first
  // few have the same number of key tiles).  In a variable-length batch, tiles past a
  // sequence's end are no items: every role skips them alike.
  struct Item { int t0, g, b, kv_lo, ntiles, base, len; };
  auto item_of = [&](int it) {
    Item x;
    x.g = it % Hkv;
    x.b = (it / Hkv) % B;
    x.t0 = (n_tok_tiles - 1 - it / (Hkv * B)) * kTok;
    x.base = seq_base(cu, x.b, T);   // first row of the sequence in q, k, v, gates, acc, out
    x.len = seq_len(cu, x.b, T);
    const int t_last = min(x.t0 + kTok - 1, x.len - 1);
    x.kv_lo = max(0, x.t0 - window + 1);
    x.ntiles = (t_last - x.kv_lo + kBlk) / kBlk;   // >= 1
    return x;
  };
  auto next_item = [&](int it) {   // the first item >= it of this CTA's stride that has tokens
    if (cu)
      while (it < n_items && (n_tok_tiles - 1 - it / (Hkv * B)) * kTok >= seq_len(cu, (it / Hkv) % B, T))
        it += gridDim.x;
    return it;
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
      tc::mbar_init(o_full + i, 1);
      tc::mbar_init(o_empty + i, 4);
      tc::mbar_init(l_full + i, 4);   // the four warps of the first key half
      tc::mbar_init(l_empty + i, 4);
    }
    tc::mbar_init(p_full, kSoftWarps);
    tc::mbar_init(p_empty, 1);
    tc::mbar_init(q_empty, 1);
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
    // Per item: Q once the previous item's S MMAs are done with it, then the K slices
    // and V tiles; the rings run across item boundaries.
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      int fill = 0, vcnt = 0, k = 0;
      bool ok = true;
      for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
        const Item x = item_of(it);
        if (k > 0) ok = tc::mbar_wait(q_empty, (k - 1) & 1, err, kErrQEmpty);
        if (!ok) break;
        tc::mbar_expect_tx(bar_q, SM::kQSlices * kSlice);
        for (int s = 0; s < SM::kQSlices; ++s)
          tc::tma_load_3d(sQ + s * kSlice, &tm_q, bar_q, s * 64, x.g * 16, x.base + x.t0);
        for (int n = 0; n < x.ntiles && ok; ++n) {
          const int row = x.base + x.kv_lo + n * kBlk;
          for (int s = 0; s < SM::kQSlices && ok; ++s, ++fill) {
            const int slot = fill % kKSlots;
            ok = tc::mbar_wait(k_empty + slot, ((fill / kKSlots) & 1) ^ 1, err, kErrKEmpty);
            if (!ok) break;
            tc::mbar_expect_tx(k_full + slot, kSlice);
            tc::tma_load_3d(sK + slot * kSlice, &tm_k, k_full + slot, s * 64, x.g, row);
          }
          if (!ok) break;
          const int vb = vcnt & 1;
          ok = tc::mbar_wait(v_empty + vb, ((vcnt >> 1) & 1) ^ 1, err, kErrVEmpty);
          if (!ok) break;
          tc::mbar_expect_tx(v_full + vb, SM::kVSlices * kSlice);
          for (int s = 0; s < SM::kVSlices; ++s)
            tc::tma_load_3d(sV + (vb * SM::kVSlices + s) * kSlice, &tm_v, v_full + vb, s * 64, x.g, row);
          ++vcnt;
        }
      }
      // let the copies in flight land (bounded)
      for (int i = 0; i < kKSlots && i < fill; ++i) {
        const int f = fill - 1 - i;
        tc::mbar_drain(k_full + (f % kKSlots), (f / kKSlots) & 1);
      }
      for (int n = max(0, vcnt - 2); n < vcnt; ++n) tc::mbar_drain(v_full + (n & 1), (n >> 1) & 1);
      if (k > 0) tc::mbar_drain(bar_q, (k - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idS = tc::idesc_bf16(128, 128, 0, 0);      // S = Q K^T  (both K-major)
      const uint32_t idPV = tc::idesc_bf16(128, DV, 0, 1);      // O = P V    (P K-major, V MN-major)
      int fill = 0, use = 0, pc = 0, k = 0;
      bool ok = true;
      auto issue_s = [&]() -> bool {
        const int sb = use & 1;
        if (!tc::mbar_wait(s_empty + sb, ((use >> 1) & 1) ^ 1, err, kErrSEmpty)) return false;
        tc::tc_fence_after();
        for (int s = 0; s < SM::kQSlices; ++s, ++fill) {
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
      auto issue_pv = [&](int n, uint32_t o_col) -> bool {
        if (!tc::mbar_wait(p_full, pc & 1, err, kErrPFull) ||
            !tc::mbar_wait(v_full + (pc & 1), (pc >> 1) & 1, err, kErrVFull))
          return false;
        tc::tc_fence_after();
        const uint8_t* vb = sV + (pc & 1) * SM::kVSlices * kSlice;
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          const uint64_t da = tc::sdesc(sP + (ks >> 2) * kSlice + (ks & 3) * 32, 16, 1024);
          const uint64_t db = tc::sdesc(vb + ks * 16 * 128, kSlice, 1024);
          tc::mma_ss(tmem + o_col, da, db, idPV, (n | ks) != 0);
        }
        tc::mma_commit(p_empty);
        tc::mma_commit(v_empty + (pc & 1));
        ++pc;
        return true;
      };
      for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
        const Item x = item_of(it);
        const int ob = k & 1;
        const uint32_t o_col = kColO + 128 * ob;
        ok = tc::mbar_wait(bar_q, k & 1, err, kErrQ);
        if (!ok) break;
        tc::tc_fence_after();
        ok = issue_s();
        if (ok && x.ntiles == 1) tc::mma_commit(q_empty);
        // O buffer ob is overwritten only after the epilogue of item k - 2 read it
        if (ok) ok = tc::mbar_wait(o_empty + ob, ((k >> 1) & 1) ^ 1, err, kErrOEmpty);
        for (int n = 0; n < x.ntiles && ok; ++n) {
          if (n + 1 < x.ntiles) {
            ok = issue_s();
            if (ok && n + 2 == x.ntiles) tc::mma_commit(q_empty);   // the item's last S reads Q
          }
          if (ok) ok = issue_pv(n, o_col);
        }
        if (ok) tc::mma_commit(o_full + ob);
      }
    }
  } else if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax
    const int gr = warp >> 2, q4 = warp & 3;       // key half, TMEM lane quadrant
    const int r = 32 * q4 + lane;                  // this thread's row: token r / 16, head r % 16
    const int pbar = 1 + q4;                       // barrier of the warp pair sharing these rows
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    bool ok = true;
    int use = 0, pc = 0, k = 0;
    for (int it = next_item(blockIdx.x); it < n_items; it = next_item(it + gridDim.x), ++k) {
      const Item x = item_of(it);
      const int ob = k & 1;
      const uint32_t o_col = kColO + 128 * ob;
      const int my_t = x.t0 + r / 16;
      const bool row_ok = my_t < x.len;
      const int my_lo = max(0, my_t - window + 1), my_hi = row_ok ? my_t : -1;   // keys [my_lo, my_hi]
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < x.ntiles; ++n, ++use, ++pc) {
        const int sb = use & 1;
        ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull));
        const uint32_t s_addr = lane_addr + kColS + 128 * sb + 64 * gr;
        const int i0 = x.kv_lo + n * kBlk + 64 * gr;     // first key of this thread's half
        const bool full = i0 >= my_lo && i0 + 63 <= my_hi;
        // the masked raw scores (the scale, positive, is applied to the maximum and inside the
        // exponent's FMA: rounding x * scale is monotone, so the maxima agree)
        float v[64];
        float lmax = -INFINITY;
        if (ok) {
          tc::tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) tc::tmem_ld16(s_addr + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
          tc::tmem_wait_ld();
          if (!full) {
#pragma unroll
            for (int j = 0; j < 64; ++j) v[j] = (i0 + j >= my_lo && i0 + j <= my_hi) ? v[j] : -INFINITY;
          }
          float cmx[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) cmx[c] = fmaxf(fmaxf(v[c], v[c + 8]), fmaxf(v[c + 16], v[c + 24]));
#pragma unroll
          for (int c = 0; c < 8; ++c) cmx[c] = fmaxf(cmx[c], fmaxf(fmaxf(v[c + 32], v[c + 40]), fmaxf(v[c + 48], v[c + 56])));
          lmax = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                       fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7]))) * scale_log2;
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) tc::mbar_arrive(s_empty + sb);
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
          const float c = mn == -INFINITY ? 1.f : ex2(m - mn);
          l *= c;
          if (__any_sync(0xffffffffu, c != 1.f) && n > 0) {
            // rescale this thread's half of the row's O once the previous P.V has finished
            ok = __all_sync(0xffffffffu, tc::mbar_wait(p_empty, (pc - 1) & 1, err, kErrPEmpty));
            if (ok) {
              tc::tc_fence_after();
#pragma unroll
              for (int q = 0; q < DV / 2 / 16; ++q) {
                float o[16];
                const uint32_t addr = lane_addr + o_col + (DV / 2) * gr + 16 * q;
                tc::tmem_ld16(addr, o);
                tc::tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] *= c;
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
        for (int c = 0; c < 8; ++c) ps[c] = 0.f;
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float p0 = ex2(fmaf(v[j], scale_log2, -base)), p1 = ex2(fmaf(v[j + 1], scale_log2, -base));
          ps[(j >> 1) & 7] += p0 + p1;
          pk[j / 2] = pack_bf16(p0, p1);
        }
        l += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        // P overwrites the buffer once the previous P.V (this item's or the last item's) has read it
        if (pc > 0) ok = __all_sync(0xffffffffu, ok && tc::mbar_wait(p_empty, (pc - 1) & 1, err, kErrPEmpty));
        uint8_t* prow = sP + gr * kSlice + r * 128;     // row r, keys of this half: K-major, 128-byte swizzle
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(p_full);
      }
      // the row sum over both halves, for the epilogue warps
      sPairMax[gr * kRowsM + r] = l;
      sPairFlag[gr * kRowsM + r] = ok;
      tc::named_sync(pbar, 64);
      const bool pair_ok = sPairFlag[r] && sPairFlag[kRowsM + r];
      const float L = sPairMax[r] + sPairMax[kRowsM + r];
      // all eight warps: both halves of every row have read the exchange before the next
      // item's first tile reuses it
      ok = tc::vote_all(5, 256, ok && pair_ok);
      if (!ok) break;
      if (gr == 0) {
        ok = __all_sync(0xffffffffu, tc::mbar_wait(l_empty + ob, ((k >> 1) & 1) ^ 1, err, kErrLEmpty));
        sL[ob * kRowsM + r] = L;
        __threadfence_block();
        __syncwarp();
        if (lane == 0 && ok) tc::mbar_arrive(l_full + ob);
      }
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue: out = bf16(acc + g_win * O / l)
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;                  // this thread's row: token r / 16, head r % 16
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    bool ok = true;
    int k = 0;
    for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
      const Item x = item_of(it);
      const int ob = k & 1;
      const uint32_t o_col = kColO + 128 * ob;
      const int my_t = x.t0 + r / 16;
      const bool row_ok = my_t < x.len;
      const size_t grow = ((size_t)x.base + min(my_t, x.len - 1)) * Hq + x.g * 16 + (r % 16);
      const float gw = row_ok ? __bfloat162float(gates[grow * 3 + 2]) : 0.f;
      const float* arow = acc + grow * DV;
      __nv_bfloat16* orow = out + grow * DV;
      // the accumulator row: its first half loaded (and the second asked of L2) while the
      // softmax warps still run the item's tiles
      float4 a4[DV / 2 / 4];
#pragma unroll
      for (int i = 0; i < DV / 2 / 4; ++i)
        a4[i] = row_ok ? *reinterpret_cast<const float4*>(arow + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
      if (row_ok) {
        prefetch_l2(arow + DV / 2);
        prefetch_l2(arow + DV / 2 + 32);
      }
      ok = __all_sync(0xffffffffu, tc::mbar_wait(l_full + ob, (k >> 1) & 1, err, kErrLFull));
      if (!ok) break;
      const float L = sL[ob * kRowsM + r];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(l_empty + ob);
      const float scl = L > 0.f ? gw / L : 0.f;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(o_full + ob, (k >> 1) & 1, err, kErrOFull));
      if (!ok) break;
      tc::tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        if (half == 1) {
#pragma unroll
          for (int i = 0; i < DV / 2 / 4; ++i)
            a4[i] = row_ok ? *reinterpret_cast<const float4*>(arow + DV / 2 + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < DV / 2 / 16; ++q) {
          float o[16];
          tc::tmem_ld16(lane_addr + o_col + (DV / 2) * half + 16 * q, o);
          tc::tmem_wait_ld();
          if (row_ok) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              const float4 av = a4[(16 * q + i) / 4];
              w[i / 2] = pack_bf16(av.x + scl * o[i], av.y + scl * o[i + 1]);
              w[i / 2 + 1] = pack_bf16(av.z + scl * o[i + 2], av.w + scl * o[i + 3]);
            }
            *reinterpret_cast<uint4*>(orow + (DV / 2) * half + 16 * q) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(orow + (DV / 2) * half + 16 * q + 8) = make_uint4(w[4], w[5], w[6], w[7]);
          }
        }
      }
      tc::tc_fence_before();   // this thread's reads of O buffer ob are done
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(o_empty + ob);
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

template <int DK, int DV>
cudaError_t launch_w(const FwdArgs& a, cudaStream_t st) {
  using SM = Smem<DK, DV>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(window_tc_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(window_tc_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SM::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  CUtensorMap mq, mk, mv;
  const uint64_t dq[3] = {(uint64_t)DK, (uint64_t)a.Hq, (uint64_t)a.total};
  const uint64_t sq[2] = {(uint64_t)DK * 2, (uint64_t)a.Hq * DK * 2};
  const uint32_t bq[3] = {64, 16, kTok};
  const uint64_t dk3[3] = {(uint64_t)DK, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sk3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hkv * DK * 2};
  const uint64_t dv3[3] = {(uint64_t)DV, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sv3[2] = {(uint64_t)DV * 2, (uint64_t)a.Hkv * DV * 2};
  const uint32_t bkv[3] = {64, 1, (uint32_t)kBlk};
  if (!make_tmap_bf16(&mq, a.q, 3, dq, sq, bq) || !make_tmap_bf16(&mk, a.k, 3, dk3, sk3, bkv) ||
      !make_tmap_bf16(&mv, a.v, 3, dv3, sv3, bkv))
    return cudaErrorInvalidValue;
  const int sms = sm_count();
  const long items = (long)((a.T + kTok - 1) / kTok) * a.Hkv * a.B;
  const int grid = (int)(items < sms ? items : sms);
  auto kernel = a.cu ? window_tc_kernel<DK, DV, true> : window_tc_kernel<DK, DV, false>;
  kernel<<<grid, kThreads, SM::kAlloc, st>>>(
      mq, mk, mv, static_cast<const __nv_bfloat16*>(a.gates), a.acc, static_cast<__nv_bfloat16*>(a.out), a.B, a.T,
      a.Hq, a.Hkv, a.window, a.scale_log2, a.cu, a.err);
  return cudaGetLastError();
}
}  // namespace

bool window_tc_supported(const FwdArgs& a) {
  return a.err != nullptr && a.G == 16 && a.dv == 128 && (a.dk == 128 || a.dk == 192) && a.window >= 1;
}

cudaError_t launch_window_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192 && a.dv == 128) return launch_w<192, 128>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch_w<128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
