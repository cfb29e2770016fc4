// K2 on the 5th-generation tensor cores: compressed attention + group-summed block scores +
// top-k ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5, §8; "一文比较 Kimi 和 Deepseek
// 的两篇稀疏注意力机制论文", "Deepseek 的论文核心点": the selection scores come from the
// compressed attention and the group's heads add them before one top-k).
//
// Persistent: one CTA per SM walks a static list of items, item = one KV group g and 8
// consecutive tokens (longest rows first).  An item's 128 query rows (token-major, 16 heads
// per token) are one tcgen05 M=128 tile held in shared memory.  The group's compressed
// keys/values stream through shared memory by TMA in tiles of 128 blocks.
//   pass A   S = Q Kc^T into TMEM (rows = (token, head)); each softmax thread keeps the
//            running max and sum of its row's 32 columns of every tile, and the four
//            groups' pairs are merged once per item -> log-sum-exp per row.
//   pass B   S^T = Kc Q^T into TMEM (rows = compressed blocks, columns = (token, head)):
//            each softmax thread owns one compressed block, forms the normalised
//            probabilities of its 128 columns, adds each token's 16 heads in registers
//            (the group sum), folds them into 64-token selection-block scores, and
//            writes P^T (bf16) to shared memory; O^T = Vc^T P^T accumulates in TMEM
//            (rows = value dims), already normalised, so no rescaling is ever needed.
//   top-k    per token over the selection-block scores: the top-k warps copy a finished
//            item's scores from shared memory into registers and select there.
//   epilogue acc[t, h, :] = g_cmp * o_cmp, read from O^T (each thread one value dim).
// Warp roles: 16 TMA producer, 17 MMA issuer (and TMEM owner), 18-19 top-k, 0-15 softmax /
// epilogue in four groups of four (warp w owns TMEM lanes 32*(w%4)..+31; group w/4 takes 32
// of every tile's 128 columns: in the second pass that is exactly two tokens).
// Items overlap: while the softmax warps finish an item (last tiles, epilogue), the TMA and
// MMA warps already load and multiply the next item's first tiles, and the top-k warps
// select the finished item's blocks while the softmax warps run the next item's pass A.
// Every wait is bounded (see tc.cuh); on a timeout the kernel records an error word, stops
// issuing work, and frees its TMEM.
#include <algorithm>
#include <cfloat>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int kSoftGroups = 4;                  // softmax warp groups, 32 tile columns each
constexpr int kSoftWarps = 4 * kSoftGroups;     // four warps per group (one per TMEM lane quarter)
constexpr int kCols = 128 / kSoftGroups;        // tile columns per softmax thread
constexpr int kTokG = kCols / 16;               // tokens per group in the second pass
constexpr int kTmaWarp = kSoftWarps, kMmaWarp = kSoftWarps + 1, kTopkWarp0 = kSoftWarps + 2, kTopkWarps = 2;
constexpr int kThreads = 32 * (kSoftWarps + 4);
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
           kErrPEmpty, kErrOFull, kErrQEmpty, kErrScFull, kErrScEmpty, kErrOEmpty };

template <int DK, int DV>
struct Smem {
  static constexpr int kQSlices = DK / 64, kVSlices = DV / 64;
  static constexpr uint32_t kQ = 0;                                         // Q: kQSlices x 16 KB
  static constexpr uint32_t kKc = kQ + kQSlices * kSlice;                   // Kc ring: kKcSlots x 16 KB
  static constexpr uint32_t kVc = kKc + kKcSlots * kSlice;                  // Vc: 2 buffers x kVSlices x 16 KB
  static constexpr uint32_t kP = kVc + 2 * kVSlices * kSlice;               // P^T: 2 x 16 KB (N = 128 rows)
  static constexpr uint32_t kScore = kP + 2 * kSlice;                       // [8][1024] fp32
  static constexpr uint32_t kLse = kScore + kTok * kMaxSel * 4;             // [128] fp32
  static constexpr uint32_t kGate = kLse + kRowsM * 4;                      // [2][128] fp32, by item parity
  static constexpr uint32_t kML = kP;                                       // [groups][128][2] fp32, while P^T is unused
  static constexpr uint32_t kBar = kGate + 2 * kRowsM * 4;                  // mbarriers
  static constexpr int kNumBars = 1 + 2 * kKcSlots + 2 * 2 + 2 * 2 + 2 + 1 + 4;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;                         // room to align the base to 1 KB
  static_assert(kAlloc <= 232448, "shared memory");
  static_assert(kLse % 16 == 0, "the log-sum-exp row is read as float4");
};


__device__ __forceinline__ int n_visible(int t, int nc) { return t < kL - 1 ? 0 : min(nc, (t - kL + 1) / kS + 1); }

using tc::named_sync;
using tc::vote_all;

// Top-k of NT tokens (one warp).  Phase 1 copies each token's scores score[k][0, nb_k) into
// registers as order-preserving integer keys (the scores are sums of probabilities, >= 0,
// so their bit patterns order like the values; key 0 marks "no candidate") and zeroes the
// entries for the next item, so the caller can release the score buffer right after it.
// Phase 2 selects per token: forced blocks 0 and the token's own block first, then the
// largest scores, ties to the lower block index; written in increasing block order to
// dst[k][0, top_k) with -1 padding.
template <int NT>
struct TopkWarp {
  uint32_t key[NT][32];
  uint32_t taken[NT];

  __device__ __forceinline__ void load(float* score, int stride, const int (&nb)[NT], const int (&own)[NT],
                                       int force_first, int force_local, int lane) {
#pragma unroll
    for (int k = 0; k < NT; ++k) {
      taken[k] = 0;
      if (nb[k] > 0) {
        if (force_first && lane == 0) taken[k] |= 1u;
        if (force_local && lane == (own[k] & 31)) taken[k] |= 1u << (own[k] >> 5);
      }
#pragma unroll
      for (int mm = 0; mm < 32; ++mm) {
        const int j = lane + 32 * mm;
        const bool in = j < nb[k];
        key[k][mm] = (in && !((taken[k] >> mm) & 1u)) ? __float_as_uint(score[k * stride + j]) + 1u : 0u;
        if (in) score[k * stride + j] = 0.f;
      }
    }
  }

  template <int K>
  __device__ __forceinline__ void select(int nb, int own, int top_k, int force_first, int force_local,
                                         int32_t* dst, int lane) {
    if (nb <= 0) return;
    if (nb <= top_k) {
      for (int j = lane; j < top_k; j += 32) dst[j] = j < nb ? j : -1;
      return;
    }
    int nforced = force_first ? 1 : 0;
    if (force_local && !(force_first && own == 0)) ++nforced;
    const int mmax = (nb + 31) >> 5;   // candidate slots in use per lane
    if (mmax <= 4) rounds<K, 4>(nforced, top_k, lane);
    else if (mmax <= 8) rounds<K, 8>(nforced, top_k, lane);
    else if (mmax <= 16) rounds<K, 16>(nforced, top_k, lane);
    else rounds<K, 32>(nforced, top_k, lane);
    int pos = 0;
    for (int mm = 0; mm < mmax; ++mm) {
      const bool sel = (taken[K] >> mm) & 1u;
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[pos + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * mm;
      pos += __popc(bal);
    }
    for (int j = pos + lane; j < top_k; j += 32) dst[j] = -1;
  }

  // The selection rounds over the first M slots of each lane (slots >= M hold no candidate).
  // The slots form groups of (up to) eight, each with its best key and slot kept in registers:
  // a lane's best is the best of its group bests, and when a lane's slot is taken only that
  // slot's group is scanned again.  Every comparison is strict, so equal keys keep the lowest
  // slot, and among lanes the lowest block index wins.
  template <int K, int M>
  __device__ __forceinline__ void rounds(int nforced, int top_k, int lane) {
    constexpr int GS = M < 8 ? M : 8;   // slots per group
    constexpr int NG = M / GS;          // groups
    uint32_t gk[NG];
    int gm[NG];
    // group G's best (G a compile-time constant, so that every slot index is one)
    auto group_best = [&](auto gc) {
      constexpr int G = decltype(gc)::value;
      uint32_t bk = key[K][G * GS];
      int bm = G * GS;
#pragma unroll
      for (int i = 1; i < GS; ++i)
        if (key[K][G * GS + i] > bk) {
          bk = key[K][G * GS + i];
          bm = G * GS + i;
        }
      gk[G] = bk;
      gm[G] = bm;
    };
    // the group of slot mw: clear the slot and scan the group again
    auto retake = [&](auto gc, int mw) {
      constexpr int G = decltype(gc)::value;
      if (mw / GS != G) return;
#pragma unroll
      for (int i = 0; i < GS; ++i)
        if (G * GS + i == mw) key[K][G * GS + i] = 0u;
      group_best(gc);
    };
    using G0 = std::integral_constant<int, 0>;
    using G1 = std::integral_constant<int, (NG > 1 ? 1 : 0)>;
    using G2 = std::integral_constant<int, (NG > 2 ? 2 : 0)>;
    using G3 = std::integral_constant<int, (NG > 3 ? 3 : 0)>;
    static_assert(NG <= 4, "at most 32 slots");
    group_best(G0{});
    if constexpr (NG > 1) group_best(G1{});
    if constexpr (NG > 2) group_best(G2{});
    if constexpr (NG > 3) group_best(G3{});
    for (int rr = nforced; rr < top_k; ++rr) {
      uint32_t bk = gk[0];
      int bm = gm[0];
#pragma unroll
      for (int g = 1; g < NG; ++g)
        if (gk[g] > bk) {
          bk = gk[g];
          bm = gm[g];
        }
      const uint32_t vmax = __reduce_max_sync(0xffffffffu, bk);
      if (vmax == 0u) break;
      // the lowest block index among the lanes holding the maximum
      const uint32_t jmin = __reduce_min_sync(0xffffffffu, bk == vmax ? (uint32_t)(lane + 32 * bm) : 0xffffffffu);
      if (lane == (int)(jmin & 31u)) {
        const int mw = (int)(jmin >> 5);
        taken[K] |= 1u << mw;
        retake(G0{}, mw);
        if constexpr (NG > 1) retake(G1{}, mw);
        if constexpr (NG > 2) retake(G2{}, mw);
        if constexpr (NG > 3) retake(G3{}, mw);
      }
    }
  }
};

// VARLEN: a packed batch of sequences of different lengths (cu); its own instantiation, so
// that the equal-length one keeps its plain row arithmetic.
template <int DK, int DV, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kc,
               const __grid_constant__ CUtensorMap tm_vc, const __nv_bfloat16* __restrict__ gates,
               float* __restrict__ acc, int32_t* __restrict__ idx_out, int B, int T, int Hq, int Hkv, int nc,
               int top_k, int force_first, int force_local, float scale_log2, float w_straddle,
               const int32_t* __restrict__ cu_in, int* __restrict__ err) {
  using SM = Smem<DK, DV>;
  const int32_t* cu = VARLEN ? cu_in : nullptr;
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
  uint64_t* q_empty = o_full + 1;    // the MMAs that read an item's Q have completed
  uint64_t* sc_full = q_empty + 1;   // an item's block scores are complete
  uint64_t* sc_empty = sc_full + 1;  // the top-k warps have read (and zeroed) them
  uint64_t* o_empty = sc_empty + 1;  // the softmax warps have read an item's O^T
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tok_tiles = (T + kTok - 1) / kTok;
  const int n_items = n_tok_tiles * Hkv * B;
  // item -> (token tile, group, batch); the longest rows come first.  In a variable-length
  // batch, tiles past a sequence's end are no items: every role skips them alike.
  struct Item { int t0, g, b, ntiles, base, len; };
  auto item_of = [&](int it) {
    Item x;
    x.g = it % Hkv;
    x.b = (it / Hkv) % B;
    x.t0 = (n_tok_tiles - 1 - it / (Hkv * B)) * kTok;
    x.base = seq_base(cu, x.b, T);   // first row of the sequence in q, gates and acc
    x.len = seq_len(cu, x.b, T);
    const int t_last = min(x.t0 + kTok - 1, x.len - 1);
    x.ntiles = (n_visible(t_last, nc) + kBlk - 1) / kBlk;
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
    tc::mbar_init(q_empty, 1);
    tc::mbar_init(sc_full, 1);
    tc::mbar_init(sc_empty, kTopkWarps);
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
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      tc::prefetch_tmap(&tm_q);
      tc::prefetch_tmap(&tm_kc);
      tc::prefetch_tmap(&tm_vc);
      int fill = 0;   // Kc slice fills so far (all items)
      int vcnt = 0;   // Vc tile fills so far
      bool ok = true;
      int k = 0;
      for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
        const Item x = item_of(it);
        // Q of this item once the previous item's S MMAs are done with the buffer
        if (k > 0) ok = tc::mbar_wait(q_empty, (k - 1) & 1, err, kErrQEmpty);
        if (!ok) break;
        tc::mbar_expect_tx(bar_q, SM::kQSlices * kSlice);
        for (int s = 0; s < SM::kQSlices; ++s)
          tc::tma_load_3d(sQ + s * kSlice, &tm_q, bar_q, s * 64, x.g * 16, x.base + x.t0);
        for (int pass = 0; pass < 2 && ok; ++pass) {
          for (int n = 0; n < x.ntiles && ok; ++n) {
            const int row = x.b * nc + n * kBlk;
            for (int s = 0; s < SM::kQSlices && ok; ++s, ++fill) {
              const int slot = fill % kKcSlots;
              ok = tc::mbar_wait(kc_empty + slot, ((fill / kKcSlots) & 1) ^ 1, err, kErrKcEmpty);
              if (!ok) break;
              tc::mbar_expect_tx(kc_full + slot, kSlice);
              tc::tma_load_3d(sKc + slot * kSlice, &tm_kc, kc_full + slot, s * 64, x.g, row);
            }
            if (pass == 1 && ok) {
              const int vb = vcnt & 1;
              ok = tc::mbar_wait(vc_empty + vb, ((vcnt >> 1) & 1) ^ 1, err, kErrVcEmpty);
              if (!ok) break;
              tc::mbar_expect_tx(vc_full + vb, SM::kVSlices * kSlice);
              for (int s = 0; s < SM::kVSlices; ++s)
                tc::tma_load_3d(sVc + (vb * SM::kVSlices + s) * kSlice, &tm_vc, vc_full + vb, s * 64, x.g, row);
              ++vcnt;
            }
          }
        }
      }
      // before leaving, let the copies still in flight land (bounded)
      for (int i = 0; i < kKcSlots && i < fill; ++i) {
        const int f = fill - 1 - i;
        tc::mbar_drain(kc_full + (f % kKcSlots), (f / kKcSlots) & 1);
      }
      for (int n = max(0, vcnt - 2); n < vcnt; ++n) tc::mbar_drain(vc_full + (n & 1), (n >> 1) & 1);
      if (k > 0) tc::mbar_drain(bar_q, (k - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      const uint32_t idA = tc::idesc_bf16(128, 128, 0, 0);     // S  = Q  Kc^T   (both K-major)
      const uint32_t idPV = tc::idesc_bf16(128, 128, 1, 1);    // O^T = Vc^T P^T (both MN-major)
      int use = 0;    // S buffer uses (all items, both passes)
      int fill = 0;   // Kc slices consumed
      int pc = 0;     // pass-B tiles (P^T phases, Vc tiles) so far
      bool ok = true;
      int k = 0;
      for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
        const Item x = item_of(it);
        ok = tc::mbar_wait(bar_q, k & 1, err, kErrQ);
        if (!ok) break;
        tc::tc_fence_after();
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
        for (int n = 0; n < x.ntiles && ok; ++n) ok = issue_s(0);
        if (ok && x.ntiles > 0) ok = issue_s(1);
        if (ok && x.ntiles <= 1) tc::mma_commit(q_empty);
        // O^T is overwritten (and o_full committed) only after the previous item's epilogue read it
        if (ok && k > 0) ok = tc::mbar_wait(o_empty, (k - 1) & 1, err, kErrOEmpty);
        for (int n = 0; n < x.ntiles && ok; ++n, ++pc) {
          if (n + 1 < x.ntiles) {
            ok = issue_s(1);
            if (ok && n + 2 == x.ntiles) tc::mma_commit(q_empty);   // the item's last S reads Q
          }
          if (!ok) break;
          ok = tc::mbar_wait(p_full, pc & 1, err, kErrPFull) &&
               tc::mbar_wait(vc_full + (pc & 1), (pc >> 1) & 1, err, kErrVcFull);
          if (!ok) break;
          tc::tc_fence_after();
          const uint8_t* vb = sVc + (pc & 1) * SM::kVSlices * kSlice;
          for (int ks = 0; ks < kBlk / 16; ++ks) {
            const uint64_t da = tc::sdesc(vb + ks * 16 * 128, kSlice, 1024);
            const uint64_t db = tc::sdesc(sP + ks * 16 * 128, kSlice, 1024);
            tc::mma_ss(tmem + kColO, da, db, idPV, (n | ks) != 0);
          }
          tc::mma_commit(p_empty);
          tc::mma_commit(vc_empty + (pc & 1));
        }
        if (ok) tc::mma_commit(o_full);
      }
    }
  } else if (warp >= kTopkWarp0) {
    // ------------------------------------------------------------ top-k
    // warp kTopkWarp0 + i takes tokens 4i .. 4i+3 of each item, two at a time: it copies
    // their scores out (zeroing them), selects from registers, and releases the score
    // buffer after the last pair has been copied
    const int w = warp - kTopkWarp0;
    bool ok = true;
    int k = 0;
    TopkWarp<2> tk;
    for (int it = next_item(blockIdx.x); it < n_items && ok; it = next_item(it + gridDim.x), ++k) {
      const Item x = item_of(it);
      ok = tc::mbar_wait(sc_full, k & 1, err, kErrScFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
#pragma unroll 1
      for (int pr = 0; pr < 2; ++pr) {
        const int t0p = x.t0 + 4 * w + 2 * pr;
        int nb[2], own[2];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int t = t0p + kk;
          nb[kk] = t < x.len ? t / kSel + 1 : 0;
          own[kk] = t / kSel;
        }
        tk.load(sScore + (4 * w + 2 * pr) * kMaxSel, kMaxSel, nb, own, force_first, force_local, lane);
        if (pr == 1) {
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(sc_empty);
        }
        int32_t* dst = idx_out + (((size_t)x.b * Hkv + x.g) * T + t0p) * top_k;
        tk.template select<0>(nb[0], own[0], top_k, force_first, force_local, dst, lane);
        tk.template select<1>(nb[1], own[1], top_k, force_first, force_local, dst + top_k, lane);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / epilogue
    // Four groups of four warps; group gr takes columns [32*gr, 32*gr+32) of every tile.
    // Warp quarter q = warp % 4 owns TMEM lanes 32q..32q+31; r is this thread's lane.
    const int gr = warp >> 2, q4 = warp & 3;
    const int r = 32 * q4 + lane;
    const int col0 = kCols * gr;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    constexpr int kNT = kSoftWarps * 32;   // softmax threads
    bool ok = true;
    int use = 0;   // S buffer uses
    int pc = 0;    // pass-B tiles
    for (int i = tid; i < kTok * kMaxSel; i += kNT) sScore[i] = 0.f;
    int k = 0;
    for (int it = next_item(blockIdx.x); it < n_items; it = next_item(it + gridDim.x), ++k) {
      const Item x = item_of(it);
      const int t0 = x.t0, g = x.g, ntiles = x.ntiles, len = x.len;
      const size_t base = x.base;
      float* gate = sGate + (k & 1) * kRowsM;
      if (gr == 0) {   // gates of the 128 rows (double-buffered: other groups may still be in the previous epilogue)
        const int t = t0 + r / 16, h = g * 16 + (r % 16);
        gate[r] = t < len ? __bfloat162float(gates[((base + t) * Hq + h) * 3]) : 0.f;
      }

      // pass A: this thread's row r = (token r/16, head r%16), its 32 columns of every tile
      {
        const int my_t = t0 + r / 16;
        const int my_hi = my_t < len ? n_visible(my_t, nc) : 0;
        float m = -INFINITY, l = 0.f;
        for (int n = 0; n < ntiles && ok; ++n, ++use) {
          const int sb = use & 1;
          ok = tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull);
          ok = __all_sync(0xffffffffu, ok);      // reconverge before the warp-wide TMEM loads
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t base = lane_addr + (sb ? kColS1 : kColS0) + col0;
          float v[kCols];
#pragma unroll
          for (int c = 0; c < kCols / 16; ++c)
            tc::tmem_ld16(base + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
          tc::tmem_wait_ld();
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(s_empty + sb);
          // masked scores; only a tile that straddles this row's range needs the per-element
          // test.  The maximum is taken on the raw scores (the scale is positive, and rounding
          // x * scale is monotone, so it equals the maximum of the scaled ones) and the scale
          // is applied inside the exponent's FMA.  Max and sum use eight independent chains each
          // (the sums as four packed pairs).
          const int i0 = n * kBlk + col0;
          if (i0 + kCols - 1 >= my_hi) {
#pragma unroll
            for (int j = 0; j < kCols; ++j) v[j] = i0 + j < my_hi ? v[j] : -INFINITY;
          }
          float cmx[8];
#pragma unroll
          for (int c = 0; c < 8; ++c) cmx[c] = v[c];
#pragma unroll
          for (int j = 8; j < kCols; ++j) cmx[j & 7] = fmaxf(cmx[j & 7], v[j]);
          const float cm = fmaxf(fmaxf(fmaxf(cmx[0], cmx[1]), fmaxf(cmx[2], cmx[3])),
                                 fmaxf(fmaxf(cmx[4], cmx[5]), fmaxf(cmx[6], cmx[7]))) * scale_log2;
          const float mn = fmaxf(m, cm);
          if (mn != -INFINITY) {
            // two columns per packed fma and add; four packed sums (eight chains)
            const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-mn, -mn);
            uint64_t ps[4];
#pragma unroll
            for (int c = 0; c < kCols / 2; ++c) {
              const float2 a = f2_unpack(f2_fma(f2_pack(v[2 * c], v[2 * c + 1]), sc2, nm2));
              const uint64_t p2 = f2_pack(ex2(a.x), ex2(a.y));
              ps[c & 3] = c < 4 ? p2 : f2_add(ps[c & 3], p2);
            }
            const float2 t = f2_unpack(f2_add(f2_add(ps[0], ps[1]), f2_add(ps[2], ps[3])));
            l = l * ex2(m - mn) + (t.x + t.y);
            m = mn;
          }
        }
        sML[(gr * 128 + r) * 2] = m;
        sML[(gr * 128 + r) * 2 + 1] = l;
      }
      ok = vote_all(3, kNT, ok);
      if (!ok) break;
      if (gr == 0) {
        float M = -INFINITY;
#pragma unroll
        for (int q = 0; q < kSoftGroups; ++q) M = fmaxf(M, sML[(q * 128 + r) * 2]);
        float L = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int q = 0; q < kSoftGroups; ++q) L += sML[(q * 128 + r) * 2 + 1] * ex2(sML[(q * 128 + r) * 2] - M);
        }
        sLse[r] = (t0 + r / 16 < len && L > 0.f) ? -(M + __log2f(L)) : -INFINITY;   // stored negated
      }
      // the previous item's scores must have been taken (and zeroed) by the top-k warps
      if (k > 0) ok = tc::mbar_wait(sc_empty, (k - 1) & 1, err, kErrScEmpty);
      ok = vote_all(3, kNT, ok);
      if (!ok) break;

      // pass B: this thread's key r of every tile; columns = tokens kTokG*gr .., 16 heads each
      int hi_tok[kTokG], nb_tok[kTokG];
#pragma unroll
      for (int kk = 0; kk < kTokG; ++kk) {
        const int t = t0 + kTokG * gr + kk;
        const bool in = t < len;
        hi_tok[kk] = in ? n_visible(t, nc) : 0;
        nb_tok[kk] = in ? t / kSel + 1 : 0;
      }
      // row r of P^T; this group's columns are 16-byte chunks (col0 % 64)/8 .. of N-block col0/64
      uint8_t* prow = sP + (col0 / 64) * kSlice + r * 128;
      const int ch0 = (col0 % 64) / 8;
      // Selection-block scores: block j = i/4 collects i = 4j-1 .. 4j+3.  Each group of four
      // lanes adds its own four blocks plus the lane just below it into the block's entry.
      // Lane 31's block (i % 4 == 3) also belongs to the first selection block of the next
      // warp (or of the next tile); that carry is added two tiles later, after waiting for
      // the P^T phase that every softmax warp releases only after its own score writes, so
      // no barrier is needed inside the loop.  Each entry receives at most two additions.
      float carry_a[kTokG], carry_b[kTokG];   // tiles n-1, n-2
#pragma unroll
      for (int kk = 0; kk < kTokG; ++kk) carry_a[kk] = carry_b[kk] = 0.f;
      auto add_carry = [&](const float (&c)[kTokG], int tile) {
        const int jt = tile * (kBlk / 4) + q4 * 8 + 8;
        if (lane == 31) {
#pragma unroll
          for (int kk = 0; kk < kTokG; ++kk)
            if (jt < nb_tok[kk]) sScore[(kTokG * gr + kk) * kMaxSel + jt] += c[kk];
        }
      };
      for (int n = 0; n < ntiles; ++n, ++use, ++pc) {
        const int sb = use & 1;
        // no barrier inside this loop: a warp that gives up leaves at once and the others
        // give up at their next wait (they see the error word); all meet after the loop
        ok = tc::mbar_wait(s_full + sb, (use >> 1) & 1, err, kErrSFull);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc::tc_fence_after();
        const uint32_t base = lane_addr + (sb ? kColS1 : kColS0) + col0;
        float v[kCols];
#pragma unroll
        for (int c = 0; c < kCols / 16; ++c)
          tc::tmem_ld16(base + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
        tc::tmem_wait_ld();
        const int i = n * kBlk + r;        // this thread's compressed block
        float tok_sum[kTokG];
        uint32_t pk[kCols / 2];
#pragma unroll
        for (int kk = 0; kk < kTokG; ++kk) {
          float sacc = 0.f;
          if (i < hi_tok[kk]) {
            // two columns per packed fma: x * scale - lse (the negated log-sum-exp of four
            // columns in one broadcast load), then the exponents and a packed running sum
            const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
            uint64_t acc2 = f2_pack(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
              const float4 nl = *reinterpret_cast<const float4*>(sLse + col0 + 16 * kk + j);
              const float2 a01 = f2_unpack(f2_fma(f2_pack(v[16 * kk + j], v[16 * kk + j + 1]), sc2, f2_pack(nl.x, nl.y)));
              const float2 a23 =
                  f2_unpack(f2_fma(f2_pack(v[16 * kk + j + 2], v[16 * kk + j + 3]), sc2, f2_pack(nl.z, nl.w)));
              const float p0 = ex2(a01.x), p1 = ex2(a01.y), p2 = ex2(a23.x), p3 = ex2(a23.y);
              acc2 = f2_add(acc2, f2_add(f2_pack(p0, p1), f2_pack(p2, p3)));
              pk[8 * kk + j / 2] = pack_bf16(p0, p1);
              pk[8 * kk + j / 2 + 1] = pack_bf16(p2, p3);
            }
            const float2 a = f2_unpack(acc2);
            sacc = a.x + a.y;
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) pk[8 * kk + j] = 0u;
          }
          // block i = this thread's r straddles two selection blocks when i % 4 == 3
          tok_sum[kk] = (lane & 3) == 3 ? sacc * w_straddle : sacc;
        }
        {
          const int j0 = n * (kBlk / 4) + q4 * 8;    // first selection block of this warp
#pragma unroll
          for (int kk = 0; kk < kTokG; ++kk) {
            const float vv = tok_sum[kk];
            float g4 = vv + __shfl_xor_sync(0xffffffffu, vv, 1);
            g4 += __shfl_xor_sync(0xffffffffu, g4, 2);
            const float prev = __shfl_up_sync(0xffffffffu, vv, 1);
            const int j = j0 + (lane >> 2);
            if ((lane & 3) == 0 && j < nb_tok[kk]) sScore[(kTokG * gr + kk) * kMaxSel + j] += g4 + (lane > 0 ? prev : 0.f);
          }
        }
        // P^T(pc) may overwrite the buffer once PV(pc-1) has read it
        if (pc > 0) ok = tc::mbar_wait(p_empty, (pc - 1) & 1, err, kErrPEmpty);
        if (n > 0 && ok) {
          // P^T(pc-1) was released by every softmax warp after its score writes of tiles
          // <= n-1; this warp has not released P^T(pc) yet, so the phase is unambiguous
          ok = tc::mbar_wait(p_full, (pc - 1) & 1, err, kErrPFull);
          if (n > 1) add_carry(carry_b, n - 2);
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
#pragma unroll
        for (int kk = 0; kk < kTokG; ++kk) {
          carry_b[kk] = carry_a[kk];
          carry_a[kk] = tok_sum[kk];
        }
#pragma unroll
        for (int c = 0; c < kCols / 8; ++c)
          *reinterpret_cast<uint4*>(prow + (((ch0 + c) ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        tc::tc_fence_before();
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(s_empty + sb);
          tc::mbar_arrive(p_full);
        }
      }
      ok = vote_all(3, kNT, ok);
      if (!ok) break;
      // the carries of the last two tiles, then hand the scores to the top-k warps
      if (ntiles > 1) add_carry(carry_b, ntiles - 2);
      if (ntiles > 0) add_carry(carry_a, ntiles - 1);
      named_sync(3, kNT);
      if (tid == 0) tc::mbar_arrive(sc_full);

      // epilogue: lane r = value dim r of O^T; this group's 32 columns = tokens kTokG*gr ..
      // A failed wait here only skips the stores: the next item's vote ends the loop for all.
      ok = tc::mbar_wait(o_full, k & 1, err, kErrOFull);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc::tc_fence_after();
        float v[kCols];
        if (ntiles > 0) {
#pragma unroll
          for (int c = 0; c < kCols / 16; ++c)
            tc::tmem_ld16(lane_addr + kColO + col0 + 16 * c, *reinterpret_cast<float(*)[16]>(v + 16 * c));
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int c = 0; c < kCols; ++c) v[c] = 0.f;
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(o_empty);
#pragma unroll
        for (int c = 0; c < kCols; ++c) {
          const int t = t0 + kTokG * gr + c / 16;
          if (t < len && r < DV) {
            const size_t row = (base + t) * Hq + g * 16 + (c % 16);
            acc[row * DV + r] = gate[col0 + c] * v[c];
          }
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

template <int DK, int DV>
cudaError_t launch_tc(const FwdArgs& a, cudaStream_t st) {
  using SM = Smem<DK, DV>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SM::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  const int sms = sm_count();
  CUtensorMap mq, mk, mv;
  const uint64_t dq[3] = {(uint64_t)DK, (uint64_t)a.Hq, (uint64_t)a.total};
  const uint64_t sq[2] = {(uint64_t)DK * 2, (uint64_t)a.Hq * DK * 2};
  const uint32_t bq[3] = {64, 16, kTok};
  const uint64_t dk3[3] = {(uint64_t)DK, (uint64_t)a.Hkv, (uint64_t)a.B * a.nc};
  const uint64_t sk3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hkv * DK * 2};
  const uint64_t dv3[3] = {(uint64_t)DV, (uint64_t)a.Hkv, (uint64_t)a.B * a.nc};
  const uint64_t sv3[2] = {(uint64_t)DV * 2, (uint64_t)a.Hkv * DV * 2};
  const uint32_t bkv[3] = {64, 1, kBlk};
  if (!make_tmap_bf16(&mq, a.q, 3, dq, sq, bq)) return cudaErrorInvalidValue;
  if (a.nc > 0) {
    if (!make_tmap_bf16(&mk, a.kc, 3, dk3, sk3, bkv) || !make_tmap_bf16(&mv, a.vc, 3, dv3, sv3, bkv))
      return cudaErrorInvalidValue;
  } else {
    mk = mq;   // never dereferenced: no tile is loaded when there is no compressed block
    mv = mq;
  }
  const long long n_items = (long long)((a.T + kTok - 1) / kTok) * a.Hkv * a.B;
  if (n_items == 0) return cudaSuccess;
  const int grid = (int)std::min<long long>(n_items, sms);
  auto kernel = a.cu ? attn_tc_kernel<DK, DV, true> : attn_tc_kernel<DK, DV, false>;
  kernel<<<grid, kThreads, SM::kAlloc, st>>>(
      mq, mk, mv, static_cast<const __nv_bfloat16*>(a.gates), a.acc, a.idx, a.B, a.T, a.Hq, a.Hkv, a.nc, a.top_k,
      a.force_first, a.force_local, a.scale_log2, a.w_straddle, a.cu, a.err);
  return cudaGetLastError();
}
}  // namespace

bool cmp_select_tc_supported(const FwdArgs& a) {
  return a.G == 16 && a.dv == 128 && (a.dk == 128 || a.dk == 192) && a.T <= kMaxSel * kSel && a.err != nullptr;
}

cudaError_t launch_cmp_select_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192) return launch_tc<192, 128>(a, st);
  return launch_tc<128, 128>(a, st);
}

}  // namespace nsa
