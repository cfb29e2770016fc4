// K3 on the fifth-generation tensor cores: selected-block attention
// ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5: the top-k blocks are expanded to all
// their tokens and attended; §10: the group's heads share every loaded block, so the
// matrix products take the heads as one dimension).
//
// An item is one (token, KV group): the group's 16 query heads over the tokens of the
// blocks the group chose for that token.  The chosen blocks are taken two at a time: a
// pair is 128 keys, the M dimension of the tcgen05 MMAs, and the 16 heads are N:
//   S^T = K_pair Q^T      (A = 128 key rows, K-major; B = the 16 query rows, K-major)
//   O^T += V_pair^T P^T   (A = V^T, MN-major as TMA lays V down; B = P^T, K-major)
// Both accumulate in TMEM (S^T: lane = key, column = head; O^T: lane = value column,
// column = head), so no thread holds an accumulator.
//
// The costs that shape the design (measured on this GPU):
//   - an MMA that accumulates into the accumulator of the MMA just before it waits for that
//     one (about 170 cycles), while independent N = 16 MMAs take 45-60: so S^T is spread
//     over four partial accumulators (K step k of each 64-column slab into partial k) and
//     O^T over eight (16-key step k into partial k), and the readers add the partials;
//   - one thread issues every MMA, so its own work per pair (waits, commits, bookkeeping)
//     adds to the pair's time: it waits once and commits once per pair.  Step n of the
//     stream of pairs is the P.V of pair n and the S of pair n + 2; its "ready" barrier
//     collects the keys of pair n + 2, the values of pair n and P^T of pair n, its "done"
//     commit frees their slots and makes S^T of pair n + 2 readable.
//
// Persistent: one CTA per SM walks the items group-major (the CTAs running together share
// one group's K/V in L2).  Warp roles:
//   warp 12    TMA producer of keys: the item's block list (into shared memory), its 16
//              query rows (3-slot item ring), each pair's K (2-slot ring of 48 KB pairs).
//   warp 14    TMA producer of values: each pair's V (2-slot ring of 32 KB pairs).  The
//              rings run across items.
//   warp 13    MMA issuer (one thread): the S of pairs 0 and 1, then per step the P.V of
//              pair n and the S of pair n + 2, so the softmax of a pair overlaps the S of the
//              pairs after it.  Alternate items accumulate into two O buffers, so an item's
//              pairs overlap the previous item's epilogue.
//   warps 0-7  softmax: warp w takes TMEM lane quadrant w % 4 (32 keys of each pair) and
//              heads 8(w / 4) .. 8(w / 4) + 7.  p = 2^(s*scale - m) with one reference m per
//              (item, head): the largest valid score of the item's first pair, agreed by the
//              four quadrants' warps at a named barrier and never moved afterwards, so no
//              warp waits for another after the first pair.  P^T (bf16) goes to shared
//              memory; each thread keeps its keys' partial row sums, added up once per item.
//   warps 8-11 epilogue, one quadrant of value columns each: acc += g_slc * O / l.
//
// A later score can exceed its fixed reference without bound, so p is not bounded by 1.
// fp32 and bf16 carry such values exactly up to 2^127; an item whose row sum in any
// quadrant passes 2^64 (or is not finite) is not written but listed, and a second kernel
// recomputes the listed items with an exact two-pass softmax on the CUDA cores.  Scores that
// far apart do not occur in attention over trained or random keys; the path keeps the result
// right when they do.
#include <cfloat>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
constexpr int kSoftWarps = 8;                      // warps 0-7
constexpr int kEpiWarp0 = 8;                       // warps 8-11
constexpr int kTmaWarp = 12, kMmaWarp = 13, kTmaVWarp = 14;
constexpr int kThreads = 480;
constexpr int kHH = 8;                             // heads per softmax warp
constexpr int kBlk = 64;
constexpr int kG = 16;                             // heads per group: the MMA N
constexpr int kKSlots = 2, kVSlots = 2;            // pair slots (also the P^T buffers: pair n uses n % 2)
static_assert(kKSlots == 2 && kVSlots == 2, "slots and phases come from the pair counter's low bits");
constexpr int kItemSlots = 3;
constexpr uint32_t kBox = kBlk * 128;              // 64 rows x 64 bf16 (128-byte swizzle): 8 KB
constexpr uint32_t kSlab = 2 * kBox;               // the pair's 128 rows x 64 columns: 16 KB
constexpr int kSChains = 4, kOChains = 8;          // partial accumulators of S^T and O^T
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                      // S buffer b, partial c: 64b + 16c
constexpr uint32_t kColO = 2 * kSChains * kG;      // O buffer b, partial c: 128 + 128b + 16c
constexpr float kRowSumLimit = 18446744073709551616.f;   // 2^64: above it the item is recomputed
constexpr int kMetaInts = 36;                      // per item slot: 32 block ids, the count

enum Err { kErrQEmpty = 61, kErrQFull, kErrKSlot, kErrProK, kErrVSlot, kErrReady, kErrSDone, kErrOEmpty, kErrOFull,
           kErrLEmpty, kErrLFull };

template <int DK, int DV>
struct Smem {
  static constexpr int kKS = DK / 64, kVS = DV / 64;
  static constexpr uint32_t kKBytes = kKS * kSlab, kVBytes = kVS * kSlab;   // a pair's K or V slabs
  static constexpr uint32_t kK = 0;                                    // [K slot]
  static constexpr uint32_t kV = kK + kKSlots * kKBytes;               // [V slot]
  static constexpr uint32_t kQBytes = kKS * kG * 128;                  // 16 rows x DK: kKS boxes of 2 KB
  static constexpr uint32_t kQ = kV + kVSlots * kVBytes;               // [item slot]
  static constexpr uint32_t kPBytes = 2 * kG * 128;                    // P^T: [key half][16 heads][128 B]
  static constexpr uint32_t kP = kQ + kItemSlots * kQBytes;            // [2]
  static constexpr uint32_t kMeta = kP + 2 * kPBytes;                  // [item slot][kMetaInts]
  static constexpr uint32_t kLsum = kMeta + kItemSlots * kMetaInts * 4;   // [2][quadrant][16] row sums
  static constexpr uint32_t kRef = kLsum + 2 * 4 * kG * 4;                 // [quadrant][16] first-pair maxima
  static constexpr uint32_t kBar = (kRef + 4 * kG * 4 + 7) & ~7u;
  static constexpr int kNumBars = 2 * kItemSlots + 2 + 2 + 2 + 2 + 2 * 2 + 2 * 2;
  static constexpr uint32_t kTmemSlot = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kTmemSlot + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 232448, "shared memory");
  static_assert(kQ % 1024 == 0 && kQBytes % 1024 == 0 && kP % 1024 == 0, "swizzled tiles need 1 KB alignment");
};

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// the sum of the n partial accumulators (16 columns each, consecutive) of this thread's lane
template <int N>
__device__ __forceinline__ void tmem_sum_partials(uint32_t addr, float (&x)[kG]) {
  float y[kG];
  tc::tmem_ld16(addr, x);
  tc::tmem_ld16(addr + kG, y);
  tc::tmem_wait_ld();
#pragma unroll
  for (int h = 0; h < kG; ++h) x[h] += y[h];
#pragma unroll
  for (int c = 2; c < N; ++c) {
    tc::tmem_ld16(addr + c * kG, y);
    tc::tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < kG; ++h) x[h] += y[h];
  }
}

template <int DK, int DV, bool VARLEN>
__global__ void __launch_bounds__(kThreads, 1)
slc_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const __nv_bfloat16* __restrict__ gates,
                   const int32_t* __restrict__ idx, float* __restrict__ acc, int B, int T, int Hq, int Hkv,
                   int top_k, float scale_log2, const int32_t* __restrict__ cu_in, int* __restrict__ redo_count,
                   int* __restrict__ redo_list, int* __restrict__ err) {
  using SM = Smem<DK, DV>;
  static_assert(DV == 128, "the value columns are the 128 TMEM lanes of O^T");
  const int32_t* cu = VARLEN ? cu_in : nullptr;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + SM::kK;
  uint8_t* sV = smem + SM::kV;
  uint8_t* sQ = smem + SM::kQ;
  uint8_t* sP = smem + SM::kP;
  int* sMeta = reinterpret_cast<int*>(smem + SM::kMeta);
  float* sLsum = reinterpret_cast<float*>(smem + SM::kLsum);               // [2][quadrant][16]
  float* sRef = reinterpret_cast<float*>(smem + SM::kRef);                 // [quadrant][16]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SM::kBar);
  // Pair n (counted over the CTA's whole walk) uses K slot, V slot, S buffer and P^T buffer n % 2.
  // Step n = the P.V of pair n and the S of pair n + 2 (the S of pairs 0 and 1 come before).
  uint64_t* q_full = bars;                       // [item slot] block list written and queries landed
  uint64_t* q_empty = q_full + kItemSlots;       // [item slot] the softmax warps are done with the item
  uint64_t* pro_k = q_empty + kItemSlots;        // [2] the keys of pair 0 / 1 landed
  uint64_t* pro_done = pro_k + 2;                // [2] the S of pair 0 / 1 is done
  uint64_t* ready = pro_done + 2;                // [n % 2] step n: K of pair n + 2, V of pair n, P^T of pair n
  uint64_t* done = ready + 2;                    // [n % 2] step n is done: S^T of pair n + 2 ready, slots free
  uint64_t* o_full = done + 2;                   // [2] an item's O^T is complete
  uint64_t* o_empty = o_full + 2;                // [2] the epilogue has read it
  uint64_t* l_full = o_empty + 2;                // [2] an item's row sums are in shared memory
  uint64_t* l_empty = l_full + 2;                // [2] the epilogue has read them
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SM::kTmemSlot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kItemSlots; ++i) {
      tc::mbar_init(q_full + i, 1);
      tc::mbar_init(q_empty + i, kSoftWarps);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(pro_k + i, 1);
      tc::mbar_init(pro_done + i, 1);
      tc::mbar_init(ready + i, 2 + kSoftWarps);   // the two producers, the softmax warps
      tc::mbar_init(done + i, 1);
      tc::mbar_init(o_full + i, 1);
      tc::mbar_init(o_empty + i, 4);
      tc::mbar_init(l_full + i, kSoftWarps);
      tc::mbar_init(l_empty + i, 4);
    }
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

  // item it = (group, batch, token), group-major; in a variable-length batch the tokens
  // past a sequence's end are no items, and every role skips them alike
  const long total = (long)Hkv * B * T;
  const long stride = gridDim.x;
  auto next_item = [&](long it) {
    if constexpr (VARLEN)
      while (it < total && (int)(it % T) >= seq_len(cu, (int)((it / T) % B), T)) it += stride;
    return it;
  };
  auto row_of = [&](int b, int t) -> size_t {   // row of token t of sequence b in q, k, v, gates, acc
    if constexpr (VARLEN) return (size_t)seq_base(cu, b, T) + t;
    else return (size_t)b * T + t;
  };

  if (warp == kTmaWarp || warp == kTmaVWarp) {
    // ------------------------------------------------------------ TMA producers (the whole
    // warp loops; lane 0 issues the copies).  Warp kTmaWarp: block lists, queries and keys;
    // warp kTmaVWarp: values.  An item has at least one pair: with no block chosen (never
    // the case for a token's own list) the pair's keys are all masked.
    const bool keys = warp == kTmaWarp;
    if (lane == 0) {
      tc::prefetch_tmap(keys ? &tm_k : &tm_v);
      if (keys) tc::prefetch_tmap(&tm_q);
    }
    const int nslab = keys ? SM::kKS : SM::kVS;
    const uint32_t slot_bytes = nslab * kSlab;
    uint8_t* const ring = keys ? sK : sV;
    const CUtensorMap* const map = keys ? &tm_k : &tm_v;
    // pair f's slot (f % 2) is free once the pair two back is done with it: its S for keys
    // (step f - 4, or the prologue for f < 4), its P.V for values (step f - 2)
    auto wait_slot = [&](uint32_t f) -> bool {
      if (keys) {
        if (f < 2) return true;
        if (f < 4) return tc::mbar_wait(pro_done + (f & 1), 0u, err, kErrKSlot);
        return tc::mbar_wait(done + (f & 1), (f >> 1) & 1u, err, kErrKSlot);
      }
      return tc::mbar_wait(done + (f & 1), ((f >> 1) & 1u) ^ 1u, err, kErrVSlot);
    };
    // where pair f's copies arrive: the keys of pairs 0 and 1 on their own barriers, the
    // others on step f - 2 (keys) or step f (values)
    auto arrive_bar = [&](uint32_t f) -> uint64_t* { return keys && f < 2 ? pro_k + f : ready + (f & 1); };
    long k = 0;
    uint32_t f = 0;
    bool ok = true;
    for (long it = next_item(blockIdx.x); it < total && ok; it = next_item(it + stride), ++k) {
      const int g = (int)(it / ((long)B * T));
      const int bt = (int)(it % ((long)B * T));
      const int b = bt / T, t = bt % T;
      const int base = (int)row_of(b, 0);
      int j = lane < top_k ? idx[(((size_t)b * Hkv + g) * T + t) * top_k + lane] : -1;
      j = j >= 0 ? min(j, t / kBlk) : -1;
      const int nblk = __popc(__ballot_sync(0xffffffffu, j >= 0));   // the list is -1 padded at its end
      if (keys) {
        const int qs = (int)(k % kItemSlots);
        ok = __all_sync(0xffffffffu, tc::mbar_wait(q_empty + qs, (uint32_t)(((k / kItemSlots) & 1) ^ 1), err,
                                                   kErrQEmpty));
        if (!ok) break;
        int* meta = sMeta + qs * kMetaInts;
        if (lane < nblk) meta[lane] = j;
        if (lane == 0) meta[32] = nblk;
        __threadfence_block();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_expect_tx(q_full + qs, SM::kQBytes);   // also publishes the block list
          for (int s = 0; s < SM::kKS; ++s)
            tc::tma_load_3d(sQ + qs * SM::kQBytes + s * kG * 128, &tm_q, q_full + qs, s * 64, g * kG, base + t);
        }
      }
      const int npairs = max(1, (nblk + 1) / 2);
      for (int p = 0; p < npairs && ok; ++p, ++f) {
        const int jr0 = __shfl_sync(0xffffffffu, j, (2 * p) & 31);
        const int jr1 = __shfl_sync(0xffffffffu, j, (2 * p + 1) & 31);
        const int j0 = 2 * p < nblk ? jr0 : t / kBlk;   // (masked: nothing was chosen)
        const int j1 = 2 * p + 1 < nblk ? jr1 : j0;     // an odd count repeats the block (masked out)
        ok = __all_sync(0xffffffffu, wait_slot(f));
        if (!ok) break;
        if (lane == 0) {
          uint8_t* dst = ring + (f & 1) * slot_bytes;
          uint64_t* bar = arrive_bar(f);
          tc::mbar_expect_tx(bar, slot_bytes);
          for (int s = 0; s < nslab; ++s) {
            tc::tma_load_3d(dst + s * kSlab, map, bar, s * 64, g, base + j0 * kBlk);
            tc::tma_load_3d(dst + s * kSlab + kBox, map, bar, s * 64, g, base + j1 * kBlk);
          }
        }
        __syncwarp();
      }
    }
    if (ok && keys) {
      // steps F - 2 and F - 1 (F = this CTA's pairs) have no pair two ahead: their key
      // arrivals carry no bytes, made once their phase is the current one
      for (uint32_t ff = max(f, 2u); ff < f + 2 && ok; ++ff) {
        ok = __all_sync(0xffffffffu, wait_slot(ff));
        if (ok && lane == 0) tc::mbar_arrive(ready + (ff & 1));
        __syncwarp();
      }
    }
    // No drain here: every copy lands on a barrier the MMA thread waits for (the queries and
    // keys of every pair, the values of every step) before the CTA's final barrier.  (A wait
    // on a step barrier from here could also see its phase bit already turned twice.)
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // Prologue: the S of pairs 0 and 1.  Step n: once its barrier is complete (keys of pair
    // n + 2, values and P^T of pair n), the P.V of pair n, then the S of pair n + 2, one
    // commit.  The two products stay in blocks of their own: alternating MMAs of the K-major
    // S with those of the MN-major V^T slowed both down.
    if (tc::elect_one()) {
      const uint32_t idS = tc::idesc_bf16(128, kG, 0, 0);    // S^T = K Q^T: both K-major
      const uint32_t idPV = tc::idesc_bf16(128, kG, 1, 0);   // O^T = V^T P^T: V^T MN-major, P^T K-major
      const uint64_t dp0 = tc::sdesc(sP, 16, 1024);
      // A pair of the stream: its counter f, its item's counter k (the low bit picks the O
      // buffer) and item slot.  Everything this thread computes per pair is 32-bit adds,
      // compares and bit operations.
      struct Pair { uint32_t f, k; int qs; bool first, last; };
      long it_c = next_item(blockIdx.x);
      uint32_t k_c = 0, f_c = 0, qph = 0;   // qph: the phase bit of item slot qs_c
      int qs_c = 0, p_c = 0, np_c = -1;
      bool ok = true;
      auto next_pair = [&](Pair& e) -> bool {   // false: the walk is over (or a wait failed)
        if (it_c >= total) return false;
        if (np_c < 0) {
          ok = tc::mbar_wait(q_full + qs_c, qph, err, kErrQFull);
          if (!ok) return false;
          np_c = max(1, (sMeta[qs_c * kMetaInts + 32] + 1) >> 1);
          p_c = 0;
        }
        e.f = f_c++;
        e.k = k_c;
        e.qs = qs_c;
        e.first = p_c == 0;
        e.last = p_c == np_c - 1;
        if (++p_c == np_c) {   // the item is done: move to the next
          it_c = next_item(it_c + stride);
          ++k_c;
          np_c = -1;
          if (++qs_c == kItemSlots) {
            qs_c = 0;
            qph ^= 1u;
          }
        }
        return true;
      };
      // the S MMAs of pair y (K step kk of slab sl into partial kk)
      auto issue_s = [&](const Pair& y) {
        const uint64_t dk0 = tc::sdesc(sK + (y.f & 1) * SM::kKS * kSlab, 16, 1024);
        const uint64_t dq0 = tc::sdesc(sQ + y.qs * SM::kQBytes, 16, 1024);
        const uint32_t d_s = tmem + kColS + kSChains * kG * (y.f & 1);
#pragma unroll 1
        for (int sl = 0; sl < SM::kKS; ++sl) {
          const uint64_t dk = dk0 + (uint64_t)(sl * kSlab / 16), dq = dq0 + (uint64_t)(sl * kG * 128 / 16);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::mma_ss(d_s + kG * kk, dk + (uint64_t)(kk * 2), dq + (uint64_t)(kk * 2), idS, sl != 0);
        }
      };
      Pair q0{}, q1{};   // pairs whose S is issued and whose P.V is not (in registers, no array)
      int nq = 0;
      for (; nq < 2 && ok; ++nq) {
        Pair e;
        if (!next_pair(e)) break;
        if (!(ok = tc::mbar_wait(pro_k + nq, 0u, err, kErrProK))) break;
        tc::tc_fence_after();
        issue_s(e);
        tc::mma_commit(pro_done + nq);
        if (nq == 0) q0 = e;
        else q1 = e;
      }
      while (ok && nq > 0) {
        const Pair x = q0;
        Pair y;
        const bool have_y = next_pair(y);
        if (!ok) break;
        const int ob = (int)(x.k & 1);
        ok = (!x.first || tc::mbar_wait(o_empty + ob, ((x.k >> 1) & 1u) ^ 1u, err, kErrOEmpty)) &&
             tc::mbar_wait(ready + (x.f & 1), (x.f >> 1) & 1u, err, kErrReady);
        if (!ok) break;
        tc::tc_fence_after();
        {
          const uint64_t dv0 = tc::sdesc(sV + (x.f & 1) * SM::kVBytes, kSlab, 1024);
          const uint64_t dp = dp0 + (uint64_t)((x.f & 1) * SM::kPBytes / 16);
          const uint32_t d_o = tmem + kColO + kOChains * kG * ob;
          const uint32_t accum = x.first ? 0u : 1u;
#pragma unroll
          for (int ks = 0; ks < 2 * kBlk / 16; ++ks)   // 16-key step ks into partial ks
            tc::mma_ss(d_o + kG * ks, dv0 + (uint64_t)(ks * 16 * 128 / 16),
                       dp + (uint64_t)(((ks >> 2) * (kG * 128) + (ks & 3) * 32) / 16), idPV, accum);
        }
        if (have_y) issue_s(y);
        tc::mma_commit(done + (x.f & 1));
        if (x.last) tc::mma_commit(o_full + ob);
        q0 = q1;
        if (have_y) q1 = y;
        else --nq;
      }
    }
  } else if (warp < kSoftWarps) {
    // ------------------------------------------------------------ softmax
    const int qd = warp & 3;                           // TMEM lane quadrant: keys 32qd .. 32qd + 31
    const int h0 = kHH * (warp >> 2);                  // this warp's heads h0 .. h0 + 7
    const int r = 32 * qd + lane;                      // this thread's key of the pair
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * qd) << 16) + h0;
    // this thread's column of P^T (K-major, 128-byte swizzle): key half, 16-byte chunk, element
    uint8_t* const pcol = sP + (r >> 6) * (kG * 128) + 2 * (r & 7);
    const int pchunk = (r & 63) >> 3;
    const int bar_g = 1 + (warp >> 2);               // named barrier of the four warps of this head half
    long k = 0, f = 0;
    bool ok = true;
    for (long it = next_item(blockIdx.x); it < total; it = next_item(it + stride), ++k) {
      const int t = (int)((it % ((long)B * T)) % T);
      const int qs = (int)(k % kItemSlots);
      // one decision for the four warps, which meet at a barrier in the item's first pair;
      // after a failed wait they leave together
      ok = tc::vote_all(bar_g, 4 * 32,
                        ok && tc::mbar_wait(q_full + qs, (uint32_t)((k / kItemSlots) & 1), err, kErrQFull));
      if (!ok) break;
      const int* meta = sMeta + qs * kMetaInts;
      const int nblk = meta[32];
      const int npairs = max(1, (nblk + 1) / 2);
      float m[kHH], lp[kHH];                           // reference (log2 units) and partial row sums
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        m[h] = -INFINITY;
        lp[h] = 0.f;
      }
      for (int p = 0; p < npairs; ++p, ++f) {
        const int sb = (int)(f & 1);
        // S^T of pair f is ready and P^T buffer f % 2 free: the prologue (pairs 0, 1) or step f - 2
        ok = __all_sync(0xffffffffu, ok && (f < 2 ? tc::mbar_wait(pro_done + f, 0u, err, kErrSDone)
                                                  : tc::mbar_wait(done + (f & 1), (uint32_t)(((f >> 1) & 1) ^ 1),
                                                                  err, kErrSDone)));
        float x[kHH], y[kHH];
#pragma unroll
        for (int h = 0; h < kHH; ++h) x[h] = 0.f;
        tc::tc_fence_after();
        if (ok) {
          const uint32_t sa = lane_addr + kColS + kSChains * kG * sb;
          tc::tmem_ld8(sa, x);
          tc::tmem_ld8(sa + kG, y);
          tc::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHH; ++h) x[h] += y[h];
#pragma unroll
          for (int c = 2; c < kSChains; ++c) {
            tc::tmem_ld8(sa + c * kG, y);
            tc::tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kHH; ++h) x[h] += y[h];
          }
        }
        tc::tc_fence_before();   // the S^T reads are ordered before the P^T arrival below
        const int jj = 2 * p + (r >> 6);
        const int j = jj < nblk ? meta[jj] : -1;
        const bool valid = j >= 0 && j * kBlk + (r & 63) <= t;
        // the reference: per head, the largest valid score of the item's first pair over the
        // four quadrants (the first key of the first pair is always valid)
        if (p == 0) {
          float wm[kHH];
#pragma unroll
          for (int h = 0; h < kHH; ++h) wm[h] = warp_max_f32(valid ? x[h] : -INFINITY);
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < kHH; ++h) sRef[qd * kG + h0 + h] = wm[h];
          }
          const bool all_ok = tc::vote_all(bar_g, 4 * 32, ok);
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            m[h] = fmaxf(fmaxf(sRef[h0 + h], sRef[kG + h0 + h]), fmaxf(sRef[2 * kG + h0 + h], sRef[3 * kG + h0 + h])) *
                   scale_log2;
          tc::named_sync(bar_g, 4 * 32);   // read before the next item rewrites it
          ok = all_ok;
          if (!ok) break;                  // all four warps together
        }
        // after a failed wait a warp runs out the item's pairs doing nothing; the four warps
        // leave together at the next item's vote
        if (!ok) continue;
        uint32_t pk[kHH / 2];
#pragma unroll
        for (int h = 0; h < kHH; h += 2) {
          const float p0 = valid ? ex2(fmaf(x[h], scale_log2, -m[h])) : 0.f;
          const float p1 = valid ? ex2(fmaf(x[h + 1], scale_log2, -m[h + 1])) : 0.f;
          lp[h] += p0;
          lp[h + 1] += p1;
          pk[h / 2] = pack_bf16(p0, p1);
        }
        uint8_t* const pc = pcol + (f & 1) * SM::kPBytes;
#pragma unroll
        for (int h = 0; h < kHH; ++h)
          *reinterpret_cast<uint16_t*>(pc + (h0 + h) * 128 + ((pchunk ^ (h & 7)) << 4)) =
              (uint16_t)(pk[h / 2] >> (16 * (h & 1)));
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(ready + (f & 1));
      }
      if (!ok) continue;   // the next item's vote ends the walk
      // the item's row sums of this quadrant: reduce the 8 partial sums over the warp's 32
      // keys (each step halves the heads a lane keeps); lane 4i holds head h0 + i
      float a4[4], a2[2], a1;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const bool hi = lane & 16;
        const float send = hi ? lp[i] : lp[i + 4];
        a4[i] = (hi ? lp[i + 4] : lp[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const bool hi = lane & 8;
        const float send = hi ? a4[i] : a4[i + 2];
        a2[i] = (hi ? a4[i + 2] : a4[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
      }
      {
        const bool hi = lane & 4;
        const float send = hi ? a2[0] : a2[1];
        a1 = (hi ? a2[1] : a2[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
      a1 += __shfl_xor_sync(0xffffffffu, a1, 1);       // head h0 + ((lane >> 2) & 7)
      const int ob = (int)(k & 1);
      ok = __all_sync(0xffffffffu, tc::mbar_wait(l_empty + ob, (uint32_t)(((k >> 1) & 1) ^ 1), err, kErrLEmpty));
      if (!ok) continue;
      if ((lane & 3) == 0) sLsum[(ob * 4 + qd) * kG + h0 + (lane >> 2)] = a1;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(l_full + ob);
        tc::mbar_arrive(q_empty + qs);                 // done with the item's block list and queries
      }
    }
  } else if (warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue: acc += g_slc O / l
    const int qd = warp & 3;
    const int d = 32 * qd + lane;                      // this thread's value column
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * qd) << 16);
    long k = 0;
    bool ok = true;
    for (long it = next_item(blockIdx.x); it < total && ok; it = next_item(it + stride), ++k) {
      const int g = (int)(it / ((long)B * T));
      const int bt = (int)(it % ((long)B * T));
      const size_t row0 = row_of(bt / T, bt % T) * Hq + (size_t)g * kG;   // (token, head 0 of the group)
      // start the accumulator rows (this warp's 128-byte column segment of each head row) and
      // the gates on their way to L2; they are read after the item's O is complete
      if (lane < kG) prefetch_l2(acc + (row0 + lane) * DV + 32 * qd);
      if (lane == kG) prefetch_l2(gates + row0 * 3);
      const int ob = (int)(k & 1);
      ok = __all_sync(0xffffffffu, tc::mbar_wait(l_full + ob, (uint32_t)((k >> 1) & 1), err, kErrLFull));
      if (!ok) break;
      // the row sums of the four quadrants (all taken against the same reference)
      const float* ls = sLsum + ob * 4 * kG;
      float L[kG];
      bool bad = false;
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        const float l0 = ls[h], l1 = ls[kG + h], l2 = ls[2 * kG + h], l3 = ls[3 * kG + h];
        bad = bad || !(l0 <= kRowSumLimit && l1 <= kRowSumLimit && l2 <= kRowSumLimit && l3 <= kRowSumLimit);
        L[h] = (l0 + l1) + (l2 + l3);
      }
      float o[kG];
      ok = __all_sync(0xffffffffu, tc::mbar_wait(o_full + ob, (uint32_t)((k >> 1) & 1), err, kErrOFull));
      if (!ok) break;
      tc::tc_fence_after();
      tmem_sum_partials<kOChains>(lane_addr + kColO + kOChains * kG * ob, o);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        tc::mbar_arrive(o_empty + ob);
        tc::mbar_arrive(l_empty + ob);
      }
      if (bad) {   // a row sum out of range: the item is recomputed exactly by the redo kernel
        if (qd == 0 && lane == 0) redo_list[atomicAdd(redo_count, 1)] = (int)it;
        continue;
      }
      float a[kG];
#pragma unroll
      for (int h = 0; h < kG; ++h) {
        a[h] = acc[(row0 + h) * DV + d];
        L[h] = L[h] > 0.f ? __bfloat162float(gates[(row0 + h) * 3 + 1]) / L[h] : 0.f;
      }
#pragma unroll
      for (int h = 0; h < kG; ++h)
        if (L[h] != 0.f) acc[(row0 + h) * DV + d] = a[h] + L[h] * o[h];
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

// The exact path for the items the tensor-core kernel listed (a row sum out of range):
// one CTA per listed item, fp32 on the CUDA cores, a two-pass softmax per head (the
// largest score first, then the probabilities), acc += g_slc * o_slc.  Shared memory:
// the item's queries, its key rows' positions and the [keys][16] scores.
constexpr int kRedoThreads = 256;
constexpr int kRedoMaxKeys = 32 * kBlk;

template <int DK>
struct RedoSmem {
  static constexpr uint32_t kScores = 0;                                  // [key][16] float
  static constexpr uint32_t kQ = kScores + kRedoMaxKeys * kG * 4;         // [16][DK] float
  static constexpr uint32_t kKeys = kQ + kG * DK * 4;                     // [key] token positions
  static constexpr uint32_t kRed = kKeys + kRedoMaxKeys * 4;              // [16][16] float
  static constexpr uint32_t kBytes = kRed + 2 * kG * kG * 4 + 16;
};

template <int DK, int DV, bool VARLEN>
__global__ void __launch_bounds__(kRedoThreads)
slc_redo_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ gates,
                const int32_t* __restrict__ idx, float* __restrict__ acc, int B, int T, int Hq, int Hkv, int top_k,
                float scale_log2, const int32_t* __restrict__ cu_in, const int* __restrict__ redo_count,
                const int* __restrict__ redo_list) {
  using RS = RedoSmem<DK>;
  const int32_t* cu = VARLEN ? cu_in : nullptr;
  extern __shared__ __align__(16) uint8_t rsm[];
  float* sS = reinterpret_cast<float*>(rsm + RS::kScores);
  float* sQ = reinterpret_cast<float*>(rsm + RS::kQ);
  int* sU = reinterpret_cast<int*>(rsm + RS::kKeys);
  float* sRed = reinterpret_cast<float*>(rsm + RS::kRed);   // [16 slices][16 heads], then [16] maxima, [16] sums
  int* sN = reinterpret_cast<int*>(sRed + 2 * kG * kG);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = *redo_count;
  for (int i = blockIdx.x; i < n; i += gridDim.x) {
    const long it = redo_list[i];
    const int g = (int)(it / ((long)B * T));
    const int bt = (int)(it % ((long)B * T));
    const int b = bt / T, t = bt % T;
    const size_t base = VARLEN ? (size_t)seq_base(cu, b, T) : (size_t)b * T;
    const size_t qrow = ((base + t) * Hq + (size_t)g * kG);
    __syncthreads();   // the previous item is done with shared memory
    for (int x = tid; x < kG * DK; x += kRedoThreads) sQ[x] = __bfloat162float(q[qrow * DK + x]);
    if (tid == 0) {   // the key positions: the chosen blocks' tokens u <= t
      int nk = 0;
      for (int jj = 0; jj < top_k; ++jj) {
        const int j = idx[(((size_t)b * Hkv + g) * T + t) * top_k + jj];
        if (j < 0) break;
        const int jb = min(j, t / kBlk);
        for (int u = jb * kBlk; u < jb * kBlk + kBlk && u <= t; ++u) sU[nk++] = u;
      }
      *sN = nk;
    }
    __syncthreads();
    const int nk = *sN;
    // scores, scaled to log2 units: warp per key, lane = (head, half of the dot product)
    {
      const int h = lane & 15, half = lane >> 4;
      for (int e = warp; e < nk; e += kRedoThreads / 32) {
        const __nv_bfloat16* kr = k + ((base + sU[e]) * Hkv + g) * DK;
        float a = 0.f;
        for (int c = half * (DK / 2); c < (half + 1) * (DK / 2); ++c) a += sQ[h * DK + c] * __bfloat162float(kr[c]);
        a += __shfl_xor_sync(0xffffffffu, a, 16);
        if (half == 0) sS[e * kG + h] = a * scale_log2;
      }
    }
    __syncthreads();
    // per head: the largest score, then p = 2^(s - max) in place and the row sum
    {
      const int h = tid & 15, sl = tid >> 4;   // 16 slices of the keys
      float mx = -INFINITY;
      for (int e = sl; e < nk; e += 16) mx = fmaxf(mx, sS[e * kG + h]);
      sRed[sl * kG + h] = mx;
      __syncthreads();
      if (tid < kG) {
        float m2 = -INFINITY;
        for (int x = 0; x < 16; ++x) m2 = fmaxf(m2, sRed[x * kG + tid]);
        sRed[kG * kG + tid] = m2;
      }
      __syncthreads();
      const float m2 = sRed[kG * kG + h];
      float l = 0.f;
      for (int e = sl; e < nk; e += 16) {
        const float pr = exp2f(sS[e * kG + h] - m2);
        sS[e * kG + h] = pr;
        l += pr;
      }
      __syncthreads();
      sRed[sl * kG + h] = l;
      __syncthreads();
      if (tid < kG) {
        float l2 = 0.f;
        for (int x = 0; x < 16; ++x) l2 += sRed[x * kG + tid];
        sRed[kG * kG + kG + tid] = l2;
      }
      __syncthreads();
    }
    // o_slc: thread = (head, 8 value columns)
    {
      const int h = tid >> 4, d0 = (tid & 15) * (DV / 16);
      float o[DV / 16];
#pragma unroll
      for (int x = 0; x < DV / 16; ++x) o[x] = 0.f;
      for (int e = 0; e < nk; ++e) {
        const float pr = sS[e * kG + h];
        const __nv_bfloat16* vr = v + ((base + sU[e]) * Hkv + g) * DV + d0;
#pragma unroll
        for (int x = 0; x < DV / 16; ++x) o[x] += pr * __bfloat162float(vr[x]);
      }
      const float L = sRed[kG * kG + kG + h];
      const float gs = __bfloat162float(gates[(qrow + h) * 3 + 1]);
      const float scl = L > 0.f ? gs / L : 0.f;
      float* ar = acc + (qrow + h) * DV + d0;
#pragma unroll
      for (int x = 0; x < DV / 16; ++x) ar[x] += scl * o[x];
    }
  }
}

template <int DK, int DV>
cudaError_t launch_tc(const FwdArgs& a, cudaStream_t st) {
  using SM = Smem<DK, DV>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(slc_attn_tc_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(slc_attn_tc_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SM::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(slc_redo_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)RedoSmem<DK>::kBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(slc_redo_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)RedoSmem<DK>::kBytes);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  CUtensorMap mk, mv, mq;
  const uint64_t dk3[3] = {(uint64_t)DK, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sk3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hkv * DK * 2};
  const uint64_t dv3[3] = {(uint64_t)DV, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sv3[2] = {(uint64_t)DV * 2, (uint64_t)a.Hkv * DV * 2};
  const uint32_t box[3] = {64, 1, kBlk};
  const uint64_t dq3[3] = {(uint64_t)DK, (uint64_t)a.Hq, (uint64_t)a.total};
  const uint64_t sq3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hq * DK * 2};
  const uint32_t qbox[3] = {64, (uint32_t)kG, 1};
  if (!make_tmap_bf16(&mk, a.k, 3, dk3, sk3, box) || !make_tmap_bf16(&mv, a.v, 3, dv3, sv3, box) ||
      !make_tmap_bf16(&mq, a.q, 3, dq3, sq3, qbox))
    return cudaErrorInvalidValue;
  const int sms = sm_count();
  const long items = (long)a.Hkv * a.B * a.T;
  const int grid = (int)(items < sms ? items : sms);
  auto kernel = a.cu ? slc_attn_tc_kernel<DK, DV, true> : slc_attn_tc_kernel<DK, DV, false>;
  kernel<<<grid, kThreads, SM::kAlloc, st>>>(mk, mv, mq, static_cast<const __nv_bfloat16*>(a.gates), a.idx, a.acc,
                                             a.B, a.T, a.Hq, a.Hkv, a.top_k, a.scale_log2, a.cu, a.redo_count,
                                             a.redo_list, a.err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // the listed items (normally none: the CTAs read a zero count and return)
  auto redo = a.cu ? slc_redo_kernel<DK, DV, true> : slc_redo_kernel<DK, DV, false>;
  redo<<<grid, kRedoThreads, RedoSmem<DK>::kBytes, st>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), static_cast<const __nv_bfloat16*>(a.gates), a.idx, a.acc, a.B, a.T,
      a.Hq, a.Hkv, a.top_k, a.scale_log2, a.cu, a.redo_count, a.redo_list);
  return cudaGetLastError();
}
}  // namespace

bool slc_attn_tc_supported(const FwdArgs& a) {
  return a.err != nullptr && a.redo_count != nullptr && a.redo_list != nullptr && a.G == 16 && a.dv == 128 &&
         (a.dk == 128 || a.dk == 192) && a.top_k <= 32;
}

cudaError_t launch_slc_attn_tc(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192 && a.dv == 128) return launch_tc<192, 128>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch_tc<128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
