// K3, streaming version: selected-block attention fed by TMA
// ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5: the top-k blocks are expanded to
// all their tokens; §10: the group's heads share every loaded block).
//
// Persistent CTAs (one per SM) walk the (KV group, batch, token) items, group-major
// so that the CTAs running at the same time share one group's K/V in L2.  Each CTA
// runs two independent pipelines on alternate items.  In a pipeline, one warp is the
// TMA producer: for every chosen block of every item it copies the whole 64-token K
// and V block (128-byte swizzle, 64-column boxes) into a 2-slot ring of 40 KB slots.
// Four consumer warps share each block: warp w computes the scores of keys 16w..16w+15
// with the group's G <= 16 heads as the 16 rows of warp-level m16n8k16 MMAs, writes
// its columns of the block's P[16 heads][64 keys] (bf16) to shared memory, and after
// one group barrier multiplies the whole P by value columns w*DV/4 .. (w+1)*DV/4 - 1.
// The softmax reference of a row is shared by the four warps and moves only when a
// score exceeds it by 2^8 (decided in that same barrier), so the warps' row sums add
// directly and the item ends without merging partial outputs.  The ring runs across
// item boundaries, so the loads of the next token overlap the end of this one.
//
// The producer also brings each item's queries (the group's 16 head rows, 128-byte
// swizzled boxes) into a 2-slot buffer by TMA; the consumer warps take their MMA operand
// fragments from there with ldmatrix, once per item.
//
// Slot release: the consumers read a slot with ldmatrix (generic proxy) and the
// producer refills it with TMA (async proxy).  A proxy fence before each release
// orders the reads before the refill; without it a refill was seen to overwrite the
// last value columns a warp read from the slot (about one item in 10^5-10^6).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
// consumer warps per pipeline: each takes 64/n keys of a block and DV/n value columns.
// (Eight, at a 96-register cap for 18 warps, spilled and ran 1.5x slower than four.)
template <int DV> constexpr int consumers() { return 4; }
constexpr int kGroups = 2;                          // independent pipelines per CTA
template <int DV> constexpr int threads() { return kGroups * (consumers<DV>() + 1) * 32; }
constexpr int kBlk = 64;
constexpr int kSlots = 2;                           // ring slots per group
constexpr int kCtasPerSm = 1;
constexpr uint32_t kBox = kBlk * 128;   // one 64-row x 64-column box: 8 KB
constexpr float kSlack = 8.f;            // log2 headroom of the lazily moved softmax reference

template <int DK, int DV>
struct Smem {
  static constexpr uint32_t kSlotBytes = (DK / 64 + DV / 64) * kBox;
  static constexpr uint32_t kRing = 0;                                       // [group][slot]
  static constexpr uint32_t kQBytes = (DK / 64) * 16 * 128;                 // queries: 16 rows, DK/64 boxes
  static constexpr uint32_t kQ = kRing + kGroups * kSlots * kSlotBytes;      // [group][2]
  static constexpr uint32_t kPBytes = 16 * 128;                              // P [16 heads][64 keys] bf16
  static constexpr uint32_t kP = kQ + kGroups * 2 * kQBytes;                 // [group][2]
  static constexpr int kConsumers = consumers<DV>();
  static constexpr uint32_t kRedBytes = 2 * kConsumers * 16 * 4 + kConsumers * 4;   // [group]: maxima, sums [warp][16], flags
  static constexpr uint32_t kRed = kP + kGroups * 2 * kPBytes;
  static constexpr uint32_t kBar = kRed + kGroups * kRedBytes;
  static constexpr int kBarsPerGroup = 2 * kSlots + 4;                       // full, empty, q_full, q_empty
  static constexpr uint32_t kBytes = kBar + kGroups * kBarsPerGroup * 8;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert(kAlloc * kCtasPerSm <= 232448, "shared memory");
  static_assert(kQ % 1024 == 0 && kQBytes % 1024 == 0, "swizzled query boxes need 1 KB alignment");
};

using tc::named_sync;
using tc::vote_all;

// byte offset of (row, 16-byte chunk c of a 64-column box) in a 128-byte-swizzled box
__device__ __forceinline__ uint32_t swz(int row, int c) { return row * 128 + ((c ^ (row & 7)) << 4); }

// VARLEN: a packed batch of sequences of different lengths (cu); its own instantiation, so
// that the equal-length one keeps its plain row arithmetic.
template <int DK, int DV, bool VARLEN>
__global__ void __launch_bounds__(threads<DV>(), kCtasPerSm)
slc_attn_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_q, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ gates,
                    const int32_t* __restrict__ idx, float* __restrict__ acc, int B, int T, int Hq, int Hkv, int G,
                    int top_k, float scale_log2, int q_rows, const int32_t* __restrict__ cu_in,
                    int* __restrict__ err) {
  using SM = Smem<DK, DV>;
  const int32_t* cu = cu_in;
  constexpr int kConsumers = SM::kConsumers;
  constexpr int kKW = kBlk / kConsumers;            // keys per consumer warp: 16 or 8
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp >= kGroups * kConsumers;
  const int grp = producer ? warp - kGroups * kConsumers : warp / kConsumers;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::kBar) + grp * SM::kBarsPerGroup;
  uint64_t* empty = full + kSlots;
  uint64_t* q_full = empty + kSlots;   // [2]
  uint64_t* q_empty = q_full + 2;      // [2]
  uint8_t* ring = smem + SM::kRing + grp * kSlots * SM::kSlotBytes;
  uint8_t* qbuf = smem + SM::kQ + grp * 2 * SM::kQBytes;
  if (tid == 0) {
    uint64_t* all = reinterpret_cast<uint64_t*>(smem + SM::kBar);
    for (int gg = 0; gg < kGroups; ++gg) {
      uint64_t* b0 = all + gg * SM::kBarsPerGroup;
      for (int s = 0; s < kSlots; ++s) {
        tc::mbar_init(b0 + s, 1);
        tc::mbar_init(b0 + kSlots + s, kConsumers);
      }
      for (int s = 0; s < 2; ++s) {
        tc::mbar_init(b0 + 2 * kSlots + s, 1);
        tc::mbar_init(b0 + 2 * kSlots + 2 + s, kConsumers);
      }
    }
    tc::fence_barrier_init();
  }
  __syncthreads();
  const long total = (long)Hkv * B * T;
  const long stride = (long)gridDim.x * kGroups;
  // item it = (group, batch, token); in a variable-length batch the tokens past a
  // sequence's end are no items, and producer and consumers skip them alike
  auto next_item = [&](long it) {
    if constexpr (VARLEN)
      while (it < total && (int)(it % T) >= seq_len(cu, (int)((it / T) % B), T)) it += stride;
    return it;
  };
  const long it0 = next_item((long)blockIdx.x * kGroups + grp);
  // the row of token t of sequence b in q, k, v, gates and acc (recomputed where it is used, so
  // that nothing extra stays live across the block loop)
  auto row_of = [&](int b, int t) -> size_t {
    if constexpr (VARLEN) return (size_t)seq_base(cu, b, T) + t;
    else return (size_t)b * T + t;
  };

  if (producer) {
    // ---------------------------------------------------------------- producer
    // (the whole warp runs the loop; lane 0 issues the copies)
    if (lane == 0) {
      tc::prefetch_tmap(&tm_k);
      tc::prefetch_tmap(&tm_v);
      tc::prefetch_tmap(&tm_q);
    }
    long fill = 0, qfill = 0;
    bool ok = true;
    for (long it = it0; it < total && ok; it = next_item(it + stride), ++qfill) {
      const int g = (int)(it / ((long)B * T));
      const int bt = (int)(it % ((long)B * T));
      const int b = bt / T, t = bt % T;
      const int base = (int)row_of(b, 0);   // first row of the sequence in q, k and v
      // this item's queries: rows g*G .. g*G+q_rows-1 of token (b, t) (q_rows = min(16, Hq);
      // rows past the group are masked by the consumers, rows past the last head are
      // zero-filled by TMA)
      {
        const int qs = (int)(qfill & 1);
        ok = tc::mbar_wait(q_empty + qs, (uint32_t)(((qfill >> 1) & 1) ^ 1), err, 24);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          tc::mbar_expect_tx(q_full + qs, (uint32_t)((DK / 64) * q_rows * 128));
          for (int s = 0; s < DK / 64; ++s)
            tc::tma_load_3d(qbuf + qs * SM::kQBytes + s * 16 * 128, &tm_q, q_full + qs, s * 64, g * G, base + t);
        }
        __syncwarp();
      }
      const int mine = lane < top_k ? idx[(((size_t)b * Hkv + g) * T + t) * top_k + lane] : -1;
      for (int jj = 0; jj < top_k && ok; ++jj) {
        const int j = __shfl_sync(0xffffffffu, mine, jj);
        if (j < 0) break;
        const int jb = min(j, t / kBlk);
        const int slot = (int)(fill % kSlots);
        ok = tc::mbar_wait(empty + slot, (uint32_t)(((fill / kSlots) & 1) ^ 1), err, 21);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        if (lane == 0) {
          uint8_t* dst = ring + slot * SM::kSlotBytes;
          tc::mbar_expect_tx(full + slot, SM::kSlotBytes);
          for (int s = 0; s < DK / 64; ++s)
            tc::tma_load_3d(dst + s * kBox, &tm_k, full + slot, s * 64, g, base + jb * kBlk);
          for (int s = 0; s < DV / 64; ++s)
            tc::tma_load_3d(dst + (DK / 64 + s) * kBox, &tm_v, full + slot, s * 64, g, base + jb * kBlk);
        }
        __syncwarp();
        ++fill;
      }
    }
    if (lane == 0) {   // let copies in flight land
      for (long f = fill - 1; f >= 0 && f >= fill - kSlots; --f)
        tc::mbar_drain(full + (f % kSlots), (uint32_t)((f / kSlots) & 1));
      for (long f = qfill - 1; f >= 0 && f >= qfill - 2; --f)   // qfill = query copies issued
        tc::mbar_drain(q_full + (f & 1), (uint32_t)((f >> 1) & 1));
    }
  } else {
    // ---------------------------------------------------------------- consumers
    // Warp cw computes the scores of keys 16cw..16cw+15 of every block and, from the whole
    // block's P (shared through SMEM), the values of columns cw*DV/4 .. (cw+1)*DV/4 - 1.
    constexpr int kNt = DV / 8 / kConsumers;     // 8-column n-tiles per warp
    const int gl = lane >> 2, cq = lane & 3;
    const int cw = warp % kConsumers;
    const int gbar = 1 + grp;                    // named barrier of this group
    uint8_t* sPg = smem + SM::kP + grp * 2 * SM::kPBytes;
    float* sMx = reinterpret_cast<float*>(smem + SM::kRed + grp * SM::kRedBytes);   // [warp][row] block maxima
    float* sL = sMx + kConsumers * 16;                                                // [warp][row] row sums
    int* sFlag = reinterpret_cast<int*>(sL + kConsumers * 16);                      // [warp] no wait failed
    long use = 0, quse = 0;
    bool ok = true;
    for (long it = it0; it < total && ok; it = next_item(it + stride), ++quse) {
      const int g = (int)(it / ((long)B * T));
      const int bt = (int)(it % ((long)B * T));
      const int b = bt / T, t = bt % T;
      const int mine = lane < top_k ? idx[(((size_t)b * Hkv + g) * T + t) * top_k + lane] : -1;
      const bool rv0 = gl < G, rv1 = gl + 8 < G;
      // the item's query fragments (A operand of the q.k MMAs), from the swizzled boxes;
      // rows past the group are zeroed.  A failed wait is carried in ok into the block
      // loop's exchange, so that the group's warps leave together.
      uint32_t qf[DK / 16][4];
      {
        const int qs = (int)(quse & 1);
        ok = tc::mbar_wait(q_full + qs, (uint32_t)((quse >> 1) & 1), err, 26);
        ok = __all_sync(0xffffffffu, ok);
        const uint8_t* qb = qbuf + qs * SM::kQBytes;
        const int row = lane & 15;
#pragma unroll
        for (int ks = 0; ks < DK / 16; ++ks) {
          const int c = 2 * (ks & 3) + (lane >> 4);
          if (ok) ldsm_x4(qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], smem_u32(qb + (ks >> 2) * 16 * 128 + swz(row, c)));
          else qf[ks][0] = qf[ks][1] = qf[ks][2] = qf[ks][3] = 0u;
          if (!rv0) qf[ks][0] = qf[ks][2] = 0u;
          if (!rv1) qf[ks][1] = qf[ks][3] = 0u;
        }
        tc::fence_async_smem();   // the buffer is refilled by TMA after the release
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(q_empty + qs);
      }
      // warm L2 for what comes from DRAM later: the next item's queries and block list
      // (this pipeline's next token; the producer reads the list about two blocks ahead
      // of the consumers, too late to hide a DRAM access), and this item's accumulator
      // rows and gates
      {
        const long itn = next_item(it + stride);
        if (itn < total) {
          const int gn = (int)(itn / ((long)B * T));
          const int btn = (int)(itn % ((long)B * T));
          const char* qn = reinterpret_cast<const char*>(q + (row_of(btn / T, btn % T) * Hq + gn * G) * DK);
          constexpr int kLines = 16 * DK * 2 / 128;               // 16 heads of queries
          for (int ln = cw * 32 + lane; ln < kLines; ln += kConsumers * 32)
            if (ln < G * DK * 2 / 128) prefetch_l2(qn + ln * 128);
          if (cw == 0 && lane == 0) {
            const int bn = btn / T, tn = btn % T;
            prefetch_l2(idx + (((size_t)bn * Hkv + gn) * T + tn) * top_k);
          }
        }
        if (lane < G)
          prefetch_l2(acc + (row_of(b, t) * Hq + g * G + lane) * DV + cw * (DV / kConsumers));
        if (cw == 1 && lane < 2) {   // the G x 3 gates of this item's rows (at most two lines)
          const char* gp = reinterpret_cast<const char*>(gates + row_of(b, t) * Hq * 3 + g * G * 3);
          prefetch_l2(lane == 0 ? gp : gp + G * 3 * 2 - 1);
        }
      }
      // per row (gl, gl + 8): the softmax reference, shared by the four warps, and this
      // warp's part of the row sums; it moves only when a score exceeds it by kSlack
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      float o[kNt][4];
#pragma unroll
      for (int x = 0; x < kNt; ++x) o[x][0] = o[x][1] = o[x][2] = o[x][3] = 0.f;
      for (int jj = 0; jj < top_k; ++jj) {
        const int j = __shfl_sync(0xffffffffu, mine, jj);
        if (j < 0) break;
        const int jb = min(j, t / kBlk);
        const int slot = (int)(use % kSlots);
        ok = ok && tc::mbar_wait(full + slot, (uint32_t)((use / kSlots) & 1), err, 23);
        ok = __all_sync(0xffffffffu, ok);   // reconverge the warp before ldmatrix / mma
        const uint8_t* kb = ring + slot * SM::kSlotBytes;
        const uint8_t* vb = kb + (DK / 64) * kBox;
        const int u0 = jb * kBlk + cw * kKW;       // this warp's keys
        float s[kKW / 8][4];
#pragma unroll
        for (int x = 0; x < kKW / 8; ++x) s[x][0] = s[x][1] = s[x][2] = s[x][3] = 0.f;
        float lmx0 = -INFINITY, lmx1 = -INFINITY;
        // this warp's 16 columns of the block's P[16 heads][64 keys] (bf16, 16-byte chunks
        // XOR-swizzled by row), computed against the current reference
        uint8_t* pbuf = sPg + (use & 1) * SM::kPBytes;
        float ps0 = 0.f, ps1 = 0.f;
        auto write_p = [&]() {
          const float base0 = m0 == -INFINITY ? 0.f : m0, base1 = m1 == -INFINITY ? 0.f : m1;
          ps0 = 0.f;
          ps1 = 0.f;
#pragma unroll
          for (int x = 0; x < kKW / 8; ++x) {
            const float p00 = ex2(s[x][0] - base0), p01 = ex2(s[x][1] - base0);
            const float p10 = ex2(s[x][2] - base1), p11 = ex2(s[x][3] - base1);
            ps0 += p00 + p01;
            ps1 += p10 + p11;
            const int ch = cw * (kKW / 8) + x;
            *reinterpret_cast<uint32_t*>(pbuf + gl * 128 + ((ch ^ (gl & 7)) << 4) + 4 * cq) = pack_bf16(p00, p01);
            *reinterpret_cast<uint32_t*>(pbuf + (gl + 8) * 128 + ((ch ^ (gl & 7)) << 4) + 4 * cq) = pack_bf16(p10, p11);
          }
        };
        if (ok) {
          if constexpr (kKW == 16) {
#pragma unroll
            for (int ks = 0; ks < DK / 16; ++ks) {
              uint32_t b0, b1, b2, b3;
              const int row = cw * 16 + (lane & 7) + ((lane >> 4) << 3);
              const int c = 2 * (ks & 3) + ((lane >> 3) & 1);
              ldsm_x4(b0, b1, b2, b3, smem_u32(kb + (ks >> 2) * kBox + swz(row, c)));
              mma16816(s[0], qf[ks], b0, b1);
              mma16816(s[kKW / 8 - 1], qf[ks], b2, b3);
            }
          } else {
            // 8 keys: one ldmatrix covers two 16-wide K steps; the even and odd steps
            // accumulate separately (two dependency chains) and are added at the end
            float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < DK / 32; ++j) {
              uint32_t b0, b1, b2, b3;
              const int row = cw * 8 + (lane & 7);
              const int c = 4 * (j & 1) + (lane >> 3);
              ldsm_x4(b0, b1, b2, b3, smem_u32(kb + (j >> 1) * kBox + swz(row, c)));
              mma16816(s[0], qf[2 * j], b0, b1);
              mma16816(s2, qf[2 * j + 1], b2, b3);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) s[0][e] += s2[e];
          }
#pragma unroll
          for (int x = 0; x < kKW / 8; ++x)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int u = u0 + x * 8 + 2 * cq + e;
              const bool vis = u <= t;
              s[x][e] = vis ? s[x][e] * scale_log2 : -INFINITY;
              s[x][2 + e] = vis ? s[x][2 + e] * scale_log2 : -INFINITY;
              lmx0 = fmaxf(lmx0, s[x][e]);
              lmx1 = fmaxf(lmx1, s[x][2 + e]);
            }
          write_p();
        }
        // One decision for the group's four warps, which share P and the reference; the
        // barrier also makes every warp's P columns visible.  A failed wait takes the
        // exchange too, so that all four warps leave together (none is left at a barrier).
        if (tc::vote_any(gbar, kConsumers * 32, !ok || lmx0 > m0 + kSlack || lmx1 > m1 + kSlack)) {
          const float mx0 = warp_max4(lmx0), mx1 = warp_max4(lmx1);
          if (cq == 0) {
            sMx[cw * 16 + gl] = mx0;
            sMx[cw * 16 + gl + 8] = mx1;
          }
          if (lane == 0) sFlag[cw] = ok;
          named_sync(gbar, kConsumers * 32);
          bool all_ok = true;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) all_ok = all_ok && sFlag[w];
          if (!all_ok) {
            ok = false;
            break;
          }
          float n0 = m0, n1 = m1;
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) {
            n0 = fmaxf(n0, sMx[w * 16 + gl]);
            n1 = fmaxf(n1, sMx[w * 16 + gl + 8]);
          }
          const float c0 = n0 == -INFINITY ? 1.f : ex2(m0 - n0), c1 = n1 == -INFINITY ? 1.f : ex2(m1 - n1);
          l0 *= c0;
          l1 *= c1;
#pragma unroll
          for (int x = 0; x < kNt; ++x) {
            o[x][0] *= c0; o[x][1] *= c0; o[x][2] *= c1; o[x][3] *= c1;
          }
          m0 = n0;
          m1 = n1;
          write_p();
          named_sync(gbar, kConsumers * 32);
        }
        l0 += ps0;
        l1 += ps1;
        // O[:, this warp's columns] += P . V over the block's 64 keys
#pragma unroll
        for (int ks = 0; ks < kBlk / 16; ++ks) {
          uint32_t a[4];
          {
            const int row = lane & 15;
            const int ch = 2 * ks + (lane >> 4);
            ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(pbuf + row * 128 + ((ch ^ (row & 7)) << 4)));
          }
#pragma unroll
          for (int np = 0; np < kNt / 2; ++np) {
            const int pg = cw * (kNt / 2) + np;       // 16-column pair within the value row
            uint32_t b0, b1, b2, b3;
            const int row = ks * 16 + (lane & 15);
            const int c = 2 * (pg & 3) + (lane >> 4);
            ldsm_x4_t(b0, b1, b2, b3, smem_u32(vb + (pg >> 2) * kBox + swz(row, c)));
            mma16816(o[2 * np], a, b0, b1);
            mma16816(o[2 * np + 1], a, b2, b3);
          }
        }
        // the slot is refilled by TMA (async proxy): order this warp's ldmatrix reads
        // (generic proxy) before the release that lets the producer overwrite it
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty + slot);
        ++use;
      }
      // the row sums over the block keys of all four warps, and the output
      l0 = warp_sum4(l0);
      l1 = warp_sum4(l1);
      if (cq == 0) {
        sL[cw * 16 + gl] = l0;
        sL[cw * 16 + gl + 8] = l1;
      }
      const size_t row0 = row_of(b, t) * Hq + g * G;
      float2 prev[2][kNt];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int x = 0; x < kNt; ++x) {
          const int r = gl + 8 * hh;
          const int c = cw * (DV / kConsumers) + x * 8 + 2 * cq;
          prev[hh][x] = r < G ? *reinterpret_cast<const float2*>(acc + (row0 + r) * DV + c) : make_float2(0.f, 0.f);
        }
      ok = vote_all(gbar, kConsumers * 32, ok);
      if (!ok) break;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = gl + 8 * hh;
        if (r >= G) continue;
        float L = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) L += sL[w * 16 + r];
        const float gs = __bfloat162float(gates[(row0 + r) * 3 + 1]);
        const float scl = L > 0.f ? gs / L : 0.f;
#pragma unroll
        for (int x = 0; x < kNt; ++x) {
          const int c = cw * (DV / kConsumers) + x * 8 + 2 * cq;
          *reinterpret_cast<float2*>(acc + (row0 + r) * DV + c) =
              make_float2(prev[hh][x].x + scl * o[x][2 * hh], prev[hh][x].y + scl * o[x][2 * hh + 1]);
        }
      }
    }
  }
  __syncthreads();
}

template <int DK, int DV>
cudaError_t launch_tma(const FwdArgs& a, cudaStream_t st) {
  using SM = Smem<DK, DV>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e =
        cudaFuncSetAttribute(slc_attn_tma_kernel<DK, DV, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SM::kAlloc);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(slc_attn_tma_kernel<DK, DV, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)SM::kAlloc);
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  CUtensorMap mk, mv;
  const uint64_t dk3[3] = {(uint64_t)DK, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sk3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hkv * DK * 2};
  const uint64_t dv3[3] = {(uint64_t)DV, (uint64_t)a.Hkv, (uint64_t)a.total};
  const uint64_t sv3[2] = {(uint64_t)DV * 2, (uint64_t)a.Hkv * DV * 2};
  const uint32_t box[3] = {64, 1, kBlk};
  CUtensorMap mq;
  const uint64_t dq3[3] = {(uint64_t)DK, (uint64_t)a.Hq, (uint64_t)a.total};
  const uint64_t sq3[2] = {(uint64_t)DK * 2, (uint64_t)a.Hq * DK * 2};
  const int q_rows = a.Hq < 16 ? a.Hq : 16;   // a box is never taller than the tensor
  const uint32_t qbox[3] = {64, (uint32_t)q_rows, 1};
  if (!make_tmap_bf16(&mk, a.k, 3, dk3, sk3, box) || !make_tmap_bf16(&mv, a.v, 3, dv3, sv3, box) ||
      !make_tmap_bf16(&mq, a.q, 3, dq3, sq3, qbox))
    return cudaErrorInvalidValue;
  const int sms = sm_count();
  const long total = (long)a.Hkv * a.B * a.T;
  const long ctas = (total + kGroups - 1) / kGroups;
  const int grid = (int)(ctas < (long)sms * kCtasPerSm ? ctas : (long)sms * kCtasPerSm);
  auto kernel = a.cu ? slc_attn_tma_kernel<DK, DV, true> : slc_attn_tma_kernel<DK, DV, false>;
  kernel<<<grid, threads<DV>(), SM::kAlloc, st>>>(
      mk, mv, mq, static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.gates), a.idx, a.acc, a.B,
      a.T, a.Hq, a.Hkv, a.G, a.top_k, a.scale_log2, q_rows, a.cu, a.err);
  return cudaGetLastError();
}
}  // namespace

bool slc_attn_tma_supported(const FwdArgs& a) {
  return a.err != nullptr && a.G <= 16 && (a.dk == 64 || a.dk == 128 || a.dk == 192) && (a.dv == 64 || a.dv == 128);
}

cudaError_t launch_slc_attn_tma(const FwdArgs& a, cudaStream_t st) {
  if (a.dk == 192 && a.dv == 128) return launch_tma<192, 128>(a, st);
  if (a.dk == 128 && a.dv == 128) return launch_tma<128, 128>(a, st);
  if (a.dk == 64 && a.dv == 64) return launch_tma<64, 64>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace nsa
