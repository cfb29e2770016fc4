// Packed variable-length batches: the row ranges every kernel uses come from a checked copy of
// the caller's cu_seqlens, so that no contents of it can take a kernel outside the packed rows.
//
// The copy is the prefix sum of the lengths, each clamped to [0, T] and the running sum capped
// at the packed row count.  For a cu_seqlens that keeps its rules (cu[0] = 0, non-decreasing,
// every length <= T, cu[B] = total) the copy equals it; otherwise the copy differs somewhere,
// the ranges it gives are still inside [0, total), and the status word gets kErrSeqRanges.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
// one warp: the lengths of 32 sequences at a time, an inclusive scan over the lanes
__global__ void seq_ranges_kernel(const int32_t* __restrict__ cu, int B, int T, int total, int32_t* __restrict__ safe,
                                  int* __restrict__ err) {
  const int lane = threadIdx.x;
  bool bad = false;
  if (lane == 0) {
    safe[0] = 0;
    bad = __ldg(cu) != 0 || __ldg(cu + B) != total;
  }
  long long carry = 0;
  for (int b0 = 0; b0 < B; b0 += 32) {
    const int b = b0 + lane;
    long long len = 0;
    if (b < B) {
      const long long d = (long long)__ldg(cu + b + 1) - (long long)__ldg(cu + b);
      len = d < 0 ? 0 : d > T ? T : d;
    }
    long long incl = len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (b < B) {
      const long long end = carry + incl < total ? carry + incl : total;
      safe[b + 1] = (int)end;
      bad |= end != (long long)__ldg(cu + b + 1);
    }
    const long long next = carry + __shfl_sync(0xffffffffu, incl, 31);
    carry = next < total ? next : total;
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(err, 0, kErrSeqRanges);
}
}  // namespace

cudaError_t launch_seq_ranges(const int32_t* cu, int B, int T, int total, int32_t* safe, int* err, cudaStream_t st) {
  seq_ranges_kernel<<<1, 32, 0, st>>>(cu, B, T, total, safe, err);
  return cudaGetLastError();
}

}  // namespace nsa
