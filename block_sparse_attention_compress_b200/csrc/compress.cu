// K1: block compression phi ("逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文" §5: every
// block of l tokens becomes one key and one value vector; "一文比较 Kimi 和 Deepseek 的两篇
// 稀疏注意力机制论文", "Deepseek 的论文核心点": a learned map compresses each block).
//
// out[b, i, h, :] = vec(x[b, s*i : s*i+l, h, :]) @ w, vec token-major (index r*d + c).
// As a GEMM: M = N_c windows per (b, h), N = d_out, K = l*d.  The A operand is
// never materialised: window i, k-chunk (r, c0) is read straight from x
// (each 64-wide k-chunk lies inside one token because d % 64 == 0).
// Append mode (decode with a growing cache): the CTA's rows are the sequences b instead of
// the windows, each at the one window its newest token completes (or none).  A row's
// arithmetic (k chunks in order, the same MMA fragments) does not depend on which rows share
// its CTA, so every block equals bitwise the one the full compression computes.
// MLP mode (phi as a two-layer MLP): the first layer is this GEMM with the epilogue
// GELU(acc + bias) (MLP1), stored in bf16; the second layer is this GEMM again over the hidden
// rows with a "block" of one row (l = s = 1).  Appending with the MLP: the first layer writes
// each due sequence's hidden row to a small buffer [B, H, d] (HID_OUT), and the second layer
// reads that row as a one-token block (HID_IN) and writes the cache row of the window; both
// follow the same per-row arithmetic as the full compression.
// Variable-length batch (cu != nullptr): sequence b's tokens are rows cu[b] .. cu[b+1] of x
// and its n_cmp(cu[b+1] - cu[b]) blocks go to out[b, 0 .. ); its rows from there up to nc are
// zeroed, so that a reader of whole 128-row tiles (masked past the sequence) only ever
// multiplies finite values by its zero weights.
#include "common.cuh"
#include "kernels.h"

namespace nsa {

namespace {
constexpr int kBM = 64, kBN = 64, kBK = 64, kThreads = 128;

// STAGES-deep cp.async ring of (A, W) k-chunks: 2 when the grid is large enough to hide the
// loads' latency; more for the append launch, whose few CTAs each run one long k chain.
__device__ __forceinline__ float gelu(float x) { return 0.5f * x * (1.f + erff(x * 0.70710678118654752f)); }

template <int D, int DOUT, int STAGES, bool APPEND, bool MLP1 = false, bool HID_OUT = false, bool HID_IN = false,
          bool PRE_F32 = false>
__global__ void __launch_bounds__(kThreads)
compress_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w, int T, int H,
                int l, int s, int nc, __nv_bfloat16* __restrict__ out, const int32_t* __restrict__ seqlens,
                int B, const int32_t* __restrict__ cu, const __nv_bfloat16* __restrict__ bias = nullptr,
                float* __restrict__ pre_out = nullptr) {
  extern __shared__ __align__(128) uint8_t csmem[];
  auto sA = reinterpret_cast<__nv_bfloat16(*)[kBM * kBK]>(csmem);                          // [STAGES]
  auto sB = reinterpret_cast<__nv_bfloat16(*)[kBK * kBN]>(csmem + STAGES * kBM * kBK * 2);  // [STAGES]
  __shared__ int sWin[APPEND ? kBM : 1];   // append mode: the window of each row's sequence, or -1
  using Swz = SwzTile<kBK>;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
  constexpr bool app = APPEND;
  const int bh = blockIdx.z, b = app ? 0 : bh / H, h = app ? bh : bh % H;
  static_assert(APPEND || (!HID_OUT && !HID_IN), "the hidden row buffer is an append-mode layout");
  const int nk = (HID_IN ? 1 : l) * D / kBK;
  // full mode: the first token row of sequence b and its number of blocks
  int base = 0, nc_b = nc;
  if constexpr (!APPEND) {
    base = seq_base(cu, b, T);
    const int L = seq_len(cu, b, T);
    nc_b = L < l ? 0 : min(nc, (L - l) / s + 1);
    if (i0 >= nc_b) {   // the whole CTA: no block of this sequence, zero its rows
      for (int e = tid; e < kBM * (kBN / 8); e += kThreads) {
        const int i = i0 + e / (kBN / 8), c = (e % (kBN / 8)) * 8;
        if (i >= nc) continue;
        const size_t o = (((size_t)b * nc + i) * H + h) * DOUT + n0 + c;
        if constexpr (PRE_F32) {
          *reinterpret_cast<float4*>(pre_out + o) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(pre_out + o + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          *reinterpret_cast<uint4*>(out + o) = make_uint4(0, 0, 0, 0);
        }
      }
      return;
    }
  }
  if constexpr (APPEND) {
    if (tid < kBM) {
      const int bb = i0 + tid;
      const int L = bb < B ? min(seqlens[bb], T) : 0;
      sWin[tid] = (L >= l && (L - l) % s == 0 && (L - l) / s < nc) ? (L - l) / s : -1;
    }
    __syncthreads();
  }
  // the source row of CTA row `row`: (sequence, window) in append mode, else (b, i0 + row)
  auto row_seq = [&](int row) { return app ? i0 + row : b; };
  auto row_win = [&](int row) { return app ? sWin[row] : (i0 + row < nc_b ? i0 + row : -1); };
  auto src_row = [&](int row, int i, int r) -> size_t {   // token row of x
    if constexpr (HID_IN) return (size_t)row_seq(row);   // the hidden row [B, H, d] of the sequence
    return app ? (size_t)row_seq(row) * T + (size_t)s * i + r : (size_t)base + (size_t)s * i + r;
  };

  auto load = [&](int kc, int buf) {
    const int kk0 = kc * kBK;
    const int r = kk0 / D, c0 = kk0 % D;
#pragma unroll
    for (int e = tid; e < kBM * (kBK / 8); e += kThreads) {
      const int row = e >> 3, ch = e & 7;
      const int i = row_win(row);
      const bool ok = i >= 0;
      const __nv_bfloat16* src = x + ((ok ? src_row(row, i, r) : 0) * H + h) * D + c0 + ch * 8;
      cp_async16(&sA[buf][Swz::offset(row, ch)], src, ok);
    }
#pragma unroll
    for (int e = tid; e < kBK * (kBN / 8); e += kThreads) {
      const int row = e >> 3, ch = e & 7;
      const __nv_bfloat16* src = w + (size_t)(kk0 + row) * DOUT + n0 + ch * 8;
      cp_async16(&sB[buf][Swz::offset(row, ch)], src, true);
    }
  };

  float acc[kBN / 8][4];
#pragma unroll
  for (int j = 0; j < kBN / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

#pragma unroll
  for (int st = 0; st + 1 < STAGES; ++st) {
    if (st < nk) load(st, st);
    cp_async_commit();
  }
  for (int kc = 0; kc < nk; ++kc) {
    if (kc + STAGES - 1 < nk) load(kc + STAGES - 1, (kc + STAGES - 1) % STAGES);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    const int buf = kc % STAGES;
#pragma unroll
    for (int ks = 0; ks < kBK / 16; ++ks) {
      uint32_t a[4];
      {
        const int row = warp * 16 + (lane & 15);
        const int ch = 2 * ks + (lane >> 4);
        ldsm_x4(a[0], a[1], a[2], a[3], smem_u32(&sA[buf][Swz::offset(row, ch)]));
      }
#pragma unroll
      for (int np = 0; np < kBN / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        const int krow = ks * 16 + (lane & 15);
        const int ch = 2 * np + (lane >> 4);
        ldsm_x4_t(b0, b1, b2, b3, smem_u32(&sB[buf][Swz::offset(krow, ch)]));
        mma16816(acc[2 * np], a, b0, b1);
        mma16816(acc[2 * np + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  const int gl = lane >> 2, cq = lane & 3;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int row = warp * 16 + gl + half * 8;
    const int i = row_win(row);
    if (i < 0) {
      if (!APPEND && i0 + row < nc) {   // past this sequence's blocks: zeros
        const size_t o = (((size_t)b * nc + i0 + row) * H + h) * DOUT + n0;
#pragma unroll
        for (int j = 0; j < kBN / 8; ++j) {
          if constexpr (PRE_F32) *reinterpret_cast<float2*>(pre_out + o + j * 8 + 2 * cq) = make_float2(0.f, 0.f);
          else *reinterpret_cast<uint32_t*>(out + o + j * 8 + 2 * cq) = 0u;
        }
      }
      continue;
    }
    if constexpr (PRE_F32) {   // the first layer's pre-activation acc + bias, kept in fp32
      float* dstf = pre_out + (((size_t)row_seq(row) * nc + i) * H + h) * DOUT + n0;
#pragma unroll
      for (int j = 0; j < kBN / 8; ++j) {
        const int col = n0 + j * 8 + 2 * cq;
        *reinterpret_cast<float2*>(dstf + j * 8 + 2 * cq) =
            make_float2(acc[j][2 * half] + __bfloat162float(bias[col]), acc[j][2 * half + 1] + __bfloat162float(bias[col + 1]));
      }
      continue;
    }
    __nv_bfloat16* dst = out + (((size_t)row_seq(row) * (HID_OUT ? 1 : nc) + (HID_OUT ? 0 : i)) * H + h) * DOUT + n0;
#pragma unroll
    for (int j = 0; j < kBN / 8; ++j) {
      float v0 = acc[j][2 * half], v1 = acc[j][2 * half + 1];
      if constexpr (MLP1) {
        const int col = n0 + j * 8 + 2 * cq;
        v0 = gelu(v0 + __bfloat162float(bias[col]));
        v1 = gelu(v1 + __bfloat162float(bias[col + 1]));
      }
      *reinterpret_cast<uint32_t*>(dst + j * 8 + 2 * cq) = pack_bf16(v0, v1);
    }
  }
}

constexpr size_t smem_bytes(int stages) { return (size_t)stages * (kBM * kBK + kBK * kBN) * 2; }

template <int D>
cudaError_t launch(const void* x, const void* w, int B, int T, int H, int l, int s, int nc, void* out,
                   cudaStream_t st, const int32_t* cu) {
  dim3 grid((nc + kBM - 1) / kBM, D / kBN, B * H);
  compress_kernel<D, D, 2, false><<<grid, kThreads, smem_bytes(2), st>>>(static_cast<const __nv_bfloat16*>(x),
                                                   static_cast<const __nv_bfloat16*>(w), T, H, l, s, nc,
                                                   static_cast<__nv_bfloat16*>(out), nullptr, B, cu);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_append(const void* x, const void* w, const int32_t* seqlens, int B, int Lmax, int H, int l,
                          int s, int ncmax, void* out, cudaStream_t st) {
  constexpr int kStages = 8;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    const cudaError_t e = cudaFuncSetAttribute(compress_kernel<D, D, kStages, true>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(kStages));
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid((B + kBM - 1) / kBM, D / kBN, H);
  compress_kernel<D, D, kStages, true><<<grid, kThreads, smem_bytes(kStages), st>>>(static_cast<const __nv_bfloat16*>(x),
                                                   static_cast<const __nv_bfloat16*>(w), Lmax, H, l, s, ncmax,
                                                   static_cast<__nv_bfloat16*>(out), seqlens, B, nullptr);
  return cudaGetLastError();
}
template <int D>
cudaError_t launch_append_mlp(const void* x, const void* w1, const void* b1, const void* w2, const int32_t* seqlens,
                              int B, int Lmax, int H, int l, int s, int ncmax, void* hidden, void* out,
                              cudaStream_t st) {
  constexpr int kStages = 8;
  auto k1 = compress_kernel<D, D, kStages, true, true, true, false>;
  auto k2 = compress_kernel<D, D, kStages, true, false, false, true>;
  static PerDevice attr;
  const cudaError_t e_attr = attr.once([&] {
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(kStages));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes(kStages));
    return e;
  });
  if (e_attr != cudaSuccess) return e_attr;
  dim3 grid((B + kBM - 1) / kBM, D / kBN, H);
  k1<<<grid, kThreads, smem_bytes(kStages), st>>>(static_cast<const __nv_bfloat16*>(x),
                                                   static_cast<const __nv_bfloat16*>(w1), Lmax, H, l, s, ncmax,
                                                   static_cast<__nv_bfloat16*>(hidden), seqlens, B, nullptr,
                                                   static_cast<const __nv_bfloat16*>(b1), nullptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k2<<<grid, kThreads, smem_bytes(kStages), st>>>(static_cast<const __nv_bfloat16*>(hidden),
                                                   static_cast<const __nv_bfloat16*>(w2), Lmax, H, l, s, ncmax,
                                                   static_cast<__nv_bfloat16*>(out), seqlens, B, nullptr, nullptr,
                                                   nullptr);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_mlp(const void* x, const void* w1, const void* b1, const void* w2, int B, int T, int H, int l,
                       int s, int nc, void* hidden, void* out, cudaStream_t st, const int32_t* cu) {
  dim3 grid((nc + kBM - 1) / kBM, D / kBN, B * H);
  compress_kernel<D, D, 2, false, true><<<grid, kThreads, smem_bytes(2), st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w1), T, H, l, s, nc,
      static_cast<__nv_bfloat16*>(hidden), nullptr, B, cu, static_cast<const __nv_bfloat16*>(b1));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // second layer: every hidden row is a "block" of one row
  compress_kernel<D, D, 2, false, false><<<grid, kThreads, smem_bytes(2), st>>>(
      static_cast<const __nv_bfloat16*>(hidden), static_cast<const __nv_bfloat16*>(w2), nc, H, 1, 1, nc,
      static_cast<__nv_bfloat16*>(out), nullptr, B, nullptr);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_compress_mlp(const void* x, const void* w1, const void* b1, const void* w2, int B, int T, int H,
                                int d, int l, int s, void* hidden, void* out, cudaStream_t st, const int32_t* cu) {
  const int nc = T < l ? 0 : (T - l) / s + 1;
  if (nc == 0 || B == 0 || H == 0) return cudaSuccess;
  switch (d) {
    case 64: return launch_mlp<64>(x, w1, b1, w2, B, T, H, l, s, nc, hidden, out, st, cu);
    case 128: return launch_mlp<128>(x, w1, b1, w2, B, T, H, l, s, nc, hidden, out, st, cu);
    case 192: return launch_mlp<192>(x, w1, b1, w2, B, T, H, l, s, nc, hidden, out, st, cu);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_compress_append(const void* x, const void* w, const int32_t* seqlens, int B, int Lmax, int H,
                                   int d, int l, int s, int ncmax, void* out, cudaStream_t st) {
  if (B == 0 || H == 0 || ncmax == 0) return cudaSuccess;
  switch (d) {
    case 64: return launch_append<64>(x, w, seqlens, B, Lmax, H, l, s, ncmax, out, st);
    case 128: return launch_append<128>(x, w, seqlens, B, Lmax, H, l, s, ncmax, out, st);
    case 192: return launch_append<192>(x, w, seqlens, B, Lmax, H, l, s, ncmax, out, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t launch_mlp_pre(const void* x, const void* w1, const void* b1, int B, int T, int H, int l, int s, int nc,
                           float* pre, cudaStream_t st, const int32_t* cu) {
  dim3 grid((nc + kBM - 1) / kBM, D / kBN, B * H);
  compress_kernel<D, D, 2, false, false, false, false, true><<<grid, kThreads, smem_bytes(2), st>>>(
      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(w1), T, H, l, s, nc, nullptr, nullptr, B,
      cu, static_cast<const __nv_bfloat16*>(b1), pre);
  return cudaGetLastError();
}

cudaError_t launch_compress_mlp_pre(const void* x, const void* w1, const void* b1, int B, int T, int H, int d, int l,
                                    int s, float* pre, cudaStream_t st, const int32_t* cu) {
  const int nc = T < l ? 0 : (T - l) / s + 1;
  if (nc == 0 || B == 0 || H == 0) return cudaSuccess;
  switch (d) {
    case 64: return launch_mlp_pre<64>(x, w1, b1, B, T, H, l, s, nc, pre, st, cu);
    case 128: return launch_mlp_pre<128>(x, w1, b1, B, T, H, l, s, nc, pre, st, cu);
    case 192: return launch_mlp_pre<192>(x, w1, b1, B, T, H, l, s, nc, pre, st, cu);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_compress_append_mlp(const void* x, const void* w1, const void* b1, const void* w2,
                                       const int32_t* seqlens, int B, int Lmax, int H, int d, int l, int s,
                                       int ncmax, void* hidden, void* out, cudaStream_t st) {
  if (B == 0 || H == 0 || ncmax == 0) return cudaSuccess;
  switch (d) {
    case 64: return launch_append_mlp<64>(x, w1, b1, w2, seqlens, B, Lmax, H, l, s, ncmax, hidden, out, st);
    case 128: return launch_append_mlp<128>(x, w1, b1, w2, seqlens, B, Lmax, H, l, s, ncmax, hidden, out, st);
    case 192: return launch_append_mlp<192>(x, w1, b1, w2, seqlens, B, Lmax, H, l, s, ncmax, hidden, out, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_compress(const void* x, const void* w, int B, int T, int H, int d, int l, int s, void* out,
                            cudaStream_t st, const int32_t* cu) {
  const int nc = T < l ? 0 : (T - l) / s + 1;
  if (nc == 0 || B == 0 || H == 0) return cudaSuccess;
  switch (d) {
    case 64: return launch<64>(x, w, B, T, H, l, s, nc, out, st, cu);
    case 128: return launch<128>(x, w, B, T, H, l, s, nc, out, st, cu);
    case 192: return launch<192>(x, w, B, T, H, l, s, nc, out, st, cu);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nsa
