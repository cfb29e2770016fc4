// Internal launch wrappers (host side) of the NSA kernels.  Every wrapper
// launches on `st`, returns cudaGetLastError(), and expects arguments that
// nsa_api.cu has already validated.
#pragma once
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace nsa {

// A kernel's attributes (the dynamic shared-memory limit) belong to one device: a launcher
// keeps one of these and sets its kernels' attributes the first time it runs on each device.
// `set` makes the calls and returns the first error; nothing is remembered after an error, so
// the next launch tries again.  Devices past the 64th are set on every launch.
class PerDevice {
 public:
  template <class F>
  cudaError_t once(F&& set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev >= 0 && dev < 64 ? uint64_t(1) << dev : 0;
    if (bit != 0 && (done_.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
    e = set();
    if (e == cudaSuccess && bit != 0) done_.fetch_or(bit, std::memory_order_acq_rel);
    return e;
  }

 private:
  std::atomic<uint64_t> done_{0};
};

// SMs of the current device (the persistent kernels' grid), 148 if the query fails.
inline int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    return 148;
  return sms;
}

// K1: phi for every (b, h): out [B, N_c, H, d] bf16 (l = 32, s = 16 validated).
cudaError_t launch_compress(const void* x, const void* w, int B, int T, int H, int d, int l, int s, void* out,
                            cudaStream_t st,
                            const int32_t* cu = nullptr);
// K1 with phi as a two-layer MLP: hidden = bf16(GELU(vec(block) @ w1 + b1)) [B, nc, H, d],
// out = bf16(hidden @ w2) [B, nc, H, d] (hidden width d; w1 [l*d, d], b1 [d], w2 [d, d]).
cudaError_t launch_compress_mlp(const void* x, const void* w1, const void* b1, const void* w2, int B, int T, int H,
                                int d, int l, int s, void* hidden, void* out, cudaStream_t st,
                                const int32_t* cu = nullptr);
// The MLP's first-layer pre-activation vec(block) @ w1 + b1 in fp32 [B, nc, H, d] (the backward's
// GELU derivative is taken there).
cudaError_t launch_compress_mlp_pre(const void* x, const void* w1, const void* b1, int B, int T, int H, int d, int l,
                                    int s, float* pre, cudaStream_t st, const int32_t* cu = nullptr);
// K1 for a growing cache: for each sequence b whose newest token (L = seqlens[b], clamped
// to Lmax) completes window i = (L - l)/s < ncmax, out[b, i, h, :] for every head.
cudaError_t launch_compress_append(const void* x, const void* w, const int32_t* seqlens, int B, int Lmax, int H,
                                   int d, int l, int s, int ncmax, void* out, cudaStream_t st);
// The same with phi as the two-layer MLP; hidden is scratch bf16 [B, H, d] for the due rows.
cudaError_t launch_compress_append_mlp(const void* x, const void* w1, const void* b1, const void* w2,
                                       const int32_t* seqlens, int B, int Lmax, int H, int d, int l, int s,
                                       int ncmax, void* hidden, void* out, cudaStream_t st);

struct FwdArgs {
  const void* q;      // [B, T, Hq, dk] bf16
  const void* k;      // [B, T, Hkv, dk]
  const void* v;      // [B, T, Hkv, dv]
  const void* gates;  // [B, T, Hq, 3]
  const void* kc;     // [B, nc, Hkv, dk]
  const void* vc;     // [B, nc, Hkv, dv]
  float* acc;         // [B, T, Hq, dv] fp32 scratch: gated compressed + selected outputs
  int32_t* idx;       // [B, Hkv, T, top_k]
  void* out;          // [B, T, Hq, dv] bf16
  int B, T, Hq, Hkv, G, dk, dv, nc;
  int top_k, window, force_first, force_local;
  float scale_log2;   // softmax scale * log2(e)
  int* err;           // device word, zeroed before the launches; nonzero = a bounded wait timed out
  // Weight of the compressed blocks that straddle two selection blocks (i % 4 == 3 for l = 32,
  // s = 16, b = 64) in each of the two: 1 (touch), 0 (contained) or 0.5 (overlap).  The others
  // lie inside one selection block and count fully there.
  float w_straddle = 1.f;
  // Variable-length batch: cu[b] .. cu[b+1] are sequence b's rows of q, k, v, gates, acc and out
  // (device, [B + 1], cu[0] = 0, lengths <= T); nullptr = B sequences of T tokens each.  Kc/Vc
  // and idx keep their per-sequence layouts with T as the (maximum) length.
  const int32_t* cu = nullptr;
  int total = 0;      // token rows (cu[B], or B * T)
  // (token, group) items of the selected branch to recompute exactly (see slc_attn_tc.cu): a
  // count zeroed before the launches, and the item indices ([B * Hkv * T] capacity).
  int* redo_count = nullptr;
  int* redo_list = nullptr;
};

// Status word code: the caller's cu_seqlens broke its rules (the kernels ran on clamped ranges).
constexpr int kErrSeqRanges = 200;
// The checked copy of cu_seqlens [B + 1] that the kernels of a packed batch read (one warp):
// lengths clamped to [0, T], running sum capped at total; kErrSeqRanges if it differs from cu or
// cu[B] != total.
cudaError_t launch_seq_ranges(const int32_t* cu, int B, int T, int total, int32_t* safe, int* err, cudaStream_t st);

// First row and length of sequence b in a (possibly variable-length) batch.
__device__ __forceinline__ int seq_base(const int32_t* cu, int b, int T) { return cu ? __ldg(cu + b) : b * T; }
__device__ __forceinline__ int seq_len(const int32_t* cu, int b, int T) {
  return cu ? __ldg(cu + b + 1) - __ldg(cu + b) : T;
}

// K2: compressed attention (writes acc = g_cmp * o_cmp) + group-summed block
// scores + top-k (writes idx).
cudaError_t launch_cmp_select(const FwdArgs& a, cudaStream_t st);
// K2 on tcgen05 + TMA (G == 16, d_v == 128, d_k in {128, 192}).
bool cmp_select_tc_supported(const FwdArgs& a);
cudaError_t launch_cmp_select_tc(const FwdArgs& a, cudaStream_t st);
// K3: selected-block attention (acc += g_slc * o_slc).
cudaError_t launch_slc_attn(const FwdArgs& a, cudaStream_t st);
bool slc_attn_tma_supported(const FwdArgs& a);
// K3 on tcgen05 + TMA (G == 16, d_v == 128, d_k in {128, 192}, top_k <= 32).
bool slc_attn_tc_supported(const FwdArgs& a);
cudaError_t launch_slc_attn_tc(const FwdArgs& a, cudaStream_t st);
cudaError_t launch_slc_attn_tma(const FwdArgs& a, cudaStream_t st);
// K4 + K5: sliding window and gated combine (out = bf16(acc + g_win * o_win)).
cudaError_t launch_swa_combine(const FwdArgs& a, cudaStream_t st);
// K4 + K5 in one pass on tcgen05 (G == 16, d_v == 128, d_k in {128, 192}).
bool window_tc_supported(const FwdArgs& a);
cudaError_t launch_window_tc(const FwdArgs& a, cudaStream_t st);

struct DecodeArgs {
  const void* q;        // [B, Hq, dk]
  const void* k;        // [B, Lmax, Hkv, dk]
  const void* v;        // [B, Lmax, Hkv, dv]
  const void* kc;       // [B, Ncmax, Hkv, dk]
  const void* vc;       // [B, Ncmax, Hkv, dv]
  const int32_t* seqlens;
  const void* gates;    // [B, Hq, 3]
  void* out;            // [B, Hq, dv]
  int32_t* idx;         // [B, Hkv, top_k] or null
  int B, Lmax, Ncmax, max_seqlen, Hq, Hkv, G, dk, dv;
  int top_k, window, force_first, force_local;
  float scale_log2;
  float w_straddle = 1.f;   // as in FwdArgs
};

// DSA: token-wise sparse attention behind a lightning indexer.
struct DsaArgs {
  const void* q;      // [B, T, Hq, dk]
  const void* k;      // [B, T, Hkv, dk]
  const void* v;      // [B, T, Hkv, dv]
  const void* qi;     // [B, T, hi, di] indexer queries
  const void* ki;     // [B, T, di] indexer keys
  const void* wi;     // [B, T, hi] indexer head weights
  void* out;          // [B, T, Hq, dv]
  int32_t* sel;       // [B, T, top_k] chosen tokens, ascending, -1 padded
  int B, T, Hq, Hkv, G, dk, dv, hi, di, top_k;
  float scale_log2;
};
// D1 + D2: indexer scores and the token-wise top-k, streamed (no score matrix in memory).
cudaError_t launch_dsa_select(const DsaArgs& a, cudaStream_t st);
cudaError_t launch_dsa_attn(const DsaArgs& a, cudaStream_t st);

// Backward of the NSA forward (linear phi, equal lengths).  Gradients in fp32; gk, gv, gkc, gvc
// must be zero on entry (the attention kernel adds into them).
struct BwdArgs {
  const void* q;      // [B, T, Hq, dk]
  const void* k;      // [B, T, Hkv, dk]
  const void* v;      // [B, T, Hkv, dv]
  const void* kc;     // [B, nc, Hkv, dk] phi(k), as the forward computed it
  const void* vc;     // [B, nc, Hkv, dv]
  const void* w_k;    // [l*dk, dk]
  const void* w_v;    // [l*dv, dv]
  const void* gates;  // [B, T, Hq, 3]
  const void* dout;   // [B, T, Hq, dv]
  const int32_t* idx; // [B, Hkv, T, top_k] the forward's chosen blocks
  float* dq;          // [B, T, Hq, dk]
  float* gk;          // [B, T, Hkv, dk]
  float* gv;          // [B, T, Hkv, dv]
  float* gkc;         // [B, nc, Hkv, dk] scratch
  float* gvc;         // [B, nc, Hkv, dv] scratch
  float* dgates;      // [B, T, Hq, 3]
  float* dw_k;        // [l*dk, dk]
  float* dw_v;        // [l*dv, dv]
  // phi as the two-layer MLP (mlp = true): w_k/w_v and dw_k/dw_v are then the first layer's
  bool mlp = false;
  const void* w_k2 = nullptr;   // [dk, dk] second layer
  const void* w_v2 = nullptr;
  const void* hid_k = nullptr;  // [B, nc, Hkv, dk] bf16 hidden rows, as the forward computed them
  const void* hid_v = nullptr;
  float* pre_k = nullptr;       // [B, nc, Hkv, dk] fp32 first-layer pre-activation; overwritten by dpre
  float* pre_v = nullptr;
  float* dw_k2 = nullptr;       // [dk, dk]
  float* dw_v2 = nullptr;
  float* db_k = nullptr;        // [dk]
  float* db_v = nullptr;
  // Variable-length batch (cu != nullptr): sequence b's rows of q, k, v, gates, dout, dq, dk,
  // dv and dgates are cu[b] .. cu[b+1]; idx, kc, vc and their gradients keep the [B, ...] layouts
  const int32_t* cu = nullptr;
  int B, T, Hq, Hkv, G, dk, dv, nc, top_k, window;
  float scale_log2;
};
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t st);

// K6: one decode step per sequence, all branches in one launch.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st);

// Self-test of the bounded-wait path: one wait on an mbarrier that nothing arrives at,
// which gives up after limit_ns and records `code` in *err.
cudaError_t launch_wait_timeout(int* err, uint64_t limit_ns, int code, cudaStream_t st);


struct MobaLayout {
  size_t err, kbar, idx, counts, offsets, chunks, fill, chunk_list, list, part_lse, part_o, total;
};
// Workspace carve-up of MoBA mode (each region 256-byte aligned).
MobaLayout moba_layout(int B, int T, int H, int bsz, int top_k);

struct MobaArgs {
  const void* q;        // [B, T, H, 128]
  const void* k;
  const void* v;
  void* out;            // [B, T, H, 128]
  int32_t* idx;         // [B, H, T, top_k + 1] or null (then kept in the workspace)
  void* workspace;      // moba_layout(...).total bytes
  int B, T, H, bsz, top_k;
  float scale_log2;
  cudaError_t (*mark)(void*, cudaStream_t);   // optional stage marker (measurement events)
  void* mark_ctx;
  int* err;             // status word (the workspace's first 4 bytes), zeroed by launch_moba
};

// MoBA mode: block means, selection, per-block query lists, past-block attention,
// own-block attention + merge.
cudaError_t launch_moba(const MobaArgs& a, cudaStream_t st);
// Past-block attention on tcgen05 (chunks of moba_past_tc_chunk() queries; block size a
// multiple of 128).  max_chunks bounds the chunk count written to chunks[E] on the device.
bool moba_past_tc_supported(const MobaArgs& a);
// Block selection on tcgen05 (128 queries per CTA as the MMA M, 64 block means per tile as N).
bool moba_select_tc_supported(const MobaArgs& a, int nblk);
cudaError_t launch_moba_select_tc(const MobaArgs& a, const void* kbar, int32_t* idx, int32_t* counts, int nblk,
                                  cudaStream_t st);
// Own block + merge on tcgen05 (same support condition).
cudaError_t launch_moba_own_tc(const MobaArgs& a, const int32_t* idx, const __nv_bfloat16* part_o,
                               const float* part_lse, cudaStream_t st);
int moba_past_tc_chunk();
cudaError_t launch_moba_past_tc(const MobaArgs& a, const int32_t* counts, const int32_t* offsets,
                                const int32_t* chunks, const int32_t* chunk_list, const int32_t* list,
                                __nv_bfloat16* part_o, float* part_lse, int nblk, int E, size_t max_chunks,
                                cudaStream_t st);

}  // namespace nsa
