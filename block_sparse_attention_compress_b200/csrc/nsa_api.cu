// C ABI of the NSA library: argument validation, workspace carving and the
// launch sequence on the caller's stream.  See include/nsa.h for the contract.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "../../include/nsa.h"
#include "kernels.h"

static_assert(nsa::kErrSeqRanges == NSA_CODE_CU_SEQLENS, "one code for the checked cu_seqlens");

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxTokensNsa = 65536;
constexpr int kMaxTokensDsa = 131072;  // the indexer's work grows as T^2 (six sweeps of the earlier keys)
constexpr int kMaxDsaTopk = 8192;   // 1024 selection blocks per token (top-k kept in shared memory)
constexpr int kMaxTokensMoba = 1 << 20;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int n_cmp(int T, int l, int s) { return T < l ? 0 : (T - l) / s + 1; }

bool dims_supported(int dk, int dv) {
  return (dk == 64 && dv == 64) || (dk == 128 && dv == 128) || (dk == 192 && dv == 128);
}

// Shape checks common to every entry point.  Returns NSA_OK or the error to report.
nsa_status check_cfg(const nsa_config* c) {
  if (!c) return NSA_ERR_INVALID_ARG;
  if (c->mode != NSA_MODE_NSA && c->mode != NSA_MODE_MOBA && c->mode != NSA_MODE_DSA) return NSA_ERR_INVALID_ARG;
  if (c->batch < 1 || c->seqlen < 1 || c->h_q < 1 || c->h_kv < 1 || c->d_k < 1 || c->d_v < 1)
    return NSA_ERR_INVALID_ARG;
  if (c->h_q % c->h_kv) return NSA_ERR_INVALID_ARG;
  if (c->top_k < 0 || c->sel_block < 1) return NSA_ERR_INVALID_ARG;
  // the kernels index (token, head) rows and take TMA row coordinates in 32 bits
  if ((int64_t)c->batch * c->seqlen * c->h_q > (int64_t)INT32_MAX) return NSA_ERR_UNSUPPORTED;
  if (!(c->softmax_scale >= 0.f) || std::isinf(c->softmax_scale)) return NSA_ERR_INVALID_ARG;
  if (c->mode == NSA_MODE_NSA) {
    if (c->cmp_block < 1 || c->cmp_stride < 1 || c->window < 1) return NSA_ERR_INVALID_ARG;
    if (c->score_map < NSA_MAP_TOUCH || c->score_map > NSA_MAP_OVERLAP) return NSA_ERR_INVALID_ARG;
    if (c->phi_mlp != 0 && c->phi_mlp != 1) return NSA_ERR_INVALID_ARG;
    if (c->phi_mlp &&
        (!c->w_cmp_k2 || !c->w_cmp_v2 || !c->b_cmp_k || !c->b_cmp_v || !aligned16(c->w_cmp_k2) ||
         !aligned16(c->w_cmp_v2) || !aligned16(c->b_cmp_k) || !aligned16(c->b_cmp_v)))
      return NSA_ERR_INVALID_ARG;
    if ((c->force_first != 0 && c->force_first != 1) || (c->force_local != 0 && c->force_local != 1))
      return NSA_ERR_INVALID_ARG;
    if (c->top_k < 1 || c->top_k < c->force_first + c->force_local) return NSA_ERR_INVALID_ARG;
    if (c->sel_block % c->cmp_stride) return NSA_ERR_INVALID_ARG;
    if (!c->w_cmp_k || !c->w_cmp_v || !aligned16(c->w_cmp_k) || !aligned16(c->w_cmp_v))
      return NSA_ERR_INVALID_ARG;
    if (c->cmp_block != 32 || c->cmp_stride != 16 || c->sel_block != 64) return NSA_ERR_UNSUPPORTED;
    if (c->h_q / c->h_kv > 16 || !dims_supported(c->d_k, c->d_v) || c->top_k > 32) return NSA_ERR_UNSUPPORTED;
    if (c->seqlen > kMaxTokensNsa) return NSA_ERR_UNSUPPORTED;
  } else if (c->mode == NSA_MODE_DSA) {
    if (c->top_k < 1) return NSA_ERR_INVALID_ARG;
    if (c->h_q / c->h_kv > 16 || !dims_supported(c->d_k, c->d_v) || c->top_k > kMaxDsaTopk ||
        c->seqlen > kMaxTokensDsa)
      return NSA_ERR_UNSUPPORTED;
  } else {
    if (c->h_q != c->h_kv || c->d_k != c->d_v) return NSA_ERR_INVALID_ARG;
    if (c->d_k != 128 || c->sel_block % 64 || c->top_k > 7 || c->seqlen > kMaxTokensMoba) return NSA_ERR_UNSUPPORTED;
  }
  if ((c->sel_idx_out && !aligned16(c->sel_idx_out)) || (c->kc_out && !aligned16(c->kc_out)) ||
      (c->vc_out && !aligned16(c->vc_out)))
    return NSA_ERR_INVALID_ARG;
  return NSA_OK;
}

struct FwdLayout {
  size_t err, kc, vc, idx, acc, redo, cu, hk, hv, total;   // hk, hv: the MLP's hidden rows (phi_mlp only)
};

FwdLayout forward_layout(const nsa_config* c) {
  const size_t B = c->batch, T = c->seqlen, nc = n_cmp(c->seqlen, c->cmp_block, c->cmp_stride);
  FwdLayout L{};
  size_t off = 0;
  L.err = off; off = align_up(off + 8);   // the status word, then the selected branch's redo count
  L.kc = off; off = align_up(off + B * nc * c->h_kv * c->d_k * 2);
  L.vc = off; off = align_up(off + B * nc * c->h_kv * c->d_v * 2);
  L.idx = off; off = align_up(off + B * c->h_kv * T * c->top_k * 4);
  // the branch accumulator; the backward reuses it for the fp32 Kc/Vc gradients (and, with the
  // MLP phi, the first layers' pre-activations), which are smaller
  const size_t bwd_rows = B * nc * c->h_kv * (c->d_k + c->d_v) * 4 * (c->phi_mlp ? 2 : 1);
  L.acc = off; off = align_up(off + std::max(B * T * c->h_q * c->d_v * 4, bwd_rows));
  L.redo = off; off = align_up(off + B * c->h_kv * T * 4);   // the selected branch's redo list
  L.cu = off; off = align_up(off + (B + 1) * 4);              // a packed batch's checked cu_seqlens
  if (c->phi_mlp) {
    L.hk = off; off = align_up(off + B * nc * c->h_kv * c->d_k * 2);
    L.hv = off; off = align_up(off + B * nc * c->h_kv * c->d_v * 2);
  }
  L.total = off;
  return L;
}

// DSA workspace: status word, the [B, T, top_k] chosen tokens.
struct DsaLayout {
  size_t err, sel, total;
};

DsaLayout dsa_layout(const nsa_config* c) {
  const size_t B = c->batch, T = c->seqlen;
  DsaLayout L{};
  size_t off = 0;
  L.err = off; off = align_up(off + 4);
  L.sel = off; off = align_up(off + B * T * (size_t)c->top_k * 4);
  L.total = off;
  return L;
}

size_t workspace_bytes(const nsa_config* c) {
  if (c->mode == NSA_MODE_MOBA) return nsa::moba_layout(c->batch, c->seqlen, c->h_q, c->sel_block, c->top_k).total;
  if (c->mode == NSA_MODE_DSA) return dsa_layout(c).total;
  return forward_layout(c).total;
}

nsa_status check_workspace(const nsa_config* c, size_t need) {
  if (need == 0) return NSA_OK;
  if (!c->workspace || (reinterpret_cast<uintptr_t>(c->workspace) % kAlign)) return NSA_ERR_WORKSPACE;
  if (c->workspace_bytes < need) return NSA_ERR_WORKSPACE;
  return NSA_OK;
}

// Weight, in each of its two selection blocks, of a compressed block that straddles them.
float straddle_weight(const nsa_config* c) {
  return c->score_map == NSA_MAP_CONTAINED ? 0.f : c->score_map == NSA_MAP_OVERLAP ? 0.5f : 1.f;
}

nsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NSA_OK : NSA_ERR_CUDA; }

// Records the caller's measurement events between kernels (see stage_events in nsa.h).
struct StageMarks {
  void* const* ev;
  int n, next;
  StageMarks(const nsa_config* c, int kernels)
      : ev(c->stage_events), n(c->stage_events && c->n_stage_events >= kernels + 1 ? kernels + 1 : 0), next(0) {}
  cudaError_t mark(cudaStream_t s) {
    if (next >= n) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[next++]), s);
  }
};

cudaError_t mark_trampoline(void* ctx, cudaStream_t s) { return static_cast<StageMarks*>(ctx)->mark(s); }

nsa_status moba_forward(const void* q, const void* k, const void* v, const nsa_config* cfg, void* out,
                        cudaStream_t s) {
  StageMarks marks(cfg, 5);
  nsa::MobaArgs a{};
  a.q = q; a.k = k; a.v = v; a.out = out; a.idx = cfg->sel_idx_out; a.workspace = cfg->workspace;
  a.B = cfg->batch; a.T = cfg->seqlen; a.H = cfg->h_q; a.bsz = cfg->sel_block; a.top_k = cfg->top_k;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->d_k);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.mark = mark_trampoline;
  a.mark_ctx = &marks;
  a.err = static_cast<int*>(cfg->workspace);   // the status word leads the workspace
  if (cudaMemsetAsync(a.err, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  return from_cuda(nsa::launch_moba(a, s));
}

// The launch sequence of an NSA forward: phi of K and V, compressed branch with the block
// scores and top-k, selected branch, window branch with the gated combine.  cu == nullptr is a
// batch of equal lengths (cfg->seqlen each); otherwise sequence b is rows cu[b] .. cu[b+1].
nsa_status nsa_forward_impl(const void* q, const void* k, const void* v, const void* gates, const nsa_config* cfg,
                            void* out, cudaStream_t s, const int32_t* cu, int total) {
  const FwdLayout L = forward_layout(cfg);
  auto ws = static_cast<uint8_t*>(cfg->workspace);
  nsa::FwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.gates = gates; a.out = out;
  a.B = cfg->batch; a.T = cfg->seqlen; a.Hq = cfg->h_q; a.Hkv = cfg->h_kv; a.G = cfg->h_q / cfg->h_kv;
  a.dk = cfg->d_k; a.dv = cfg->d_v; a.nc = n_cmp(cfg->seqlen, cfg->cmp_block, cfg->cmp_stride);
  a.top_k = cfg->top_k; a.window = cfg->window;
  a.force_first = cfg->force_first; a.force_local = cfg->force_local;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->d_k);
  a.scale_log2 = scale * 1.4426950408889634f;
  void* kc = cfg->kc_out ? cfg->kc_out : ws + L.kc;
  void* vc = cfg->vc_out ? cfg->vc_out : ws + L.vc;
  a.kc = kc; a.vc = vc;
  a.idx = cfg->sel_idx_out ? cfg->sel_idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  a.acc = reinterpret_cast<float*>(ws + L.acc);
  a.err = reinterpret_cast<int*>(ws + L.err);
  a.redo_count = a.err + 1;
  a.redo_list = reinterpret_cast<int*>(ws + L.redo);
  a.total = total;
  a.w_straddle = straddle_weight(cfg);

  StageMarks marks(cfg, 5);   // the first stage also holds the status word's reset and the range check
  cudaError_t e = marks.mark(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(a.err, 0, 2 * sizeof(int), s);   // the status word and the redo count
  if (cu) {   // every kernel reads the checked copy
    int32_t* safe = reinterpret_cast<int32_t*>(ws + L.cu);
    if (e == cudaSuccess) e = nsa::launch_seq_ranges(cu, a.B, a.T, total, safe, a.err, s);
    cu = safe;
  }
  a.cu = cu;
  const int l = cfg->cmp_block, st = cfg->cmp_stride;
  if (e == cudaSuccess)
    e = cfg->phi_mlp ? nsa::launch_compress_mlp(k, cfg->w_cmp_k, cfg->b_cmp_k, cfg->w_cmp_k2, a.B, a.T, a.Hkv, a.dk, l,
                                                st, ws + L.hk, kc, s, cu)
                     : nsa::launch_compress(k, cfg->w_cmp_k, a.B, a.T, a.Hkv, a.dk, l, st, kc, s, cu);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess)
    e = cfg->phi_mlp ? nsa::launch_compress_mlp(v, cfg->w_cmp_v, cfg->b_cmp_v, cfg->w_cmp_v2, a.B, a.T, a.Hkv, a.dv, l,
                                                st, ws + L.hv, vc, s, cu)
                     : nsa::launch_compress(v, cfg->w_cmp_v, a.B, a.T, a.Hkv, a.dv, l, st, vc, s, cu);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_cmp_select(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_slc_attn(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_swa_combine(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  return from_cuda(e);
}

// A variable-length batch runs on the tensor-core kernels only (their shapes).
bool varlen_supported(const nsa_config* c) {
  nsa::FwdArgs a{};
  a.B = c->batch; a.T = c->seqlen; a.Hq = c->h_q; a.Hkv = c->h_kv; a.G = c->h_q / c->h_kv;
  a.dk = c->d_k; a.dv = c->d_v; a.window = c->window; a.top_k = c->top_k;
  int dummy = 0;
  a.err = &dummy;   // the kernels' status word exists on this path
  return nsa::cmp_select_tc_supported(a) && nsa::slc_attn_tma_supported(a) && nsa::window_tc_supported(a);
}

}  // namespace

extern "C" {

const char* nsa_status_string(nsa_status s) {
  switch (s) {
    case NSA_OK: return "NSA_OK";
    case NSA_ERR_INVALID_ARG: return "NSA_ERR_INVALID_ARG";
    case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED";
    case NSA_ERR_WORKSPACE: return "NSA_ERR_WORKSPACE";
    case NSA_ERR_CUDA: return "NSA_ERR_CUDA";
    case NSA_ERR_TIMEOUT: return "NSA_ERR_TIMEOUT";
  }
  return "NSA_ERR_UNKNOWN";
}

nsa_status nsa_device_status(const void* workspace, int32_t* code_out, void* stream) {
  if (!workspace) return NSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NSA_ERR_CUDA;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return NSA_ERR_CUDA;
  if (code_out) *code_out = word;
  return word == 0 ? NSA_OK : word == NSA_CODE_CU_SEQLENS ? NSA_ERR_INVALID_ARG : NSA_ERR_TIMEOUT;
}

nsa_status nsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us, void* stream) {
  if (!workspace || workspace_bytes < sizeof(int32_t) || (reinterpret_cast<uintptr_t>(workspace) % 4) ||
      limit_us < 1 || limit_us > 1000000)
    return NSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* err = static_cast<int*>(workspace);
  if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return NSA_ERR_CUDA;
  return nsa::launch_wait_timeout(err, (uint64_t)limit_us * 1000ull, 99, s) == cudaSuccess ? NSA_OK : NSA_ERR_CUDA;
}

size_t nsa_workspace_size(const nsa_config* cfg, int decode_batch) {
  if (check_cfg(cfg) != NSA_OK || decode_batch < 0) return 0;
  if (decode_batch == 0) return workspace_bytes(cfg);
  if (cfg->mode != NSA_MODE_NSA) return 0;
  return kAlign;   // nsa_decode: the status word only
}

nsa_status nsa_compress(const void* x, const void* w, int32_t B, int32_t T, int32_t H, int32_t d, int32_t d_out,
                        int32_t l, int32_t s, void* out, void* stream) {
  if (!x || !w || !out || B < 1 || T < 1 || H < 1 || d < 1 || d_out < 1 || l < 1 || s < 1)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(out)) return NSA_ERR_INVALID_ARG;
  if (l != 32 || s != 16 || d_out != d || (d != 64 && d != 128 && d != 192)) return NSA_ERR_UNSUPPORTED;
  return from_cuda(nsa::launch_compress(x, w, B, T, H, d, l, s, out, static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_compress_append(const void* x_cache, const void* w, const int32_t* seqlens, int32_t B, int32_t Lmax,
                               int32_t H, int32_t d, int32_t d_out, int32_t l, int32_t s, void* out_cache,
                               int32_t ncmax, void* stream) {
  if (!x_cache || !w || !seqlens || !out_cache || B < 1 || Lmax < 1 || H < 1 || d < 1 || d_out < 1 || l < 1 ||
      s < 1 || ncmax < 1)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(x_cache) || !aligned16(w) || !aligned16(out_cache) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return NSA_ERR_INVALID_ARG;
  if (l != 32 || s != 16 || d_out != d || (d != 64 && d != 128 && d != 192)) return NSA_ERR_UNSUPPORTED;
  return from_cuda(nsa::launch_compress_append(x_cache, w, seqlens, B, Lmax, H, d, l, s, ncmax, out_cache,
                                               static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_compress_mlp(const void* x, const void* w1, const void* b1, const void* w2, int32_t B, int32_t T,
                            int32_t H, int32_t d, int32_t l, int32_t s, void* hidden, void* out, void* stream) {
  if (!x || !w1 || !b1 || !w2 || !hidden || !out || B < 1 || T < 1 || H < 1 || d < 1 || l < 1 || s < 1)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w1) || !aligned16(b1) || !aligned16(w2) || !aligned16(hidden) || !aligned16(out))
    return NSA_ERR_INVALID_ARG;
  if (l != 32 || s != 16 || (d != 64 && d != 128 && d != 192)) return NSA_ERR_UNSUPPORTED;
  return from_cuda(nsa::launch_compress_mlp(x, w1, b1, w2, B, T, H, d, l, s, hidden, out,
                                            static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_compress_append_mlp(const void* x_cache, const void* w1, const void* b1, const void* w2,
                                   const int32_t* seqlens, int32_t B, int32_t Lmax, int32_t H, int32_t d, int32_t l,
                                   int32_t s, void* hidden, void* out_cache, int32_t ncmax, void* stream) {
  if (!x_cache || !w1 || !b1 || !w2 || !seqlens || !hidden || !out_cache || B < 1 || Lmax < 1 || H < 1 || d < 1 ||
      l < 1 || s < 1 || ncmax < 1)
    return NSA_ERR_INVALID_ARG;
  if (!aligned16(x_cache) || !aligned16(w1) || !aligned16(b1) || !aligned16(w2) || !aligned16(hidden) ||
      !aligned16(out_cache) || (reinterpret_cast<uintptr_t>(seqlens) & 3u))
    return NSA_ERR_INVALID_ARG;
  if (l != 32 || s != 16 || (d != 64 && d != 128 && d != 192)) return NSA_ERR_UNSUPPORTED;
  return from_cuda(nsa::launch_compress_append_mlp(x_cache, w1, b1, w2, seqlens, B, Lmax, H, d, l, s, ncmax, hidden,
                                                   out_cache, static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_forward(const void* q, const void* k, const void* v, const void* gates, const nsa_config* cfg,
                       void* out, void* stream) {
  nsa_status st = check_cfg(cfg);
  if (st != NSA_OK) return st;
  if (cfg->mode == NSA_MODE_DSA) return NSA_ERR_INVALID_ARG;   // DSA runs through nsa_dsa_forward only
  if (!q || !k || !v || !out || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return NSA_ERR_INVALID_ARG;
  if (cfg->mode == NSA_MODE_NSA && (!gates || (reinterpret_cast<uintptr_t>(gates) & 1u)))
    return NSA_ERR_INVALID_ARG;
  st = check_workspace(cfg, workspace_bytes(cfg));
  if (st != NSA_OK) return st;
  if (cfg->mode == NSA_MODE_MOBA) return moba_forward(q, k, v, cfg, out, static_cast<cudaStream_t>(stream));
  return nsa_forward_impl(q, k, v, gates, cfg, out, static_cast<cudaStream_t>(stream), nullptr,
                          cfg->batch * cfg->seqlen);
}

nsa_status nsa_forward_varlen(const void* q, const void* k, const void* v, const void* gates,
                              const int32_t* cu_seqlens, int32_t total_tokens, const nsa_config* cfg, void* out,
                              void* stream) {
  nsa_status st = check_cfg(cfg);
  if (st != NSA_OK) return st;
  if (cfg->mode != NSA_MODE_NSA) return NSA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out || !gates || !cu_seqlens || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(gates) & 1u) || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u))
    return NSA_ERR_INVALID_ARG;
  if (total_tokens < 1 || (int64_t)total_tokens > (int64_t)cfg->batch * cfg->seqlen) return NSA_ERR_INVALID_ARG;
  if (!varlen_supported(cfg)) return NSA_ERR_UNSUPPORTED;
  st = check_workspace(cfg, workspace_bytes(cfg));
  if (st != NSA_OK) return st;
  return nsa_forward_impl(q, k, v, gates, cfg, out, static_cast<cudaStream_t>(stream), cu_seqlens, total_tokens);
}

namespace {
nsa_status backward_impl(const void* q, const void* k, const void* v, const void* gates, const int32_t* sel_idx,
                         const void* dout, const int32_t* cu, int32_t total, const nsa_config* cfg,
                         const nsa_grads& g, cudaStream_t s) {
  nsa_status st = check_cfg(cfg);
  if (st != NSA_OK) return st;
  if (cfg->mode != NSA_MODE_NSA) return NSA_ERR_UNSUPPORTED;
  const bool mlp = cfg->phi_mlp != 0;
  if (!q || !k || !v || !gates || !sel_idx || !dout || !g.dq || !g.dk || !g.dv || !g.dgates || !g.dw_k || !g.dw_v)
    return NSA_ERR_INVALID_ARG;
  if (mlp && (!g.db_k || !g.db_v || !g.dw_k2 || !g.dw_v2)) return NSA_ERR_INVALID_ARG;
  auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(g.dq) || !aligned16(g.dk) ||
      !aligned16(g.dv) || (reinterpret_cast<uintptr_t>(gates) & 1u) || !a4(sel_idx) || !a4(g.dgates) ||
      !a4(g.dw_k) || !a4(g.dw_v))
    return NSA_ERR_INVALID_ARG;
  if (mlp && (!a4(g.db_k) || !a4(g.db_v) || !a4(g.dw_k2) || !a4(g.dw_v2))) return NSA_ERR_INVALID_ARG;
  if (cu) {
    if (reinterpret_cast<uintptr_t>(cu) & 3u) return NSA_ERR_INVALID_ARG;
    if (total < 1 || (int64_t)total > (int64_t)cfg->batch * cfg->seqlen) return NSA_ERR_INVALID_ARG;
  }
  st = check_workspace(cfg, workspace_bytes(cfg));
  if (st != NSA_OK) return st;
  const FwdLayout L = forward_layout(cfg);
  auto ws = static_cast<uint8_t*>(cfg->workspace);
  nsa::BwdArgs a{};
  a.q = q; a.k = k; a.v = v; a.gates = gates; a.dout = dout; a.idx = sel_idx;
  a.w_k = cfg->w_cmp_k; a.w_v = cfg->w_cmp_v;
  a.B = cfg->batch; a.T = cfg->seqlen; a.Hq = cfg->h_q; a.Hkv = cfg->h_kv; a.G = cfg->h_q / cfg->h_kv;
  a.dk = cfg->d_k; a.dv = cfg->d_v; a.nc = n_cmp(cfg->seqlen, cfg->cmp_block, cfg->cmp_stride);
  a.top_k = cfg->top_k; a.window = cfg->window;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->d_k);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.kc = ws + L.kc; a.vc = ws + L.vc;
  int32_t* safe = cu ? reinterpret_cast<int32_t*>(ws + L.cu) : nullptr;   // the checked copy of cu
  a.dq = g.dq; a.gk = g.dk; a.gv = g.dv; a.dgates = g.dgates; a.dw_k = g.dw_k; a.dw_v = g.dw_v;
  // the Kc/Vc gradients (and the MLP's pre-activations) use the forward's accumulator region
  const size_t nkc = (size_t)a.B * a.nc * a.Hkv;
  a.gkc = reinterpret_cast<float*>(ws + L.acc);
  a.gvc = a.gkc + nkc * a.dk;
  if (mlp) {
    a.mlp = true;
    a.w_k2 = cfg->w_cmp_k2; a.w_v2 = cfg->w_cmp_v2;
    a.hid_k = ws + L.hk; a.hid_v = ws + L.hv;
    a.pre_k = a.gvc + nkc * a.dv;
    a.pre_v = a.pre_k + nkc * a.dk;
    a.dw_k2 = g.dw_k2; a.dw_v2 = g.dw_v2; a.db_k = g.db_k; a.db_v = g.db_v;
  }
  const size_t nk = (size_t)(cu ? total : a.B * a.T) * a.Hkv;   // the packed K/V rows
  const int l = cfg->cmp_block, cs = cfg->cmp_stride;
  cudaError_t e = cudaMemsetAsync(ws + L.err, 0, sizeof(int), s);
  if (cu) {
    if (e == cudaSuccess) e = nsa::launch_seq_ranges(cu, a.B, a.T, total, safe, reinterpret_cast<int*>(ws + L.err), s);
    cu = safe;
  }
  a.cu = cu;
  if (e == cudaSuccess) e = cudaMemsetAsync(g.dk, 0, nk * a.dk * 4, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(g.dv, 0, nk * a.dv * 4, s);
  if (e == cudaSuccess && nkc) e = cudaMemsetAsync(a.gkc, 0, nkc * (a.dk + a.dv) * 4, s);
  if (e == cudaSuccess && a.nc == 0) {   // no compressed block: phi's weights get no gradient
    e = cudaMemsetAsync(g.dw_k, 0, (size_t)l * a.dk * a.dk * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g.dw_v, 0, (size_t)l * a.dv * a.dv * 4, s);
  }
  if (mlp) {   // the compressed rows and hidden rows as the forward computed them, and pre in fp32
    if (e == cudaSuccess)
      e = nsa::launch_compress_mlp(k, cfg->w_cmp_k, cfg->b_cmp_k, cfg->w_cmp_k2, a.B, a.T, a.Hkv, a.dk, l, cs,
                                   ws + L.hk, ws + L.kc, s, cu);
    if (e == cudaSuccess)
      e = nsa::launch_compress_mlp(v, cfg->w_cmp_v, cfg->b_cmp_v, cfg->w_cmp_v2, a.B, a.T, a.Hkv, a.dv, l, cs,
                                   ws + L.hv, ws + L.vc, s, cu);
    if (e == cudaSuccess)
      e = nsa::launch_compress_mlp_pre(k, cfg->w_cmp_k, cfg->b_cmp_k, a.B, a.T, a.Hkv, a.dk, l, cs, a.pre_k, s, cu);
    if (e == cudaSuccess)
      e = nsa::launch_compress_mlp_pre(v, cfg->w_cmp_v, cfg->b_cmp_v, a.B, a.T, a.Hkv, a.dv, l, cs, a.pre_v, s, cu);
  } else {
    if (e == cudaSuccess) e = nsa::launch_compress(k, cfg->w_cmp_k, a.B, a.T, a.Hkv, a.dk, l, cs, ws + L.kc, s, cu);
    if (e == cudaSuccess) e = nsa::launch_compress(v, cfg->w_cmp_v, a.B, a.T, a.Hkv, a.dv, l, cs, ws + L.vc, s, cu);
  }
  if (e == cudaSuccess) e = nsa::launch_backward(a, s);
  return from_cuda(e);
}
}  // namespace

nsa_status nsa_backward(const void* q, const void* k, const void* v, const void* gates, const int32_t* sel_idx,
                        const void* dout, const nsa_config* cfg, float* dq, float* dk, float* dv, float* dgates,
                        float* dw_k, float* dw_v, void* stream) {
  if (cfg && cfg->phi_mlp) return NSA_ERR_UNSUPPORTED;   // the MLP's gradients go through nsa_backward_ex
  nsa_grads g{};
  g.dq = dq; g.dk = dk; g.dv = dv; g.dgates = dgates; g.dw_k = dw_k; g.dw_v = dw_v;
  return backward_impl(q, k, v, gates, sel_idx, dout, nullptr, 0, cfg, g, static_cast<cudaStream_t>(stream));
}

nsa_status nsa_backward_ex(const void* q, const void* k, const void* v, const void* gates, const int32_t* sel_idx,
                           const void* dout, const int32_t* cu_seqlens, int32_t total_tokens, const nsa_config* cfg,
                           const nsa_grads* grads, void* stream) {
  if (!grads) return NSA_ERR_INVALID_ARG;
  return backward_impl(q, k, v, gates, sel_idx, dout, cu_seqlens, total_tokens, cfg, *grads,
                       static_cast<cudaStream_t>(stream));
}

nsa_status nsa_dsa_forward(const void* q, const void* k, const void* v, const void* q_idx, const void* k_idx,
                           const void* w_idx, int32_t idx_heads, int32_t idx_dim, const nsa_config* cfg, void* out,
                           int32_t* sel_out, void* stream) {
  nsa_status st = check_cfg(cfg);
  if (st != NSA_OK) return st;
  if (cfg->mode != NSA_MODE_DSA) return NSA_ERR_INVALID_ARG;
  if (!q || !k || !v || !q_idx || !k_idx || !w_idx || !out) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_idx) || !aligned16(k_idx) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(w_idx) & 1u) || (sel_out && (reinterpret_cast<uintptr_t>(sel_out) & 3u)))
    return NSA_ERR_INVALID_ARG;
  if (idx_heads < 1 || idx_dim < 1) return NSA_ERR_INVALID_ARG;
  if (idx_heads > 64 || (idx_dim != 64 && idx_dim != 128)) return NSA_ERR_UNSUPPORTED;
  st = check_workspace(cfg, workspace_bytes(cfg));
  if (st != NSA_OK) return st;
  const DsaLayout L = dsa_layout(cfg);
  auto ws = static_cast<uint8_t*>(cfg->workspace);
  nsa::DsaArgs a{};
  a.q = q; a.k = k; a.v = v; a.qi = q_idx; a.ki = k_idx; a.wi = w_idx; a.out = out;
  a.sel = sel_out ? sel_out : reinterpret_cast<int32_t*>(ws + L.sel);
  a.B = cfg->batch; a.T = cfg->seqlen; a.Hq = cfg->h_q; a.Hkv = cfg->h_kv; a.G = cfg->h_q / cfg->h_kv;
  a.dk = cfg->d_k; a.dv = cfg->d_v; a.hi = idx_heads; a.di = idx_dim; a.top_k = cfg->top_k;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->d_k);
  a.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  StageMarks marks(cfg, 2);
  cudaError_t e = cudaMemsetAsync(ws + L.err, 0, sizeof(int), s);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_dsa_select(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_dsa_attn(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  return from_cuda(e);
}

nsa_status nsa_decode(const void* q, const void* k_cache, const void* v_cache, const void* kc_cache,
                      const void* vc_cache, const int32_t* seqlens, int32_t max_seqlen, const void* gates,
                      const nsa_config* cfg, void* out, void* stream) {
  nsa_status st = check_cfg(cfg);
  if (st != NSA_OK) return st;
  if (cfg->mode != NSA_MODE_NSA) return NSA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !kc_cache || !vc_cache || !seqlens || !gates || !out) return NSA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kc_cache) || !aligned16(vc_cache) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(gates) & 1u))
    return NSA_ERR_INVALID_ARG;
  if (max_seqlen < 1 || max_seqlen > cfg->seqlen) return NSA_ERR_INVALID_ARG;
  nsa::DecodeArgs a{};
  a.q = q; a.k = k_cache; a.v = v_cache; a.kc = kc_cache; a.vc = vc_cache; a.seqlens = seqlens;
  a.gates = gates; a.out = out; a.idx = cfg->sel_idx_out;
  a.B = cfg->batch; a.Lmax = cfg->seqlen; a.Ncmax = n_cmp(cfg->seqlen, cfg->cmp_block, cfg->cmp_stride);
  a.max_seqlen = max_seqlen; a.Hq = cfg->h_q; a.Hkv = cfg->h_kv; a.G = cfg->h_q / cfg->h_kv;
  a.dk = cfg->d_k; a.dv = cfg->d_v; a.top_k = cfg->top_k; a.window = cfg->window;
  a.force_first = cfg->force_first; a.force_local = cfg->force_local;
  const float scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.f / std::sqrt((float)cfg->d_k);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.w_straddle = straddle_weight(cfg);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = check_workspace(cfg, kAlign);
  if (st != NSA_OK) return st;
  StageMarks marks(cfg, 1);
  cudaError_t e = cudaMemsetAsync(cfg->workspace, 0, sizeof(int), s);
  if (e == cudaSuccess) e = marks.mark(s);
  if (e == cudaSuccess) e = nsa::launch_decode(a, s);
  if (e == cudaSuccess) e = marks.mark(s);
  return from_cuda(e);
}

}  // extern "C"
