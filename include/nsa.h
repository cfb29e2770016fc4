/*
 * nsa.h -- C ABI of the B200 (sm_100a) Native Sparse Attention library.
 *
 * The operations are those described on these pages (cited by title and section):
 *   [NOTES] zjai.club episode notes, "逐篇讲解DeepSeek、Kimi、MiniMax注意力机制新论文
 *           （含投屏版）——“硬件上的暴力美学”", §5-§10, §13-§17.
 *   [BLOG]  sunshychen.top, "一文比较 Kimi 和 Deepseek 的两篇稀疏注意力机制论文",
 *           sections "Kimi 的论文核心点" and "Deepseek 的论文核心点".
 *   [EN]    youtublog.net/en, "Songlin Yang Explains Attention Mechanisms from
 *           DeepSeek, Kimi, and MiniMax" (paragraphs on the three branches and GQA).
 *
 * Conventions shared by every entry point
 *   - Tensors are caller-owned, contiguous, row-major device pointers whose
 *     base is 16-byte aligned.  bf16 unless stated.  The library allocates
 *     and frees nothing; scratch memory is the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  The return value reports only what the host can see:
 *     argument validation (nothing is launched when it fails), a workspace
 *     that is too small, and launch errors.  Faults inside a kernel surface
 *     at the caller's next synchronisation.
 *   - Stateless and re-entrant: concurrent calls on different streams are
 *     safe when their outputs and workspaces do not overlap.
 *   - Shapes: B batch, T tokens, H_q query heads, H_kv KV heads, G = H_q/H_kv
 *     query heads per KV head (query head h uses KV head h / G), d_k, d_v.
 */
#ifndef NSA_H_
#define NSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NSA_API __attribute__((visibility("default")))
#else
#define NSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NSA_OK = 0,
  NSA_ERR_INVALID_ARG = 1,  /* a null pointer, a bad shape or an inconsistent config */
  NSA_ERR_UNSUPPORTED = 2,  /* a legal config these kernels do not implement */
  NSA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or smaller than nsa_workspace_size() */
  NSA_ERR_CUDA = 4,         /* a kernel launch failed (cudaGetLastError) */
  NSA_ERR_TIMEOUT = 5       /* a bounded device-side wait gave up (see nsa_device_status) */
} nsa_status;

/* Status word value (nsa_device_status): the contents of cu_seqlens broke its rules. */
#define NSA_CODE_CU_SEQLENS 200

typedef enum {
  NSA_MODE_NSA = 0,   /* compressed + selected + sliding-window branches, gated sum */
  NSA_MODE_MOBA = 1,  /* MoBA: mean-pooled block keys, per-head top-k plus the own block */
  NSA_MODE_DSA = 2    /* DSA: lightning-indexer scores, token-wise top-k (nsa_dsa_forward only) */
} nsa_mode;

/* How the probabilities of the compressed blocks (span [s*i, s*i+l)) add up into the score of
 * a selection block (span [b*j, b*j+b)) when the two block sizes differ.  The method's
 * description says only that the selection scores come from the compressed attention
 * ([BLOG] "Deepseek 的论文核心点"); it fixes no mapping for l = 32, s = 16, b = 64. */
typedef enum {
  NSA_MAP_TOUCH = 0,      /* every compressed block adds its whole probability to each
                             selection block its span meets (the default) */
  NSA_MAP_CONTAINED = 1,  /* only the compressed blocks that lie inside a selection block count */
  NSA_MAP_OVERLAP = 2     /* each adds its probability times the fraction of its span inside */
} nsa_score_map;

/*
 * Problem description.  Fields marked (NSA) are ignored in MoBA mode.
 *
 *   mode          nsa_mode.
 *   batch, seqlen B and T of the prefill (nsa_forward); in nsa_decode,
 *                 `batch` is the number of sequences and `seqlen` the capacity
 *                 L_max of the caches (their second dimension).  Every mode needs
 *                 batch * seqlen * h_q <= 2^31 - 1 (the kernels index rows in 32
 *                 bits), else NSA_ERR_UNSUPPORTED.
 *   h_q, h_kv     query and KV heads; h_q % h_kv == 0.  MoBA needs h_q == h_kv.
 *   d_k, d_v      head dims.  Implemented: NSA (d_k,d_v) in {(64,64),(128,128),
 *                 (192,128)}, G <= 16, T <= 65536; MoBA d_k = d_v = 128, sel_block a
 *                 multiple of 64, T <= 2^20.
 *   cmp_block,    (NSA) compression block l and stride s ([NOTES] §5: each block
 *   cmp_stride    of l tokens becomes one key and one value).  Implemented: 32, 16.
 *   sel_block     selection block size b: 64 for NSA ([NOTES] §17: 64-token blocks,
 *                 top-16), the MoBA block size (512 in [NOTES] §17) for MoBA.
 *   top_k         NSA: blocks per (token, KV head), forced ones included (<= 32).
 *                 MoBA: past blocks per (token, head), the own block excluded (<= 7).
 *   window        (NSA) sliding window w: the last w tokens including the query.
 *   force_first,  (NSA) always select block 0 / the query's own block (0 or 1);
 *   force_local   top_k >= force_first + force_local.
 *   softmax_scale scale of q.k in every attention; 0 means 1/sqrt(d_k).
 *   w_cmp_k       (NSA) phi weights for keys, bf16 [l*d_k, d_k]: compressed key
 *                 i = vec(K[s*i : s*i+l]) @ w_cmp_k, vec token-major (index r*d+c).
 *   w_cmp_v       (NSA) phi weights for values, bf16 [l*d_v, d_v].
 *   sel_idx_out   optional int32 output of the chosen blocks: NSA [B, H_kv, T, top_k],
 *                 MoBA [B, H_q, T, top_k+1]; ascending, padded with -1.  NULL: not written.
 *   kc_out,vc_out optional bf16 outputs of the compressed keys/values
 *                 [B, N_c, H_kv, d_k|d_v], N_c = (T-l)/s+1 (0 if T < l).  NULL: kept
 *                 in the workspace.
 *   workspace,    caller-owned device scratch, 256-byte aligned, at least
 *   workspace_bytes nsa_workspace_size(cfg, 0) bytes (nsa_decode: (cfg, batch)).
 *   stage_events  optional, for measurement: an array of n_stage_events cudaEvent_t
 *   n_stage_events handles.  When n_stage_events >= (kernels launched) + 1, event 0 is
 *                 recorded on `stream` before the first kernel and event i after the
 *                 i-th, so that cudaEventElapsedTime gives each kernel's duration.
 *                 nsa_forward has 5 stages in NSA mode (phi of K, which also holds the
 *                 status word's reset and, for a packed batch, the check of cu_seqlens; phi of V,
 *                 compressed attention + selection, selected attention, window +
 *                 combine) and 5 in MoBA mode (block means, selection, query lists,
 *                 past-block attention, own block + merge); nsa_decode has 1.
 *                 NULL or too few: nothing is recorded.
 *   score_map     (NSA) nsa_score_map; 0 (NSA_MAP_TOUCH) when left zero.
 *   phi_mlp       (NSA) 0: phi is the linear map above.  1: phi is a two-layer MLP of hidden
 *                 width d ([BLOG] "Deepseek 的论文核心点": the blocks are compressed with an
 *                 MLP): for keys
 *                   hidden = bf16(GELU(vec(K[s*i : s*i+l]) @ w_cmp_k + b_cmp_k)),
 *                   compressed key i = bf16(hidden @ w_cmp_k2),
 *                 GELU(x) = x * (1 + erf(x / sqrt(2))) / 2; values alike with the _v weights.
 *                 w_cmp_k is then the first layer [l*d_k, d_k], b_cmp_k its bias bf16 [d_k],
 *                 w_cmp_k2 the second layer bf16 [d_k, d_k] (values: d_v).  An intra-block
 *                 position embedding pe [l, d] added to every block before the first layer is
 *                 exactly the bias b = vec(pe) @ w_cmp_k.  nsa_forward and
 *                 nsa_forward_varlen take phi_mlp = 1; nsa_compress_mlp and
 *                 nsa_compress_append_mlp compute the same map for a decode cache, which
 *                 nsa_decode reads like any other compressed cache.
 *   w_cmp_k2, w_cmp_v2, b_cmp_k, b_cmp_v   (NSA, phi_mlp = 1) as above, 16-byte aligned.
 */
typedef struct {
  int32_t mode;
  int32_t batch, seqlen, h_q, h_kv, d_k, d_v;
  int32_t cmp_block, cmp_stride, sel_block, top_k, window;
  int32_t force_first, force_local;
  float softmax_scale;
  const void* w_cmp_k;
  const void* w_cmp_v;
  int32_t* sel_idx_out;
  void* kc_out;
  void* vc_out;
  void* workspace;
  size_t workspace_bytes;
  void* const* stage_events;
  int32_t n_stage_events;
  int32_t score_map;
  int32_t phi_mlp;
  const void* w_cmp_k2;
  const void* w_cmp_v2;
  const void* b_cmp_k;
  const void* b_cmp_v;
} nsa_config;

/* Bytes of workspace nsa_forward (decode_batch == 0) or nsa_decode (decode_batch > 0) needs
 * for `cfg`; 0 if cfg is invalid.  The first 4 bytes of either workspace hold a status word
 * that the call zeroes and that a device-side wait which timed out sets to a nonzero code
 * (read it after synchronising to detect NSA_ERR_TIMEOUT). */
NSA_API size_t nsa_workspace_size(const nsa_config* cfg, int decode_batch);

/*
 * nsa_compress -- block compression phi ([NOTES] §5; [BLOG] "Deepseek 的论文核心点":
 * each block of l tokens is mapped to one short key or value vector).
 *   x    bf16 [B, T, H, d]      keys or values
 *   w    bf16 [l*d, d_out]      phi weights (one matrix for all heads)
 *   out  bf16 [B, N_c, H, d_out] with N_c = (T-l)/s+1; row i = vec(x[s*i : s*i+l]) @ w,
 *        accumulated in fp32, rounded once to bf16.
 * Implemented: d in {64,128,192}, d_out == d, (l, s) = (32, 16).
 */
NSA_API nsa_status nsa_compress(const void* x, const void* w, int32_t B, int32_t T, int32_t H, int32_t d,
                        int32_t d_out, int32_t l, int32_t s, void* out, void* stream);

/*
 * nsa_compress_mlp -- phi as a two-layer MLP of hidden width d ([BLOG] "Deepseek 的论文核心点":
 * the blocks are compressed with an MLP; the form is the one nsa_forward takes with
 * phi_mlp = 1).
 *   x       bf16 [B, T, H, d]       keys or values
 *   w1      bf16 [l*d, d]           first layer;  b1 bf16 [d] its bias
 *   w2      bf16 [d, d]             second layer
 *   hidden  bf16 [B, N_c, H, d]     caller-owned scratch, overwritten
 *   out     bf16 [B, N_c, H, d]     row i = bf16(bf16(GELU(vec(x[s*i : s*i+l]) @ w1 + b1)) @ w2),
 *                                   GELU(x) = x (1 + erf(x / sqrt 2)) / 2, each product
 *                                   accumulated in fp32; equal bitwise to the compressed keys
 *                                   (values) nsa_forward writes to kc_out (vc_out).
 * All pointers 16-byte aligned device memory.  Implemented: d in {64,128,192},
 * (l, s) = (32, 16).  Status codes as for nsa_compress.
 */
NSA_API nsa_status nsa_compress_mlp(const void* x, const void* w1, const void* b1, const void* w2, int32_t B,
                                    int32_t T, int32_t H, int32_t d, int32_t l, int32_t s, void* hidden, void* out,
                                    void* stream);

/*
 * nsa_forward -- prefill forward.
 *   q     bf16 [B, T, H_q, d_k]
 *   k     bf16 [B, T, H_kv, d_k]
 *   v     bf16 [B, T, H_kv, d_v]
 *   gates bf16 [B, T, H_q, 3] (NSA; order compressed, selected, window) -- per-token
 *         per-head branch weights ([NOTES] §6: each branch output is scaled by a gate
 *         computed from the current token, then the three are added).  NULL in MoBA mode.
 *   out   bf16 [B, T, H_q, d_v]
 *
 * NSA mode, for every token t and query head h (group g = h / G):
 *   o_cmp  softmax attention over the compressed blocks i with s*i+l-1 <= t ([NOTES] §5);
 *   score  per 64-token block j: sum over the group's heads and over the visible
 *          compressed blocks i whose span meets block j of their probabilities
 *          ([NOTES] §8; [BLOG] "Deepseek 的论文核心点");
 *   idx    the top_k blocks by score (forced blocks first, ties to the lower index),
 *          shared by the whole group ([NOTES] §7-§8);
 *   o_slc  softmax attention over the tokens u <= t of the chosen blocks;
 *   o_win  softmax attention over u in [t-w+1, t];
 *   out    g_cmp*o_cmp + g_slc*o_slc + g_win*o_win, rounded to bf16.
 * MoBA mode, per token t and head h ([BLOG] "Kimi 的论文核心点"; [NOTES] §16-§17):
 *   the top_k complete past blocks j < t/b by q.mean(K_j) plus the own block t/b,
 *   one softmax over their tokens u <= t.
 * cfg->mode = NSA_MODE_DSA is rejected with NSA_ERR_INVALID_ARG before anything runs
 * (DSA has its own entry point, nsa_dsa_forward).
 */
NSA_API nsa_status nsa_forward(const void* q, const void* k, const void* v, const void* gates,
                       const nsa_config* cfg, void* out, void* stream);

/*
 * nsa_forward_varlen -- prefill forward of a batch of sequences of different lengths, packed
 * one after another ([NOTES] §5-§8: every sequence is attended on its own, exactly as
 * nsa_forward computes it for that sequence alone).  NSA mode only.
 *   cu_seqlens   int32 [B + 1] device: sequence b is rows cu_seqlens[b] .. cu_seqlens[b+1]-1
 *                of q, k, v, gates and out; cu_seqlens[0] = 0, non-decreasing, every length
 *                <= cfg->seqlen (empty sequences allowed), cu_seqlens[B] = total_tokens.  The
 *                contents are checked on the device, never read by the host: the kernels take
 *                their ranges from a copy in the workspace whose lengths are clamped to
 *                [0, cfg->seqlen] and whose running sum stops at total_tokens, so that no
 *                contents take them outside the packed rows.  Contents outside the rules leave
 *                NSA_CODE_CU_SEQLENS in the status word (nsa_device_status then returns
 *                NSA_ERR_INVALID_ARG) and an output computed on the clamped ranges.
 *   total_tokens the packed row count (host), 1 <= total_tokens <= B * cfg->seqlen.
 *   q bf16 [total, H_q, d_k];  k [total, H_kv, d_k];  v [total, H_kv, d_v];
 *   gates bf16 [total, H_q, 3];  out bf16 [total, H_q, d_v].
 * cfg->batch = B and cfg->seqlen = the largest length (or any bound of it).  Per-sequence
 * outputs keep the layouts of nsa_forward with T = cfg->seqlen: kc_out/vc_out
 * [B, N_c(T), H_kv, d] (rows past N_c(length) zero), sel_idx_out [B, H_kv, T, top_k]
 * (rows past the length unwritten).  Workspace: nsa_workspace_size(cfg, 0) bytes.
 * Runs on the tensor-core kernels, which need G = 16, d_v = 128, d_k in {128, 192} and
 * cfg->seqlen <= 65536; other shapes return NSA_ERR_UNSUPPORTED.  Other status codes as for
 * nsa_forward.
 */
NSA_API nsa_status nsa_forward_varlen(const void* q, const void* k, const void* v, const void* gates,
                                      const int32_t* cu_seqlens, int32_t total_tokens, const nsa_config* cfg,
                                      void* out, void* stream);

/*
 * nsa_backward -- gradients of the NSA forward ([NOTES] §13: NSA is trained natively, forward
 * and backward).  NSA mode, linear phi (phi_mlp = 0), batch of equal lengths; nsa_backward_ex
 * takes the MLP phi and variable-length batches.
 *   q, k, v, gates  the forward's inputs (as for nsa_forward);
 *   sel_idx   int32 [B, H_kv, T, top_k]: the blocks the forward chose (its sel_idx_out).  The
 *             choice is discrete: no gradient flows through the scores and the top-k;
 *   dout      bf16 [B, T, H_q, d_v]: the gradient of the output;
 *   dq fp32 [B, T, H_q, d_k];  dk fp32 [B, T, H_kv, d_k];  dv fp32 [B, T, H_kv, d_v];
 *   dgates fp32 [B, T, H_q, 3];  dw_k fp32 [l*d_k, d_k];  dw_v fp32 [l*d_v, d_v]
 *             (all written; dk and dv include the paths through phi).
 * dq, dk, dv, dw_k and dw_v are fp32 sums taken in no fixed order (atomics across tokens, and
 * across a CTA's warps for dq), so their last bits can differ from run to run; dgates is
 * reproducible.  Workspace: nsa_workspace_size(cfg, 0) bytes, as for nsa_forward.  Status codes as for
 * nsa_forward.
 */
NSA_API nsa_status nsa_backward(const void* q, const void* k, const void* v, const void* gates,
                                const int32_t* sel_idx, const void* dout, const nsa_config* cfg, float* dq,
                                float* dk, float* dv, float* dgates, float* dw_k, float* dw_v, void* stream);

/*
 * nsa_backward_ex -- nsa_backward for every shape the forward takes: phi as the two-layer MLP
 * (cfg->phi_mlp = 1, its weights in cfg as for nsa_forward) and packed variable-length batches
 * (cu_seqlens as for nsa_forward_varlen).
 *   cu_seqlens    int32 [B + 1] on the device, or NULL for B sequences of cfg->seqlen tokens;
 *   total_tokens  the packed row count (cu_seqlens[B]) when cu_seqlens is given;
 *   q, k, v, gates, dout, and the dq, dk, dv, dgates outputs are then packed [total, ...]
 *   like the forward's; sel_idx keeps the forward's [B, H_kv, T, top_k] layout (T =
 *   cfg->seqlen, the longest sequence).
 *   grads         the outputs:
 *     dq, dk, dv, dgates, dw_k, dw_v  as for nsa_backward (with the MLP, dw_k and dw_v are the
 *                                     first layers' gradients [l*d, d]);
 *     db_k, db_v    fp32 [d_k], [d_v]      the first layers' bias gradients   } phi_mlp = 1
 *     dw_k2, dw_v2  fp32 [d_k, d_k], [d_v, d_v]  the second layers' gradients } only
 * With the MLP, the gradient goes through the second layer, GELU and the first layer:
 * dW2 = hidden^T dXc, dpre = (dXc W2^T) * GELU'(pre), db1 = sum of dpre, and dpre then takes
 * the place of dXc in the linear map's gradients; the bf16 rounding of the hidden rows is
 * passed through (its derivative taken as 1).  Order of sums and reproducibility as for
 * nsa_backward.  Status codes as for nsa_backward.
 */
typedef struct {
  float* dq;
  float* dk;
  float* dv;
  float* dgates;
  float* dw_k;
  float* dw_v;
  float* db_k;
  float* db_v;
  float* dw_k2;
  float* dw_v2;
} nsa_grads;

NSA_API nsa_status nsa_backward_ex(const void* q, const void* k, const void* v, const void* gates,
                                   const int32_t* sel_idx, const void* dout, const int32_t* cu_seqlens,
                                   int32_t total_tokens, const nsa_config* cfg, const nsa_grads* grads,
                                   void* stream);

/*
 * nsa_dsa_forward -- token-wise sparse attention behind a lightning indexer (DSA; 10100.com,
 * "机器之心PRO · 会员通讯 Week 45", "Which Attention is All You Need?", section "Linear v.s.
 * Sparse", point 6: a light indexer scores every earlier token, the k best are kept, and full
 * attention runs over them).  cfg->mode = NSA_MODE_DSA; used fields: batch, seqlen, h_q, h_kv,
 * d_k, d_v, top_k (1 .. 8192), softmax_scale, workspace.
 *   q bf16 [B, T, H_q, d_k];  k [B, T, H_kv, d_k];  v [B, T, H_kv, d_v]
 *   q_idx bf16 [B, T, idx_heads, idx_dim]   indexer queries (idx_heads 1 .. 64)
 *   k_idx bf16 [B, T, idx_dim]              indexer keys, one per token (idx_dim 64 or 128)
 *   w_idx bf16 [B, T, idx_heads]            indexer head weights
 *   out   bf16 [B, T, H_q, d_v]
 *   sel_out int32 [B, T, top_k] (optional): the chosen tokens, ascending, -1 padded.
 * For every token t: score[s] = sum_j w_idx[t, j] * ReLU(q_idx[t, j] . k_idx[s]) for s <= t
 * (fp32); the top_k keys by score (ties to the lower index; all of them when t + 1 <= top_k);
 * per query head, softmax attention over the chosen tokens (its GQA group's K/V).
 * Workspace: nsa_workspace_size(cfg, 0) bytes: a status word and the [B, T, top_k] chosen
 * tokens (no score matrix is kept: the scores are recomputed as the selection needs them).
 * Shapes: G = h_q / h_kv <= 16, (d_k, d_v) as nsa_forward, T <= 131072.  Status codes as for
 * nsa_forward.  stage_events: 2 stages (indexer + top-k, attention).
 */
NSA_API nsa_status nsa_dsa_forward(const void* q, const void* k, const void* v, const void* q_idx,
                                   const void* k_idx, const void* w_idx, int32_t idx_heads, int32_t idx_dim,
                                   const nsa_config* cfg, void* out, int32_t* sel_out, void* stream);

/*
 * nsa_decode -- one decode step per sequence ([NOTES] §13: decoding is bound by
 * the KV bytes read per step).  NSA mode only.
 *   q         bf16 [B, H_q, d_k]        the new token's queries
 *   k_cache   bf16 [B, L_max, H_kv, d_k], v_cache bf16 [B, L_max, H_kv, d_v]
 *   kc_cache  bf16 [B, N_c(L_max), H_kv, d_k], vc_cache [.., d_v]: phi of the caches
 *             (nsa_compress); only the first N_c(seqlens[b]) rows are read.
 *   seqlens   int32 [B] device: tokens in sequence b's cache including the new one
 *             (1 <= seqlens[b] <= max_seqlen); the query sits at position seqlens[b]-1.
 *             Values outside that range are clamped into it on the device.
 *   max_seqlen an upper bound of seqlens (host), 1 <= max_seqlen <= cfg->seqlen <= 65536.
 *   gates     bf16 [B, H_q, 3];  out bf16 [B, H_q, d_v].
 * cfg->batch = B, cfg->seqlen = L_max; sel_idx_out (optional) is [B, H_kv, top_k];
 * cfg->workspace: nsa_workspace_size(cfg, B) bytes (the status word).  One launch: per
 * (sequence, KV head), compressed attention with the group-summed block scores and
 * top-k, then the selected blocks and the window, then the gated sum -- the same
 * arithmetic as the last row of nsa_forward.
 */
NSA_API nsa_status nsa_decode(const void* q, const void* k_cache, const void* v_cache,
                      const void* kc_cache, const void* vc_cache, const int32_t* seqlens,
                      int32_t max_seqlen, const void* gates, const nsa_config* cfg,
                      void* out, void* stream);

/*
 * nsa_compress_append -- keeps a compressed cache current while decoding ([NOTES] §5: each
 * block of l tokens, taken every s tokens, is one compressed key/value; with a growing cache a
 * new block is complete every s tokens).
 *   x_cache  bf16 [B, Lmax, H, d]          keys (or values) of the cache
 *   w        bf16 [l*d, d_out]             phi weights, as for nsa_compress
 *   seqlens  int32 [B] device              L per sequence: tokens 0 .. L-1 are in the cache
 *   out_cache bf16 [B, ncmax, H, d_out]    the compressed cache
 * For every sequence b with L = min(seqlens[b], Lmax) >= l, (L - l) % s == 0 and
 * i = (L - l)/s < ncmax: out_cache[b, i, h, :] = vec(x_cache[b, s*i : s*i+l, h, :]) @ w for
 * every head h, the block that token L-1 completes.  No other row is written.  Each block is
 * bitwise equal to the same row of nsa_compress over the whole cache.  Call it after
 * appending token L-1 (for example before each nsa_decode); it is a no-op for the sequences
 * not at a block boundary.  Status codes as for nsa_compress (seqlens must be 4-byte aligned).
 */
NSA_API nsa_status nsa_compress_append(const void* x_cache, const void* w, const int32_t* seqlens, int32_t B,
                                       int32_t Lmax, int32_t H, int32_t d, int32_t d_out, int32_t l, int32_t s,
                                       void* out_cache, int32_t ncmax, void* stream);

/*
 * nsa_compress_append_mlp -- nsa_compress_append with phi as the two-layer MLP of
 * nsa_compress_mlp (same w1, b1, w2), so that a cache compressed by nsa_forward with
 * phi_mlp = 1 stays current while decoding.
 *   hidden   bf16 [B, H, d]   caller-owned scratch, overwritten for the sequences at a
 *                             block boundary
 * Writes out_cache[b, i, h, :] for the same (b, i) as nsa_compress_append, each bitwise
 * equal to row i of nsa_compress_mlp over the whole cache; no other row of out_cache.
 * Status codes as for nsa_compress_mlp (seqlens must be 4-byte aligned).
 */
NSA_API nsa_status nsa_compress_append_mlp(const void* x_cache, const void* w1, const void* b1, const void* w2,
                                           const int32_t* seqlens, int32_t B, int32_t Lmax, int32_t H, int32_t d,
                                           int32_t l, int32_t s, void* hidden, void* out_cache, int32_t ncmax,
                                           void* stream);

/*
 * nsa_forward_noalloc -- nsa_forward for callers that cannot allocate device memory.
 * The pages have no counterpart: this is a library convenience, not part of the method.
 *
 * Some callers are handed only their input and output buffers and cannot call
 * cudaMalloc: a plugin inside a host application that owns every device allocation,
 * or latency-critical code that must not allocate because cudaMalloc can synchronise
 * the device.  This entry point computes exactly what nsa_forward computes, with its
 * scratch in one fixed device array compiled into the library instead of the caller's
 * workspace (cfg->workspace and cfg->workspace_bytes are ignored).
 *   - Limit: the scratch array holds 32 MiB (33554432 bytes), and every GPU that loads
 *     the library keeps it until the process exits.  A problem whose
 *     nsa_workspace_size(cfg, 0) exceeds it is rejected with NSA_ERR_WORKSPACE before
 *     anything runs.  32 MiB covers, for example, 1024 tokens with 4 query heads of
 *     d_v = 64, or about 1000 tokens with 64 query heads of d_v = 128.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before
 *     any stream capture.
 *   - It allocates nothing and frees nothing.  Every call shares the one array, which
 *     keeps the previous call's contents; nothing in it needs to start at zero, since
 *     each call writes every scratch byte it later reads.  Calls whose execution
 *     overlaps on the GPU (different streams, or different host threads) race on the
 *     array: serialise them.
 *   - A device-side timeout inside a call (see nsa_device_status) is written to the
 *     array's status word; nsa_device_status_noalloc reads it.
 * Arguments, layouts and the other status codes are those of nsa_forward (NSA and MoBA
 * modes; NSA_MODE_DSA gets NSA_ERR_INVALID_ARG).  If the address lookup fails the call
 * returns NSA_ERR_CUDA and the next call on that device tries the lookup again.
 */
NSA_API nsa_status nsa_forward_noalloc(const void* q, const void* k, const void* v, const void* gates,
                                       const nsa_config* cfg, void* out, void* stream);

/*
 * nsa_device_status -- the outcome of the device-side work of earlier calls that used
 * `workspace` (the pointer passed as cfg->workspace; nsa_decode and nsa_forward zero its
 * first 4 bytes, the status word, when they start).  The tensor-core kernels bound every
 * wait on an mbarrier (one second); a wait that gives up writes a nonzero code to the word,
 * and the kernel stops issuing work and returns instead of hanging.
 * Synchronises `stream` (a cudaStream_t, NULL = the default stream), reads the word and
 * returns NSA_OK if it is 0, NSA_ERR_INVALID_ARG if it is NSA_CODE_CU_SEQLENS (the contents of
 * a variable-length call's cu_seqlens broke their rules), NSA_ERR_TIMEOUT otherwise (code_out,
 * if not NULL, receives the word: which wait gave up).  NSA_ERR_INVALID_ARG for a null workspace, NSA_ERR_CUDA if the
 * synchronisation or the copy fails.
 */
NSA_API nsa_status nsa_device_status(const void* workspace, int32_t* code_out, void* stream);

/*
 * nsa_device_status_noalloc -- nsa_device_status for the scratch array built into the
 * library, the one nsa_forward_noalloc uses on the current device (the pages have no
 * counterpart).  Synchronises `stream`, reads the array's status word (the outcome of the
 * latest nsa_forward_noalloc on this device) and returns NSA_OK or NSA_ERR_TIMEOUT, with
 * the word in code_out if not NULL.  NSA_ERR_CUDA if the address lookup, the
 * synchronisation or the copy fails.  Allocates nothing.
 */
NSA_API nsa_status nsa_device_status_noalloc(int32_t* code_out, void* stream);

/*
 * nsa_selftest_wait_timeout -- test hook for the timeout path above; no part of the method.
 * Zeroes the status word of `workspace` (device memory, at least 4 bytes, 4-byte aligned),
 * then launches one thread that waits, with a limit of limit_us microseconds (1 .. 1000000),
 * on an mbarrier that nothing arrives at.  The wait gives up, writes code 99 to the status
 * word and the kernel returns; nsa_device_status then reports NSA_ERR_TIMEOUT.  Nothing else
 * is touched and the context stays usable.  NSA_ERR_INVALID_ARG for a null, misaligned or
 * too small workspace or a limit out of range; NSA_ERR_CUDA if the launch fails.
 */
NSA_API nsa_status nsa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                             void* stream);

/* Human-readable name of a status code (static storage). */
NSA_API const char* nsa_status_string(nsa_status s);

#ifdef __cplusplus
}
#endif

#endif /* NSA_H_ */
