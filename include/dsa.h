/*
 * dsa.h -- C ABI of libdsa, the B200 (sm_100a) DeepSeek-style sparse attention hot path.
 *
 * The path has four steps, each a call below:
 *   1. dsa_index_scores   lightning-indexer scores with the causal mask
 *   2. dsa_topk           per-query top-k of those scores
 *   3. dsa_sparse_attn    attention over the selected rows of the expanded K/V
 *   4. (fused into 3)     optional headwise sigmoid / silu output gate
 * plus dsa_forward, which runs 1-4 in one call, and dsa_window_attn, the sliding-window
 * layer of the DSA-SWA-SWA hybrid block.
 *
 * Sources (web pages, cited by title and section):
 *   [AXK2]  "Transformers 中的 AXK2 架构解析：SK Telecom A.X-K2 稀疏注意力 MoE 大模型集成指南",
 *           sections "注意力前向的骨架：MLA + 显式稀疏掩码", "SK Telecom 三大改进 / 1. Sparse
 *           Gated Attention（SGA）", "AXK2Config：核心配置与默认值", "使用注意事项小结".
 *   [SPARK] Spark-X2.5-1.7B-Base headwise attention output gate walkthrough, sections
 *           "在 Spark-X2.5-1.7B-Base 中如何开启？", "前向流程：从 gate_score 计算到相乘".
 *   [DSV2]  DeepSeek-V2 attention parameter guide ("参数详解", items 4-6).
 *   [PANGU] openPangu-2.0 technical-report reading, §3.2 (SWA), §3.3 (Lightning Indexer,
 *           fixed K), §3.5 Table 1 (cost model).
 *
 * Conventions shared by every call
 *   - Every tensor is dense, row-major, last index fastest, and lives in device memory
 *     of the current CUDA device, allocated and owned by the caller.  The library never
 *     allocates, frees or synchronises; inputs are read-only; outputs are overwritten in
 *     full (including the -inf / -1 / zero padding described per call).
 *   - Calls are asynchronous: they validate their arguments on the host, enqueue kernels
 *     on `stream` and return.  Argument errors are reported before anything is launched
 *     (DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED) and leave the outputs untouched.
 *     A launch failure returns DSA_ERR_CUDA.  Waits inside kernels are bounded (about
 *     2 s); a wait that gives up records DSA_ERR_TIMEOUT in a per-device status word that
 *     dsa_device_status() reads after the stream has been synchronised.  While a timeout
 *     is recorded, later in-kernel waits give up at once; dsa_device_status(1) clears it.
 *   - Base pointers must be 16-byte aligned.  bf16 head dimensions must be multiples of
 *     8, float32 ones multiples of 4.
 *   - q_off = T - S throughout: query s of a batch row sits at key position s + q_off,
 *     i.e. the queries are the last S of the T positions (prefill: S == T; decode: S == 1).
 *   - No C++ exception crosses this boundary.  Calls on distinct streams are thread-safe.
 *     dsa_last_error() returns a thread-local text for the last failed call.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* dsa_stream_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* a null pointer, a non-positive size, an impossible shape   */
  DSA_ERR_UNSUPPORTED = 2, /* a valid shape the library has no kernel for, misalignment */
  DSA_ERR_CUDA = 3,        /* a CUDA runtime / launch error                             */
  DSA_ERR_TIMEOUT = 4,     /* a bounded in-kernel wait gave up (see dsa_device_status)  */
  DSA_ERR_INTERNAL = 5     /* an in-kernel consistency check failed                     */
} dsa_status;

/* Element types.  DSA_E4M3 (float8 e4m3, 1 byte) is an indexer input type only: q_idx and
 * k_idx of dsa_index_scores (and of dsa_forward through index_dtype). */
typedef enum { DSA_F32 = 0, DSA_BF16 = 1, DSA_E4M3 = 2 } dsa_dtype;

/* Element type of dsa_forward's indexer inputs: the attention dtype, or e4m3. */
typedef enum { DSA_INDEX_AS_DTYPE = 0, DSA_INDEX_E4M3 = 1 } dsa_index_dtype;

/* Where the indexer applies ReLU.  [AXK2] SGA prints the score as a plain weighted sum
 * (DSA_RELU_NONE, the default reading); its prose adds "then ReLU" after the weighted sum
 * (DSA_RELU_POST_SUM); DSA_RELU_PER_HEAD applies ReLU to each head's dot product before
 * weighting, the upstream DeepSeek form, offered as an option. */
typedef enum { DSA_RELU_NONE = 0, DSA_RELU_POST_SUM = 1, DSA_RELU_PER_HEAD = 2 } dsa_relu_mode;

/* Headwise output gate, [SPARK] "前向流程" step 3: sigmoid or silu of one logit per
 * (token, head), evaluated in float32; any other mode is rejected (the page's ValueError). */
typedef enum { DSA_GATE_OFF = 0, DSA_GATE_SIGMOID = 1, DSA_GATE_SILU = 2 } dsa_gate_mode;

/* How dsa_forward computes the indexer scores and the top-k: per-head scores written out and
 * selected (sections 1 and 2), the head-collapsed scores (section 1b), or the per-head
 * scores filtered inside the indexer and selected from the candidates (section 2b). */
typedef enum {
  DSA_INDEXER_PER_HEAD = 0,
  DSA_INDEXER_COLLAPSED = 1,
  DSA_INDEXER_FUSED = 2
} dsa_indexer_mode;

/* Form of the attention cache dsa_forward attends over: per-head expanded K/V (section 3)
 * or one latent row per token shared by all heads (section 3c). */
typedef enum { DSA_ATTN_EXPANDED = 0, DSA_ATTN_LATENT = 1 } dsa_attn_form;

/* Attention algorithm for dsa_forward, dsa_sparse_attn and dsa_window_attn. */
typedef enum {
  DSA_ATTN_AUTO = 0,      /* pick by the cost model (bytes gathered vs. dense tile work)  */
  DSA_ATTN_GATHER = 1,    /* gather the selected K/V rows per query (decode-shaped work) */
  DSA_ATTN_MASKED_TILE = 2 /* dense tensor-core tiles under the selection bitmask         */
} dsa_attn_algo;

/* ---------------------------------------------------------------------------------
 * 1. Lightning-indexer scores.  [AXK2] SGA: index_score[b,s,t] =
 *    sum_h weight[b,s,h] * softmax_scale * (q[b,s,h,:] . k[b,t,:]); causality is imposed
 *    while scoring.  [PANGU] §3.5 Table 1: this is the quadratic prefill term,
 *    S^2 * N_head^I * D^I.
 *
 *   q_idx   [B,S,HI,DI]  dtype       indexer queries (after their projection and RoPE)
 *   k_idx   [B,T,DI]     dtype       indexer key cache (one head, shared by all HI heads)
 *   w       [B,S,HI]     float32     per-head weights (the weights_proj output)
 *   scale   > 0, finite              softmax_scale
 *   scores  [B,S,T]      float32     out: the score for t <= s + q_off, -inf for t > s+q_off
 *
 *   Arithmetic: each head's dot product is accumulated in float32 from the dtype inputs;
 *   the score is scale * sum_h w[h] * dot_h (float32).  With integer-valued inputs and a
 *   power-of-two scale (the synthetic workloads) every intermediate is exact.
 *   Requires 1 <= HI <= 256, 1 <= DI <= 128, T >= S.
 *   dtype DSA_E4M3: q_idx and k_idx are float8 e4m3 (the upstream indexer's FP8 operands,
 *   [AXK2] SGA notes; integers in [-2, 2] are exact in e4m3), products accumulated in
 *   float32 on the tensor cores at twice the bf16 rate; HI in {16, 32}, DI == 128, else
 *   DSA_ERR_UNSUPPORTED.  The Hadamard rotation the upstream applies before quantising is
 *   the caller's (it is part of producing the inputs).
 * --------------------------------------------------------------------------------- */
dsa_status dsa_index_scores(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                            const float* w, float scale, dsa_relu_mode relu, int B, int S,
                            int T, int HI, int DI, float* scores, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 1b. Head-collapsed indexer scores.  Without a per-head ReLU the [AXK2] SGA score is
 *    linear in the queries: sum_h w[s,h] * (q[s,h,:] . k[t,:]) = k[t,:] . qc[s,:] with
 *    qc[s,:] = sum_h w[s,h] * q[s,h,:].  This entry point forms qc once per query (float32,
 *    heads in order, kept as a bf16 hi + lo pair, about 2^-17 relative precision) and
 *    scores every key against it: 1/HI of the tensor-core work of dsa_index_scores, for
 *    the same scores (identical for the integer workloads, within float32 rounding of the
 *    hi/lo split otherwise).  The per-head cost model of [PANGU] §3.5 Table 1 does not
 *    apply to it; it is reported separately.
 *
 *   Arguments as dsa_index_scores, plus a workspace of
 *   dsa_index_scores_collapsed_workspace_bytes(B, S, DI) bytes (16-byte aligned) for qc.
 *   Requires dtype DSA_BF16, DI in {64, 128} and relu != DSA_RELU_PER_HEAD (the collapse
 *   does not hold with a ReLU per head): DSA_ERR_UNSUPPORTED otherwise.
 * --------------------------------------------------------------------------------- */
size_t dsa_index_scores_collapsed_workspace_bytes(int B, int S, int DI);
dsa_status dsa_index_scores_collapsed(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                                      const float* w, float scale, dsa_relu_mode relu, int B,
                                      int S, int T, int HI, int DI, float* scores, void* ws,
                                      size_t ws_bytes, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 1c. Hadamard rotation of the indexer inputs.  [AXK2] SGA notes: the upstream indexer
 *    rotates q_I and k_I with a Hadamard transform (rotate_activation) before quantising
 *    them for FP8 scoring; the transform is orthogonal, so rotating both leaves every score
 *    unchanged while spreading the values evenly over the dimensions.
 *
 *   x, out  [rows, d]  dtype (DSA_F32 or DSA_BF16), out = x @ H / sqrt(d), H the d x d
 *           Sylvester Hadamard matrix; d in {64, 128}; out may be x (in place).
 *   Float32 arithmetic, one rounding to dtype.  Pointers 16-byte aligned.
 * --------------------------------------------------------------------------------- */
dsa_status dsa_hadamard_rotate(dsa_dtype dtype, const void* x, long long rows, int d, void* out,
                               dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 2. Per-query top-k.  [AXK2] SGA: the indexer returns int32 indices [B,S,topk];
 *    "AXK2Config" (index_topk): topk = min(index_topk, number of keys).  [PANGU] §3.3:
 *    the number of selected keys is a fixed K.
 *
 *   scores  [B,S,T]  float32   (as written by dsa_index_scores; only t <= s+q_off is read)
 *   K       >= 1               columns of idx (callers pass min(index_topk, T))
 *   idx     [B,S,K]  int32     out: the min(K, n) valid keys that come first in the order
 *                              (higher score, then lower index), n = min(T, s+q_off+1),
 *                              written in ascending key order, then -1 padding.
 *   -0.0 and +0.0 compare equal.  NaN scores give an unspecified (but in-range) selection.
 *   Exact and deterministic: a radix select on the float bit patterns, no float math.
 * --------------------------------------------------------------------------------- */
dsa_status dsa_topk(const float* scores, int B, int S, int T, int K, int32_t* idx,
                    dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 2b. Fused indexer -> top-k.  The same selection as dsa_index_scores followed by dsa_topk
 *    ([AXK2] SGA scores, [PANGU] §3.3 a fixed K per query), without writing the S x T
 *    score matrix: the indexer keeps, per query row, only the keys whose score reaches a
 *    threshold tau, and the top-k is selected exactly from those candidates.
 *
 *    tau comes from a sampled pass (every kstride-th key tile of the row, kstride =
 *    max(4, key tiles / 32)): the r-th largest sampled score, r being the sample rank the
 *    K-th key is expected at plus a six-sigma margin.  Rows with at most 2K + 1024 causal
 *    keys keep every key.  The result does not depend on the sample: when every row has
 *    at least K and at most 2K + 1024 candidates, the candidates hold every key of the row's
 *    top-k (and every key tied with its K-th), so the exact select over them is the top-k;
 *    otherwise the call runs the full-score indexer and top-k itself (on the device, no
 *    host synchronisation) and reports that in *fallback_out.  Either way idx is what
 *    dsa_index_scores + dsa_topk give, bit for bit.
 *
 *   dtype bf16; HI in {16, 32}, DI in {64, 128} (the tensor-core indexer), else
 *   DSA_ERR_UNSUPPORTED.  Other arguments as dsa_index_scores; K as dsa_topk.
 *   idx          [B,S,K_eff] int32 out, ascending, -1 padded (as dsa_topk)
 *   ws           device workspace of dsa_index_topk_workspace_bytes(B,S,T,K) bytes, 16-byte
 *                aligned (the sample, thresholds, candidate lists and the score matrix the
 *                fallback would need), owned by the caller
 *   fallback_out optional device int32: 1 if the fallback ran, else 0
 * --------------------------------------------------------------------------------- */
size_t dsa_index_topk_workspace_bytes(int B, int S, int T, int K);
dsa_status dsa_index_topk(dsa_dtype dtype, const void* q_idx, const void* k_idx,
                          const float* w, float scale, dsa_relu_mode relu, int B, int S, int T,
                          int HI, int DI, int K, int32_t* idx, void* ws, size_t ws_bytes,
                          int32_t* fallback_out, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 3+4. Sparse attention over the selected keys, with the optional headwise gate.
 *    [AXK2] "注意力前向的骨架": the selected positions form an additive mask folded with
 *    the causal mask, all other positions are -inf; the cache holds the expanded per-head
 *    K/V.  [DSV2] items 4-6: q/k heads are qk_nope + qk_rope wide, v heads v_head_dim.
 *    [SPARK] "前向流程": out[b,s,h,:] *= act(gate[b,s,h]) (act in float32).
 *
 *   q     [B,S,H,DQK]  dtype      k [B,T,H,DQK] dtype      v [B,T,H,DV] dtype
 *   idx   [B,S,K]      int32      selected keys; -1, values outside [0,T) and keys in the
 *                                 future of the query (t > s+q_off) are skipped.  A row's
 *                                 valid entries must be distinct.
 *   gate  [B,S,H]      dtype      gate logits, or NULL when gate_mode == DSA_GATE_OFF
 *   sm_scale                      softmax scale; <= 0 selects 1/sqrt(DQK)
 *   out   [B,S,H,DV]   dtype      out: softmax-weighted sum of the selected v rows (float32
 *                                 accumulation, one rounding to dtype, gate applied before
 *                                 that rounding); a row with no valid key gets zeros.
 *   algo                          DSA_ATTN_GATHER gathers each query's selected K/V rows
 *                                 (all heads share the index set, so one key is one
 *                                 contiguous K row and one V row); DSA_ATTN_MASKED_TILE runs
 *                                 dense tensor-core tiles of 128 queries x 128 keys under the
 *                                 selection bitmask, which is what the page describes (dense
 *                                 attention with the additive sparse mask); DSA_ATTN_AUTO
 *                                 picks by the cost model (gathered bytes vs. dense flops).
 *                                 Both give the same result within rounding.  The masked
 *                                 tile needs bf16, DQK in {128, 192}, DV == 128.
 *   ws / ws_bytes                 scratch: split-key partial results (gather) or the
 *                                 selection bitmask (masked tile); the size comes from
 *                                 dsa_sparse_attn_workspace_bytes (0 -> NULL is fine).
 *   Requires DQK <= 256, DV <= 256, H <= 64 (H a multiple of 2 above 16, of 4 above 32),
 *   and H*DQK, H*DV rows that are multiples of 16 bytes.
 * --------------------------------------------------------------------------------- */
size_t dsa_sparse_attn_workspace_bytes(dsa_dtype dtype, int B, int S, int T, int H, int DQK,
                                       int DV, int K, dsa_attn_algo algo);
/* The algorithm DSA_ATTN_AUTO resolves to for this shape (DSA_ATTN_GATHER or
 * DSA_ATTN_MASKED_TILE; a request the shape cannot take resolves to DSA_ATTN_AUTO). */
dsa_attn_algo dsa_sparse_attn_algo(dsa_dtype dtype, int B, int S, int T, int H, int DQK, int DV,
                                   int K, dsa_attn_algo algo);
dsa_status dsa_sparse_attn(dsa_dtype dtype, const void* q, const void* k, const void* v,
                           const int32_t* idx, int K, const void* gate,
                           dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                           int H, int DQK, int DV, dsa_attn_algo algo, void* out, void* ws,
                           size_t ws_bytes, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 3b. Sparse attention with attention sinks.  [PANGU] §3.4 (PAS): each layer's learnable
 *    key-value pairs act at inference as a fixed set of virtual KV entries; here they are
 *    `nsink` per-head rows (the expanded form, like the cache) that join every query's
 *    softmax, unmasked, beside its selected keys.
 *
 *   sink_k [nsink,H,DQK] dtype, sink_v [nsink,H,DV] dtype, 1 <= nsink <= 128 (the pages'
 *   128 entries fill one key block of the masked-tile kernel); other arguments and the
 *   contract as dsa_sparse_attn, with the workspace from
 *   dsa_sparse_attn_sinks_workspace_bytes.
 * --------------------------------------------------------------------------------- */
size_t dsa_sparse_attn_sinks_workspace_bytes(dsa_dtype dtype, int B, int S, int T, int H,
                                             int DQK, int DV, int K, int nsink,
                                             dsa_attn_algo algo);
dsa_status dsa_sparse_attn_sinks(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                 const int32_t* idx, int K, const void* sink_k,
                                 const void* sink_v, int nsink, const void* gate,
                                 dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                                 int H, int DQK, int DV, dsa_attn_algo algo, void* out, void* ws,
                                 size_t ws_bytes, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * 3c. Sparse attention over a shared latent cache (the MQA form of MLA).
 *    [AXK2] "注意力前向的骨架" step 2: kv_a_proj_with_mqa compresses K/V into a
 *    kv_lora_rank latent plus a RoPE key slice shared by all heads; [AXK2] "注意力后端选择":
 *    the indexer's positions are for flash-mla (flash_mla_with_kvcache), which attends over
 *    that latent cache.  With the up-projections absorbed into q and the output, every head
 *    attends over the same cached row: logit(h,t) = sm_scale * q[h,:] . kv[t,:] and
 *    out[h,:] = sum_t p(h,t) kv[t, 0:DV].  [PANGU] §3.4: for MLA the PAS sinks are latent
 *    rows as well.
 *
 *   q       [B,S,H,DQK]  bf16     absorbed queries ([latent | rope] per head)
 *   kv      [B,T,DQK]    bf16     latent cache: keys are whole rows, values their first DV
 *                                 dims
 *   idx     [B,S,K]      int32    as dsa_sparse_attn (-1, out-of-range and future entries
 *                                 are skipped; valid entries distinct)
 *   sink_kv [nsink,DQK]  bf16     latent sink rows visible to every query, or NULL with
 *                                 nsink == 0; 0 <= nsink <= 128
 *   gate    [B,S,H]      bf16     or NULL with DSA_GATE_OFF
 *   out     [B,S,H,DV]   bf16     float32 accumulation, one rounding, gate before it; a row
 *                                 with no valid key gets zeros
 *   Requires bf16, DQK == 576 and DV == 512 (kv_lora_rank 512 + a 64-dim RoPE slice),
 *   1 <= H <= 128, 16-byte aligned pointers.  Tensor-core kernel: S = Q kv^T per block of 48
 *   selected rows with M = 128 heads, then O += P V.  Workspace (split-key partials of
 *   decode-shaped calls) from dsa_sparse_attn_latent_workspace_bytes; 0 -> NULL is fine.
 * --------------------------------------------------------------------------------- */
size_t dsa_sparse_attn_latent_workspace_bytes(int B, int S, int H, int K, int nsink);
dsa_status dsa_sparse_attn_latent(dsa_dtype dtype, const void* q, const void* kv,
                                  const int32_t* idx, int K, const void* sink_kv, int nsink,
                                  const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                                  int B, int S, int T, int H, int DQK, int DV, void* out,
                                  void* ws, size_t ws_bytes, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * The whole DSA step: 1 -> 2 -> 3+4.  [AXK2] "注意力前向的骨架" steps 4-5.
 * Scores and indices go to the caller's buffers when scores_out / idx_out are given,
 * else to the workspace.  Without scores_out the score buffer may be smaller than
 * B*S*T floats: the queries are then processed in row blocks that fit.
 * --------------------------------------------------------------------------------- */
typedef struct {
  dsa_dtype dtype;
  int B, S, T;             /* q_off = T - S                                              */
  int HI, DI;              /* indexer heads / head dim                                   */
  float index_scale;       /* indexer softmax_scale (> 0)                                */
  dsa_relu_mode relu;
  int K;                   /* index_topk; the path uses K_eff = min(K, T)                */
  int H, DQK, DV;          /* attention heads, qk_nope+qk_rope, v_head_dim               */
  float sm_scale;          /* <= 0 selects 1/sqrt(DQK)                                   */
  dsa_gate_mode gate_mode;
  dsa_attn_algo attn_algo;
  const void* q_idx;       /* [B,S,HI,DI]                                                */
  const void* k_idx;       /* [B,T,DI]                                                   */
  const float* w;          /* [B,S,HI]                                                   */
  const void* q;           /* [B,S,H,DQK]                                                */
  const void* k;           /* [B,T,H,DQK]                                                */
  const void* v;           /* [B,T,H,DV]                                                 */
  const void* gate;        /* [B,S,H] or NULL                                            */
  void* out;               /* [B,S,H,DV] out                                             */
  float* scores_out;       /* optional [B,S,T] out                                       */
  int32_t* idx_out;        /* optional [B,S,K_eff] out                                   */
  void* const* events;     /* optional: 4 caller-owned cudaEvent_t recorded on the stream
                              before the indexer, after it, after the top-k and after the
                              attention (per-stage timing); NULL for none                */
  dsa_indexer_mode indexer; /* DSA_INDEXER_PER_HEAD (0, the pages' per-head work),
                              DSA_INDEXER_COLLAPSED (the section 1b form) or
                              DSA_INDEXER_FUSED (section 2b: per-head scores filtered in
                              the indexer; bf16 tensor-core indexer shapes; with scores_out
                              or a workspace below dsa_forward_workspace_bytes it runs as
                              DSA_INDEXER_PER_HEAD -- the results are the same)          */
  dsa_index_dtype index_dtype; /* DSA_INDEX_AS_DTYPE (0): q_idx / k_idx have `dtype`;
                              DSA_INDEX_E4M3: they are e4m3 (per-head indexer only)      */
  const void* sink_k;      /* optional [nsink,H,DQK] attention sinks (section 3b)        */
  const void* sink_v;      /* [nsink,H,DV]                                               */
  int nsink;               /* 0 (none) .. 128                                            */
  dsa_attn_form attn_form; /* DSA_ATTN_EXPANDED (0): k, v and the sinks as above;
                              DSA_ATTN_LATENT: k is the latent cache [B,T,DQK] of section
                              3c, v is unused (NULL), sink_k holds [nsink,DQK] latent sink
                              rows, sink_v is unused; attn_algo is ignored                */
  int32_t* topk_fallback_out; /* optional device int32, DSA_INDEXER_FUSED only: written 1
                              when the candidate filter did not hold for some row and the
                              full-score indexer and top-k ran instead, else 0            */
} dsa_forward_args;

/* Bytes of workspace dsa_forward needs to run without row blocking. */
size_t dsa_forward_workspace_bytes(const dsa_forward_args* a);
/* Smallest workspace dsa_forward accepts (one row block). */
size_t dsa_forward_min_workspace_bytes(const dsa_forward_args* a);
dsa_status dsa_forward(const dsa_forward_args* a, void* ws, size_t ws_bytes,
                       dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Sliding-window causal attention with grouped KV heads: the SWA layers of the
 * DSA-SWA-SWA hybrid.  [PANGU] §3.2: window fixed at 512 tokens, SWA:DSA layers 2:1.
 * [SPARK] "为什么 Spark-X2.5 要加这一层门控？": window 512, GQA, headwise gate.
 *
 *   q [B,S,H,DQK], k [B,T,HKV,DQK], v [B,T,HKV,DV], gate [B,S,H] or NULL, out [B,S,H,DV];
 *   query head h reads KV head h / (H/HKV); query s sees keys
 *   s+q_off-window < t <= s+q_off.  Same arithmetic contract as dsa_sparse_attn; algo
 *   DSA_ATTN_MASKED_TILE (and AUTO for S >= 64 where supported) runs tensor-core tiles over
 *   the band, DSA_ATTN_GATHER streams the band's K/V rows.  No workspace.
 * --------------------------------------------------------------------------------- */
dsa_status dsa_window_attn(dsa_dtype dtype, const void* q, const void* k, const void* v,
                           const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                           int window, int B, int S, int T, int H, int HKV, int DQK, int DV,
                           dsa_attn_algo algo, void* out, dsa_stream_t stream);
/* The same with attention sinks ([PANGU] §3.4: every layer has its PAS entries): sink_k
 * [nsink,HKV,DQK], sink_v [nsink,HKV,DV], 1 <= nsink <= 128, visible to every query (query
 * head h through KV head h / (H/HKV)). */
dsa_status dsa_window_attn_sinks(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                 const void* sink_k, const void* sink_v, int nsink,
                                 const void* gate, dsa_gate_mode gate_mode, float sm_scale,
                                 int window, int B, int S, int T, int H, int HKV, int DQK,
                                 int DV, dsa_attn_algo algo, void* out, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * dsa_sparse_attn without any workspace: for callers that cannot allocate device memory.
 * The pages have no counterpart of this call; it exists for embedding.
 *
 * Some callers get only their input and output buffers and may not create device memory
 * themselves -- a plugin inside an inference runtime whose memory planner owns all device
 * memory, or a decode loop with a fixed budget that must not pay for the implicit
 * synchronisation and fragmentation of a new allocation.  This call computes exactly what
 * dsa_sparse_attn computes with DSA_ATTN_GATHER (same kernels, same split of the keys), but
 * keeps the split-key partial results in a fixed array of
 * dsa_sparse_attn_noalloc_max_scratch_bytes() bytes (16 MiB) inside the library's own
 * device memory, which every GPU that loads the library holds until the process exits.
 *
 *   - Nothing is allocated or freed by any call (no cudaMalloc, no allocating library call).
 *   - The first call in a CUDA context (normally the current device's primary context)
 *     looks up the array's device address there (cudaGetSymbolAddress) and keeps it for that
 *     context; make that first call before any stream capture.  A later context on the same
 *     device (after cudaDeviceReset, or a driver-API context made current by the caller) is
 *     a new context: its first call looks the address up again, so no stale address is used.
 *   - Shapes whose partial results need more than the fixed size are rejected with
 *     DSA_ERR_UNSUPPORTED before anything is launched (the message states both sizes); use
 *     dsa_sparse_attn with a workspace for those.  The decode shape of 64 rows x 32 heads x
 *     128-wide values with 2048 selected keys fits.
 *   - Every call on a device shares the one array, which keeps the previous call's
 *     contents; nothing in it needs to start at zero (each call writes every partial it
 *     reads).  Calls that can overlap on the GPU (different streams, or different host
 *     threads) race on the array and must be serialised by the caller.
 *   Arguments and results are those of dsa_sparse_attn (without algo and workspace).
 * --------------------------------------------------------------------------------- */
size_t dsa_sparse_attn_noalloc_max_scratch_bytes(void);
dsa_status dsa_sparse_attn_noalloc(dsa_dtype dtype, const void* q, const void* k, const void* v,
                                   const int32_t* idx, int K, const void* gate,
                                   dsa_gate_mode gate_mode, float sm_scale, int B, int S, int T,
                                   int H, int DQK, int DV, void* out, dsa_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Status and introspection.
 * --------------------------------------------------------------------------------- */
const char* dsa_status_string(dsa_status s);
/* Thread-local description of the last failed call on this thread ("" if none). */
const char* dsa_last_error(void);
/* Reads and (if reset != 0) clears the current device's in-kernel status word.
 * Synchronous with respect to the device: call it after synchronising the streams used.
 * Returns DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_INTERNAL (or DSA_ERR_CUDA if it cannot read). */
dsa_status dsa_device_status(int reset);
/* Library version, e.g. "dsa-b200 0.1.0 sm_100a". */
const char* dsa_version(void);

/* Testing aid for the failure detection (the pages have no counterpart: they describe no
 * failure handling).  Arms a one-shot fault: the next gather-attention launch in this process
 * (dsa_sparse_attn / dsa_sparse_attn_sinks with the gather algorithm, dsa_sparse_attn_noalloc,
 * or a dsa_forward / dsa_window_attn call that takes the gather kernel) makes its first CTA
 * fill none of its shared-memory key slots.  That CTA's consumer warps then wait on a slot
 * that never fills until their bounded wait (about 2 s) runs out; the wait records
 * DSA_ERR_TIMEOUT in the device status word, every later wait of that launch gives up at
 * once, and the launch ends with undefined output.  Nothing faults or hangs: no copy is left
 * in flight, and dsa_device_status(1) reports DSA_ERR_TIMEOUT and clears the word, after which
 * the device is usable as before.  Returns DSA_OK. */
dsa_status dsa_test_arm_wait_timeout(void);

/* Testing aid for the top-k (host code, no device needed).  dsa_topk ranks scores by their
 * order-preserving 32-bit key: the float's bits with the sign bit set for v >= +0.0 (-0.0
 * counts as +0.0), every bit flipped for v < 0.  This returns the smallest float whose key has
 * its top 12 bits at or above b, for b in 0..4096 -- the host build of the bound dsa_topk's
 * second read compares the scores against, so that (key(v) >> 20) >= b exactly when
 * v >= dsa_test_topk_bucket_floor(b), for every non-NaN v.  Buckets 0..7 hold only NaN images
 * and -inf, whose bound is -inf; a bucket past the one of +inf gives NaN, which no comparison
 * passes. */
float dsa_test_topk_bucket_floor(unsigned b);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* DSA_H_ */
