/*
 * spec.h -- C ABI of a B200 (sm_100a) library for the tree-verification step
 * of EAGLE-3 speculative decoding.
 *
 * What the step computes ("EAGLE-3投机解码：树验证器方法", fanquanpp.github.io,
 * sections 验证-接受语义 and 树draft vs 链draft):
 *   - the target model runs ONE forward pass over a whole draft tree, given as
 *     a token array plus parent indices, on top of the sequence's K/V cache;
 *   - every tree node attends to the cached prefix and to its own ancestors
 *     only (the tree's structure is fixed before verification);
 *   - a draft node is accepted iff its token equals the target's argmax at its
 *     parent; the walk from the root keeps the longest accepted path (lowest
 *     index child first) and emits one bonus token, the target's argmax at the
 *     last accepted node -- so each step emits accepted_len + 1 tokens, exactly
 *     what greedy autoregressive decoding would emit;
 *   - only the root's and the accepted nodes' K/V stay in the cache, moved to
 *     consecutive slots.
 *
 * Conventions for every function below:
 *   - return value: SPEC_OK (0) or a negative SPEC_ERR_* code; on error the
 *     cached state of every sequence is unchanged and spec_last_error() holds
 *     a message;
 *   - "device" pointers are CUDA device memory of the GPU that was current at
 *     spec_init; "host" pointers are ordinary CPU memory;
 *   - the library borrows every buffer it is given (weights, K/V cache,
 *     workspace) and never frees one; they must outlive the handle;
 *   - a handle is not thread-safe; all GPU work runs on the stream given to
 *     spec_init.
 */
#ifndef SPEC_H
#define SPEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPEC_API __attribute__((visibility("default")))
#else
#define SPEC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define SPEC_OK 0
#define SPEC_ERR_ARG (-1)      /* null pointer, bad dimension, misaligned buffer */
#define SPEC_ERR_TREE (-2)     /* parents[0] != -1, or some parents[i] outside [0, i) */
#define SPEC_ERR_TOKEN (-3)    /* a token outside [0, vocab) */
#define SPEC_ERR_CAPACITY (-4) /* n_nodes > max_nodes, batch > max_batch, length + n_nodes > max_seq, buffer too small */
#define SPEC_ERR_ROOT (-5)     /* tokens[0] is not the sequence's pending token */
#define SPEC_ERR_CUDA (-6)     /* a CUDA call failed; the message names the cudaError_t */
#define SPEC_ERR_TIMEOUT (-7)  /* a bounded wait inside a kernel expired */
#define SPEC_ERR_STATE (-8)    /* sequence not prefilled, or truncation beyond its length */
#define SPEC_ERR_RANGE (-9)    /* bf16 models: a q / K / V value outside the fp16 range of the cache (|v| > 65504) */

/* model dtypes */
#define SPEC_DTYPE_F32 0       /* weights, activations and K/V in fp32; plain FFMA arithmetic */
#define SPEC_DTYPE_BF16 1      /* weights bf16; GEMM activations as split bf16 (hi + lo); q, K/V cache and
                                  attention probabilities fp16; fp32 accumulation, residual and softmax.
                                  q, K and V (after the rotary embedding) must lie within the fp16 range,
                                  |v| <= 65504: a step that meets a value beyond it (or a NaN) stores it
                                  saturated, leaves every sequence's state as it was, and fails with
                                  SPEC_ERR_RANGE */

/* flags of spec_verify_tree_batch */
#define SPEC_DEVICE_OUTPUTS 1  /* outputs are device pointers (or NULL); return without synchronising */
#define SPEC_DEBUG_LOGITS 2    /* also store fp32 logits [total nodes][vocab] to the buffer of spec_set_debug_logits */
#define SPEC_NO_GRAPH 4        /* launch kernel by kernel instead of replaying a captured CUDA graph */
#define SPEC_FEATURES 8        /* also write the draft-head features of the root and the accepted nodes to
                                  the buffer of spec_set_feature_out (needs cfg.feature_layers) */

typedef struct spec_config {
  int32_t n_layers;
  int32_t hidden;       /* d */
  int32_t n_q_heads;    /* Hq */
  int32_t n_kv_heads;   /* Hkv; Hq % Hkv == 0 (query head j reads kv head j / (Hq/Hkv)) */
  int32_t head_dim;     /* hd; bf16 models need 128, fp32 models <= 128 and even */
  int32_t ffn;          /* SwiGLU width */
  int32_t vocab;
  int32_t dtype;        /* SPEC_DTYPE_* */
  float rms_eps;        /* RMSNorm epsilon */
  float rope_theta;     /* rotary base (rotate-half pairing, no frequency scaling) */
  int32_t max_batch;    /* sequences held in the cache */
  int32_t max_seq;      /* cache slots per sequence */
  int32_t max_nodes;    /* tree nodes per sequence per step, root included; <= 128 */
  int32_t draft_head;   /* 1: the handle also runs the EAGLE-3 draft head (bf16 only): its weights in
                           spec_weights, its layer's K/V one more cache layer (counted by spec_kv_bytes) */
  int32_t feature_layers[3]; /* the low, mid and high features the EAGLE-3 draft head takes (its
                           draft-stage description: the target's low-, mid- and high-level hidden
                           states of every position): the residual stream after this many decoder
                           layers, each in [1, n_layers]; {0, 0, 0}: no feature tap.  The pages name
                           no layers; 2, n_layers / 2 and n_layers - 3 is one choice. */
  int32_t draft_vocab;  /* reduced draft vocabulary (VocabTrim / FR-Spec / SpecVocab in the aitangshan.cn
                           walkthrough, sections 1 and 3.2): 0 = the draft head scores the whole vocabulary;
                           2 .. vocab = its LM head is spec_weights.draft_lm_head, the target's rows of the
                           token ids draft_vocab_ids, its softmax and its drafts cover only those tokens
                           (verification is unchanged).  Needs draft_head. */
} spec_config;

/* Per-layer weights, device pointers, row-major [out][in] in the model dtype:
 * wq [Hq*hd][d], wk/wv [Hkv*hd][d], wo [d][Hq*hd], w_gate/w_up [ffn][d],
 * w_down [d][ffn]; attn_norm / mlp_norm [d]. */
typedef struct spec_layer_weights {
  const void* wq;
  const void* wk;
  const void* wv;
  const void* wo;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* attn_norm;
  const void* mlp_norm;
} spec_layer_weights;

/* Model weights.  `layers` is a HOST array of n_layers entries (copied by
 * spec_init); every weight pointer in it, and embed [vocab][d], final_norm [d],
 * lm_head [vocab][d], are device pointers 16-byte aligned.  The draft-head
 * fields may be NULL when cfg.draft_head == 0: draft_fc_fuse [d][3d],
 * draft_fc_in [d][2d], draft_layer (host pointer to one entry), draft_final_norm [d]. */
typedef struct spec_weights {
  const void* embed;
  const void* final_norm;
  const void* lm_head;
  const spec_layer_weights* layers;
  const void* draft_fc_fuse;
  const void* draft_fc_in;
  const spec_layer_weights* draft_layer;
  const void* draft_final_norm;
  const void* draft_lm_head;        /* cfg.draft_vocab > 0: [draft_vocab][d], device, 16-byte aligned */
  const int32_t* draft_vocab_ids;   /* cfg.draft_vocab > 0: [draft_vocab] token ids, device, strictly
                                       increasing in [0, vocab) (checked by spec_init: SPEC_ERR_ARG) */
} spec_weights;

typedef struct spec_handle spec_handle;

/* Bytes of device memory for the K/V cache.  Layout [layer][plane][seq][kv head][slot][hd]:
 * fp32 models hold planes K, V (fp32); bf16 models hold K, V and K_lo in fp16, where
 * K_lo = fp16(k - fp16(k)) carries the rounding error of K so that the attention
 * scores see ~22 bits of each key. */
SPEC_API size_t spec_kv_bytes(const spec_config* cfg);
/* Bytes of device workspace (activations, split-K partials, per-sequence state). */
SPEC_API size_t spec_workspace_bytes(const spec_config* cfg);

/* Validate dimensions, record the borrowed device buffers, build the TMA
 * descriptors.  kv_cache and workspace are device buffers of at least the
 * sizes above; cuda_stream is a cudaStream_t (NULL: the legacy default stream,
 * on which steps are launched kernel by kernel because it cannot be captured
 * into a CUDA graph).
 * Every sequence starts empty. */
SPEC_API int spec_init(const spec_config* cfg, const spec_weights* w, void* kv_cache, size_t kv_bytes, void* workspace,
              size_t ws_bytes, void* cuda_stream, spec_handle** out);

/* Reset sequence `seq` and run the prompt (host int32[n], n >= 1) through the
 * target in causal chunks of at most max_nodes tokens, caching every position.
 * *pending_token (host) receives the argmax at the last position: the root of
 * the next tree.  Synchronises the stream. */
SPEC_API int spec_prefill(spec_handle* h, int seq, const int32_t* tokens, int n, int32_t* pending_token);
/* spec_prefill that also writes the draft-head features of every prompt position (the
 * residual stream after feature_layers[0], [1] and [2] decoder layers, rounded to bf16) to
 * feats_out: device bf16 [n][3][hidden], 16-byte aligned, owned by the caller.  These are
 * the features the EAGLE-3 draft head records during prefill (its draft-stage description).
 * SPEC_ERR_STATE when the handle has no feature layers. */
SPEC_API int spec_prefill_features(spec_handle* h, int seq, const int32_t* tokens, int n, int32_t* pending_token,
                                   void* feats_out);

/* One verification step for one sequence (host pointers, synchronises).
 * tokens[0] must be the pending token; parents[0] == -1 and 0 <= parents[i] < i.
 * accepted_tokens needs room for n_nodes - 1 entries.  Emitted tokens are
 * accepted_tokens[0 .. *accepted_len) followed by *bonus_token, which becomes
 * the next pending token. */
SPEC_API int spec_verify_tree(spec_handle* h, int seq, const int32_t* tokens, const int32_t* parents, int n_nodes,
                     int32_t* accepted_len, int32_t* accepted_tokens, int32_t* bonus_token);

/* Batched verification.  Host inputs: seq_ids[B] (distinct), node_offsets[B+1]
 * (node_offsets[0] == 0), tokens / parents concatenated per sequence, parents
 * local to their sequence.  Outputs per sequence b: accepted_len[b],
 * accepted_nodes[b * max_nodes + k] (local node indices), accepted_tokens
 * (same layout), bonus[b].  Without SPEC_DEVICE_OUTPUTS they are host pointers
 * and the call synchronises; with it they are device pointers (or NULL) and the
 * call returns once the work is queued -- errors found on the device are then
 * reported by the next spec_sync. */
SPEC_API int spec_verify_tree_batch(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens,
                           const int32_t* parents, const int32_t* node_offsets, int32_t* accepted_len,
                           int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus, int flags);

/* The target's argmax (and top-1 / top-2 logits) at every node of a batch of
 * trees, without acceptance and without changing any cached state.  Inputs as
 * in spec_verify_tree_batch; outputs are host arrays of node_offsets[B]
 * entries.  Synchronises. */
SPEC_API int spec_score_trees(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens, const int32_t* parents,
                     const int32_t* node_offsets, int32_t* argmax, float* top1, float* top2, int flags);

/* ---- EAGLE-3 draft head (cfg.draft_head = 1, bf16 models) ----------------
 * The draft stage of "EAGLE-3: Scaling up Inference Acceleration of Large
 * Language Models via Training-Time Test" (summary page, draft-stage section):
 * the target's low, mid and high features l, m, h of a position (d each) are
 * concatenated and reduced by one FC layer to the fused feature g = [l|m|h].
 * W_fuse^T; g is concatenated with the embedding e of the token one step ahead
 * and reduced by a second FC layer, x = [g|e].W_in^T; one pre-norm decoder layer
 * of the target's shape (its own K/V cache) turns x into a, and the target's LM
 * head, after the draft head's final RMSNorm, scores a.  Readings where the page
 * is silent: concatenation orders [l|m|h] and [g|e]; e from the target's
 * embedding table; tree nodes attend to the draft prefix and their ancestors
 * at positions prefix + depth, as in verification.
 *
 * feats are DEVICE pointers to bf16 [rows][3][d] (l, m, h per row); tokens,
 * parents and node_offsets are host arrays as in spec_verify_tree_batch. */
#define SPEC_DRAFT_TOPK 10     /* draft candidates per node (the pages' tree top-k) */

/* Build the draft layer's K/V for positions 0 .. n-1 of `seq` from n rows of
 * features and tokens (n <= max_seq), replacing what was there.  Synchronises. */
SPEC_API int spec_draft_prefill(spec_handle* h, int seq, const void* feats, const int32_t* tokens, int n);
/* As spec_draft_prefill, but the n rows extend the draft prefix of `seq` (positions len ..
 * len + n - 1, attending to the rows before them): the rows a verification step adds.
 * SPEC_ERR_STATE when the sequence has no draft prefix; SPEC_ERR_CAPACITY past max_seq (both
 * before any work, the prefix unchanged).  An error during the work leaves the prefix marked
 * unusable: rebuild it with spec_draft_prefill.  Synchronises. */
SPEC_API int spec_draft_append(spec_handle* h, int seq, const void* feats, const int32_t* tokens, int n);
/* One draft-head step over a batch of trees on the draft prefixes: per node,
 * the SPEC_DRAFT_TOPK best vocabulary entries of the draft distribution, by
 * logit descending then index ascending, in top_idx / top_val [nodes][TOPK]
 * (selected inside the LM-head GEMM, per 128-row vocabulary tile, then merged:
 * the draft logits are not stored).
 * The draft prefixes are not extended (the trees' K/V are scratch).  Flags:
 * SPEC_DEVICE_OUTPUTS (outputs are device pointers, no synchronisation),
 * SPEC_DEBUG_LOGITS (also the fp32 draft logits to the debug buffer),
 * SPEC_NO_GRAPH.  Errors as in spec_verify_tree_batch; SPEC_ERR_STATE when a
 * sequence has no draft prefix. */
SPEC_API int spec_draft_step(spec_handle* h, int B, const int32_t* seq_ids, const void* feats, const int32_t* tokens,
                             const int32_t* parents, const int32_t* node_offsets, int32_t* top_idx, float* top_val,
                             int flags);
/* Draft prefix length of `seq` (host output). */
SPEC_API int spec_draft_len(spec_handle* h, int seq, int32_t* len);

/* Dynamic draft tree for B sequences ("EAGLE-3: Scaling up Inference Acceleration of Large
 * Language Models via Training-Time Test", draft-stage description: multi-step drafting, where
 * from the second step on the draft's own output a replaces the target feature; and its account
 * of EAGLE-2: the draft's confidence stands in for the acceptance rate and shapes the tree).
 * Reading taken where the pages leave steps open: a node's value is the sum of the draft's
 * log-probabilities (full-vocabulary softmax) along its root path; step t = 0 .. steps-1 runs
 * the draft head over the tree built so far (the root's feature is the fused target feature,
 * every other node's the output a of its parent); the nodes that joined last (the root at step
 * 0) offer their topk best tokens and the topk best offers join (ties: earlier offer); after the
 * last step the `total` best offers, joined or not (ties: lower depth, then earlier offer), form
 * the tree, which is closed under ancestors.
 * root_feats: device bf16 [B][3][hidden], 16-byte aligned, the low/mid/high target features of
 * each sequence's last verified position (as SPEC_FEATURES returns them); root_tokens: host
 * int32 [B], the pending tokens (the roots).  Each sequence needs a draft prefix (the rows up to
 * the last verified position, spec_draft_prefill), which the call leaves unchanged.  topk is 4,
 * 8, 10 or 16; 1 + (steps-1)*topk <= max_nodes, 1 + steps*topk <= 128, topk + (steps-1)*topk^2
 * <= 1024 offers, total <= that and total + 1 <= max_nodes (SPEC_ERR_CAPACITY otherwise).
 * Outputs (host): out_tokens / out_parents int32 [B][total+1], root first, nodes by depth and
 * then value, parents[i] < i (a tree spec_verify_tree_batch accepts); out_values (may be NULL)
 * float [B][total+1], each node's value (0 for the root).  Synchronises. */
SPEC_API int spec_draft_tree(spec_handle* h, int B, const int32_t* seq_ids, const void* root_feats,
                             const int32_t* root_tokens, int steps, int topk, int total, int32_t* out_tokens,
                             int32_t* out_parents, float* out_values);

/* Device buffer for SPEC_FEATURES, bf16 [B][max_nodes][3][hidden], 16-byte aligned, owned by the
 * caller.  A verification step with SPEC_FEATURES writes, for batch entry b and k = 0 ..
 * accepted_len[b], row [b][k] = the residual stream after feature_layers[0], [1] and [2] decoder
 * layers (rounded to bf16) at the k-th node of the emitted path: the root for k = 0, then the
 * accepted nodes in order, i.e. the positions P .. P + accepted_len that the step adds to the cache.
 * Rows beyond accepted_len[b] are left as they were.  bytes must cover the step's batch:
 * B * max_nodes * 3 * hidden * 2 (checked per step; SPEC_ERR_CAPACITY otherwise).  SPEC_ERR_STATE
 * when the handle has no feature layers; device_buf NULL detaches the buffer. */
SPEC_API int spec_set_feature_out(spec_handle* h, void* device_buf, size_t bytes);

/* Temperature sampling instead of greedy choices (both leave the target's output distribution
 * unchanged: "EAGLE-3投机解码：树验证器方法", section 验证-接受语义, and the sampling rule of
 * Leviathan et al., "Fast Inference from Transformers via Speculative Decoding", which that page
 * cites).  temperature = 0 (the default) restores greedy decoding.
 *
 * With temperature T > 0, every token the target chooses -- the pending token of a prefill, the
 * choice at each tree node of a verification or scoring step -- is a draw from softmax(logits / T),
 * taken as argmax_v(logit_v / T + g_v) with g_v a standard Gumbel variable.  The noise of a row
 * depends only on (seed, sequence id, the row's position, v): g_v = -ln(-ln u) with
 * u = (2 (x >> 9) + 1) 2^-24 and x word 0 of Philox4x32-10 (Salmon et al., SC 2011) at counter
 * (v, position, sequence id, 0) and key (seed & 0xffffffff, seed >> 32).  A tree node at position
 * P + depth accepts, as in the greedy walk, the first child whose token equals its draw; the bonus is
 * the draw at the last accepted node.  Each draft token thus acts as a point-mass proposal in the
 * speculative-sampling rule (accepted with probability p(x) given the earlier siblings' rejections),
 * and the emitted stream is exactly autoregressive sampling with the same noise.  spec_score_trees
 * then returns the draws as "argmax" and the perturbed scores logit / T + g as top1 / top2.  The
 * draft head's top-k is unaffected.  SPEC_ERR_ARG for a negative, infinite or NaN temperature or
 * one whose reciprocal overflows.  Takes effect for calls made after it (cached graphs are rebuilt). */
SPEC_API int spec_set_sampling(spec_handle* h, float temperature, uint64_t seed);

/* Device buffer (fp32, >= max_batch * max_nodes * vocab entries) for SPEC_DEBUG_LOGITS. */
SPEC_API int spec_set_debug_logits(spec_handle* h, float* device_buf, size_t bytes);

/* Roll sequence `seq` back to new_len cached positions (new_len < current
 * length, or equal for a no-op); the token cached at new_len becomes pending. */
SPEC_API int spec_truncate(spec_handle* h, int seq, int new_len);
/* Cached length and pending token of `seq` (host outputs; synchronises). */
SPEC_API int spec_seq_len(spec_handle* h, int seq, int32_t* len, int32_t* pending);
/* Wait for queued work; report (and clear) errors recorded on the device. */
SPEC_API int spec_sync(spec_handle* h);

/* Host-only check of one tree, usable without a GPU or a handle: 1 <= n <=
 * max_nodes (else SPEC_ERR_CAPACITY), parents[0] == -1 and 0 <= parents[i] < i
 * (else SPEC_ERR_TREE), every token in [0, vocab) (else SPEC_ERR_TOKEN); null
 * pointers give SPEC_ERR_ARG.  The verification calls apply the same checks. */
SPEC_API int spec_validate_tree(const int32_t* tokens, const int32_t* parents, int n, int vocab, int max_nodes);

/* Kernel classes timed by the profiler (index into spec_profile_read's arrays). */
#define SPEC_PROF_EMBED_META 0   /* tree metadata + embedding + first RMSNorm */
#define SPEC_PROF_GEMM_QKV 1
#define SPEC_PROF_ROPE_KV 2      /* split-K sum + rotary + K/V cache store */
#define SPEC_PROF_ATTENTION 3    /* tree attention chunks + merge */
#define SPEC_PROF_GEMM_O 4
#define SPEC_PROF_RESID_NORM 5   /* split-K sum + residual + RMSNorm */
#define SPEC_PROF_GEMM_GATE_UP 6 /* gate/up GEMM with fused SwiGLU */
#define SPEC_PROF_GEMM_DOWN 7
#define SPEC_PROF_LM_HEAD 8      /* LM-head GEMM with fused argmax */
#define SPEC_PROF_LM_REDUCE 9
#define SPEC_PROF_WALK 10        /* acceptance walk + state update */
#define SPEC_PROF_COMPACT 11     /* K/V compaction */
#define SPEC_PROF_GEMM_LAYER 12  /* one launch: O, gate/up, down, then the next QKV or the LM head */
#define SPEC_PROF_DRAFT_FC 13    /* draft head: feature split, fusion FC, input FC */
#define SPEC_PROF_TOPK 14        /* draft head: merge of the LM-head tiles' top-k candidates */
#define SPEC_PROF_FEATURES 15    /* draft-head feature tap and gather (SPEC_FEATURES) */
#define SPEC_PROF_TREE 16        /* dynamic draft tree: root features, expansion, rerank */
#define SPEC_PROF_CLASSES 17

/* enable != 0: subsequent steps launch kernel by kernel (no graph) with a CUDA
 * event pair around every launch on the handle's stream. */
SPEC_API int spec_profile(spec_handle* h, int enable);
/* Synchronise, then add the recorded device milliseconds and launch counts per
 * class into ms[SPEC_PROF_CLASSES] and launches[SPEC_PROF_CLASSES] (host
 * arrays, either may be NULL) and forget the records. */
SPEC_API int spec_profile_read(spec_handle* h, double* ms, int64_t* launches);
/* Bytes one synchronous verification step copies host->device (parameter
 * block) and device->host (outputs and error word). */
SPEC_API int spec_io_bytes(spec_handle* h, size_t* h2d, size_t* d2h);
/* Human-readable execution plan (residency, GEMM tiling and split-K, attention
 * chunking) for a batch of B trees of n_nodes nodes on prefixes of `prefix`
 * tokens, written to buf (n bytes, NUL-terminated). */
SPEC_API int spec_info(spec_handle* h, int B, int n_nodes, int prefix, char* buf, size_t n);
/* Optional timeline of decoder layer `layer` (bf16 models), in %globaltimer
 * stamps (uint64 ns); NULL turns it off.  device_buf holds 2 * SMs * 64 + 8192
 * entries: first the layer's GEMM launch, [2 * SMs CTAs][4 phases][16] (0-7:
 * producer starts the phase, may load its activations, has issued its last
 * load; epilogue starts the phase, first accumulator complete, split-K
 * rendezvous passed, units done, phase counted at the grid barrier; 8-11 for the
 * first unit: partial stored, split partials summed, finishing stores done,
 * unit done), then its attention launch and the next layer's, [2][256 CTAs][16] (start, Q landed,
 * first K/V block landed, first scores ready, output accumulated, partial
 * written, chunk rendezvous passed, merge done, first block's max found, first
 * block's P written, first scores issued, last P seen by the issuer).  Entries
 * of CTAs that did not run stay as they were. */
SPEC_API int spec_set_trace(spec_handle* h, uint64_t* device_buf, size_t bytes, int layer);
/* Number of kernels the most recent step enqueued. */
SPEC_API int spec_step_launches(spec_handle* h);

/* LM head with fused per-row argmax, for callers that cannot allocate device
 * memory.  (The pages have no counterpart: this is a deployment variant of the
 * step's last kernel.)  Some callers are not allowed to call cudaMalloc: code
 * running inside a CUDA-graph capture, runtimes that own every buffer and hand
 * out no allocation rights, plug-in hosts that forbid allocation after start-up.
 * This entry point needs no allocation and no handle: its scratch (a split-bf16
 * copy of the normalised rows and per-vocabulary-tile top-2 partials) is one
 * fixed array of about 3.5 MiB inside the library, which every GPU that loads
 * the library holds until the process exits.
 *
 * Computes, for each of M hidden rows h (device fp32 [M][d], before the final
 * norm): RMSNorm(h) * final_norm (device bf16 [d]) times lm_head^T (device bf16
 * [V][d], 16-byte aligned), and writes argmax[M] (lowest index on ties),
 * top1[M] and top2[M] (device arrays).  Limits: 1 <= M <= 64, d a multiple of
 * 128 up to 8192, V up to 262144; larger sizes return SPEC_ERR_CAPACITY before
 * any GPU work.  Work is queued on cuda_stream (NULL: legacy default stream);
 * the call does not synchronise.
 *
 * Device-side failure: every wait inside the call is bounded (2 s).  If one
 * gives up, the GPU stays usable and every row gets argmax = -1 and
 * top1 = top2 = NaN; the return code cannot say so, because the call returns
 * before the GPU runs.  After synchronising the stream, argmax[0] < 0 means
 * the outputs are void.  The error word behind this is part of the scratch and
 * is cleared at the start of each call.
 *
 * The first call on a device looks up the scratch array's device address and
 * sets kernel attributes, so make that first call before any stream capture.
 * Every call uses the same scratch and leaves its contents behind; only the
 * error word has to start at zero, and the call clears it itself (a memset on
 * cuda_stream, no allocation).  Calls that overlap on the GPU (on different
 * streams, or from different threads) race on the scratch: serialise them. */
SPEC_API int spec_lm_head_argmax_noalloc(const float* hidden, const void* final_norm, const void* lm_head, int M,
                                         int d, int V, float eps, int32_t* argmax, float* top1, float* top2,
                                         void* cuda_stream);

/* Self-test of the bounded waits.  Every wait inside the library's kernels
 * (split-K and attention-chunk rendezvous, grid barriers between GEMM phases,
 * pipeline mbarriers) gives up after a time limit, records a timeout in the
 * step's error word and returns; the step then fails with SPEC_ERR_TIMEOUT and
 * the CUDA context stays usable.  This call runs the same two wait primitives
 * on one GPU thread against a counter that nothing increments and an mbarrier
 * that nothing arrives on, each limited to limit_us microseconds (1 .. 10^6).
 * device_scratch: 16 bytes of device memory, 4-byte aligned, owned by the
 * caller (overwritten).  On return *expired holds how many of the two waits
 * gave up (2 when the mechanism works).  Returns SPEC_ERR_TIMEOUT when the
 * device reported the timeout (the expected outcome), SPEC_OK if it did not,
 * SPEC_ERR_ARG / SPEC_ERR_CUDA on bad arguments or a CUDA error.  Runs on the
 * legacy default stream and synchronises the device. */
SPEC_API int spec_wait_selftest(void* device_scratch, uint32_t limit_us, int32_t* expired);

/* Message of the last error on this handle ("" if none). */
SPEC_API const char* spec_last_error(spec_handle* h);
/* Free host-side state (graphs, descriptors); never frees borrowed buffers. */
SPEC_API void spec_free(spec_handle* h);

#ifdef __cplusplus
}
#endif

#endif /* SPEC_H */
