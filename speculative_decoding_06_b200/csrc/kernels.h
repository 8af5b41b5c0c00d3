// Internal kernel interfaces of the tree-verification library (host <-> device
// argument structs and launchers).  Not part of the public C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace spec {

struct Top2;

// GEMM epilogues:
//   QKV    split-K partials; the last CTA of each 128-feature tile (one head of
//          q|k|v) sums the splits, applies the norm scale and the rotary
//          embedding, and writes q (fp16) or the K/V cache slot (fp16)
//   RESID  split-K partials; the last CTA of each tile adds the sum to the fp32
//          residual stream for its 128 columns, writes the next GEMM's operand
//          x*w (split bf16) and the tile's per-token sums of squares of x
//   SWIGLU gate rows 0-63, up rows 64-127 of a tile; silu(g)*u as split bf16
//   ARGMAX per-token (best, index, runner-up) of the tile's vocabulary rows
//   TOPK   per token, the tile's k best logits and (max, sum of exp) (draft LM head)
enum { GEMM_EPI_QKV = 0, GEMM_EPI_SWIGLU = 1, GEMM_EPI_ARGMAX = 2, GEMM_EPI_RESID = 3, GEMM_EPI_STORE = 4,
       GEMM_EPI_TOPK = 5 };

struct StepView;

struct GemmTcArgs {
  int n_out;          // output features (weight rows) across all segments
  int K;              // reduction length, multiple of 64
  int M;              // valid tokens (columns); token rows >= M are ignored
  int tiles_o, tiles_t, splits, kb_per_split;
  // stream-K (SWIGLU, ARGMAX, TOPK; splits = 1): tiles [0, sk_tiles) are shared
  // out, every CTA taking an equal contiguous share of their sk_tiles x K/64
  // k-blocks first; a share that starts inside a tile writes fp32 sums to part +
  // CTA * 128 * BN ([BN tokens][128 rows]) and counts itself at counters[tile];
  // the CTA holding the tile's first k-block adds them and finishes the tile.
  // The other tiles go round-robin, whole (sk_tiles = all the tiles when they are
  // fewer than the CTAs, else the last round's remainder).  Needs sk_tiles x
  // K/64 >= 2 x grid.
  int streamk, sk_tiles;
  int seg_rows[3];    // rows served by mA0, mA1, mA2; unused for SWIGLU
  // RMSNorm folded into the epilogue: the operand rows are x*w, not yet
  // normalised; the result is scaled per token by rsqrt(sum(ss)/norm_d + eps)
  // with ss the n_ss partial sums of squares of x (null: no scaling)
  const float* ss_in;
  int n_ss, ss_ld, norm_d;
  float eps;
  // split-K partials [splits][tokens][n_out] and per-tile arrival counters
  float* part;
  size_t split_stride;
  int* counters;      // [2 * tiles_o * tiles_t], zero at launch; a phase's own (never reused within a step)
  // SWIGLU, STORE (the accumulator itself, no split-K)
  __nv_bfloat16* out_bf16;  // split bf16 [2 x tokens][ld_out]
  int ld_out;
  // ARGMAX
  Top2* top_part;     // [tiles_o][top_ld]
  int top_ld;
  float* dbg_logits;  // optional [M][n_out] (the logits themselves, before any sampling noise; ARGMAX, TOPK)
  // TOPK: per token and tile, kCandSlots candidates that hold the tile's `topk` (<= 16)
  // best logits (unused slots -inf) into cand_v / cand_i [tokens][cand_ld][kCandSlots]
  // and (max, sum of exp(l - max)) into cand_lse [tokens][cand_ld]; cand_ld = tiles_o
  int topk, cand_ld;
  float* cand_v;
  int32_t* cand_i;
  float2* cand_lse;
  // sampling (inv_temp > 0): the row's choice is argmax_v(logit_v * inv_temp + gumbel(seed, sid, pos, v))
  // with sid = row_sid[t] and pos = row_pos[t]; inv_temp = 0: the plain argmax
  const int32_t* row_pos;
  float inv_temp;
  uint32_t seed_lo, seed_hi;
  // QKV
  const int32_t* row_seq;
  const int32_t* row_local;
  const int32_t* row_slot;  // cache slot P_b + local (-1 beyond max_seq)
  const int32_t* row_sid;   // sequence id
  const int32_t* P_step;
  const int32_t* seq_ids;
  const float2* rope_cs;  // [tokens][64]
  __half* q_out;          // [2][Hkv][q_rows][128]: part 0 = fp16(q), part 1 = fp16(q - part 0);
                          // row t*G + g holds head kvh*G + g of token t
  int q_rows;             // rows per kv head in q_out (>= tokens * G)
  __half* k_cache;        // this layer's K base: [max_batch][Hkv][max_seq][128]
  __half* klo_cache;      // this layer's K_lo plane (fp16(k - fp16(k))), same layout
  __half* v_cache;
  size_t kv_seq_stride, kv_head_stride;
  int Hq, Hkv, max_seq;
  // RESID
  float* x;                         // [tokens][n_out]
  const __nv_bfloat16* norm_w_next; // [n_out]
  __nv_bfloat16* xn_out;            // split bf16 [2 x tokens][n_out]
  float* ss_out;                    // [tiles_o][ss_ld]
  uint32_t* err;
};

constexpr int kMaxGemmPhases = 4;
constexpr int kCandSlots = 24;  // TOPK candidates per (token, vocabulary tile)
constexpr int kGemmTraceMarks = 16;  // %globaltimer marks per CTA and phase (optional timeline)

// kernel parameters: the tensor maps of every phase (a0, a1, a2, b) and the phases
struct GemmMaps {
  CUtensorMap m[4 * kMaxGemmPhases];
};
struct GemmPhases {
  int n_phases;
  int epi[kMaxGemmPhases];
  int* phase_bar;  // [n_phases - 1] CTAs done with each phase, zero at launch
  uint32_t* err;
  uint64_t* trace; // optional [grid][kMaxGemmPhases][kGemmTraceMarks] %globaltimer stamps
  GemmTcArgs ph[kMaxGemmPhases];
};

struct GemmPhase {
  int epi;
  const CUtensorMap *mA0, *mA1, *mA2, *mB;
  GemmTcArgs args;
};
// One launch, a list of phases separated by grid-wide barriers.  The grid must
// be co-resident in full when n_phases > 1 or any phase uses split-K.
struct GemmMultiLaunch {
  int bn, grid, n_phases;
  int* phase_bar;
  uint32_t* err;
  uint64_t* trace;
  GemmPhase ph[kMaxGemmPhases];
};

struct GemmTcLaunch {
  int bn, epi, grid;
  const CUtensorMap *mA0, *mA1, *mA2, *mB;
  GemmTcArgs args;
};

cudaError_t gemm_multi_launch(const GemmMultiLaunch& L, cudaStream_t stream, bool pdl);
cudaError_t gemm_tc_launch(const GemmTcLaunch& L, cudaStream_t stream, bool pdl);  // one phase
uint32_t gemm_tc_smem_bytes(int bn);
const void* gemm_tc_function(int bn);

// One verification step, as seen by the kernels.  Node ("row") r in [0, M)
// belongs to batch entry b with node_off[b] <= r < node_off[b+1]; its local
// index is r - node_off[b]; parents hold local indices.
struct StepView {
  const int32_t* tokens;    // [M]
  const int32_t* parents;   // [M]
  const int32_t* node_off;  // [B+1]
  const int32_t* seq_ids;   // [B]
  const int32_t* order;     // [B] batch entries by decreasing key count (attention's work order)
  int B, M;
  int32_t* row_seq;         // [M] batch entry
  int32_t* row_local;       // [M] local node index
  int32_t* row_slot;        // [M] cache slot P_b + local index, -1 when it would pass max_seq
  int32_t* row_sid;         // [M] sequence id
  int32_t* row_pos;         // [M] position P_b + depth
  uint64_t* row_anc;        // [M][2] ancestor bits over local indices (self included)
  float2* rope_cs;          // [M][head_dim/2] (cos, sin)
  int32_t* P_step;          // [B] cached length at step start
  int32_t* seq_len;         // [max_batch] persistent
  int32_t* pending;         // [max_batch] persistent
  int32_t* hist;            // [max_batch][max_seq] persistent token history
  int max_seq;
  uint32_t* err;            // this step's error bits
  uint32_t* err_sticky;     // accumulated until read by the host
};

struct KvView {
  void* base;               // [layer][plane][max_batch][Hkv][max_seq][hd]
  int max_batch, Hkv, max_seq, hd;
  size_t elem;              // 2 (bf16 models: fp16 planes) or 4 (fp32)
  int planes;               // K, V (fp32 models); K, V, K_lo (bf16 models: K = K + K_lo to ~22 bits)
  __host__ __device__ size_t head_stride() const { return (size_t)max_seq * hd; }
  __host__ __device__ size_t seq_stride() const { return (size_t)Hkv * max_seq * hd; }
  __host__ __device__ size_t kv_stride() const { return (size_t)max_batch * seq_stride(); }
  __host__ __device__ size_t layer_stride() const { return (size_t)planes * kv_stride(); }
};

enum { STEP_VERIFY = 0, STEP_PREFILL = 1, STEP_SCORE = 2, STEP_DRAFT = 3, STEP_DRAFT_KV = 4 };

// metadata + embedding + first RMSNorm.  bf16 models: xn = split(x*w) (the
// norm scale is applied by the next GEMM) and ss[0][r] = sum x^2, ss[i>0][r] = 0.
// With e_out (draft head, bf16): the embedding row goes to e_out as split bf16
// at columns [e_col, e_col + d) of rows of e_ld elements, and x, xn, ss are
// left alone.
cudaError_t launch_embed_meta(int dtype, const StepView& sv, const void* embed, const void* norm_w, int d, float eps,
                              float* x, void* xn, float* ss, int n_ss, int ss_ld, const double* inv_freq, int half,
                              int mode, cudaStream_t s, bool pdl, __nv_bfloat16* e_out = nullptr, int e_ld = 0,
                              int e_col = 0);
// bf16 rows [rows][cols] -> split bf16 operand [2 x rows][cols] (lo parts zero)
cudaError_t launch_split_rows(const __nv_bfloat16* src, int rows, int cols, __nv_bfloat16* dst, cudaStream_t s,
                              bool pdl);
// the longest top-k list of the draft head (value desc, index asc)
constexpr int kTopKMax = 16;
// top-k per row (k in {4, 8, 10, 16}) from the LM head's TOPK candidates: cand_v / cand_i
// [M][tiles][kCandSlots] (a superset of each tile's k best), cand_lse [M][tiles] (max, sum of
// exp(l - max));
// with lse != NULL also the row's log-sum-exp; indices mapped through id_map when given
cudaError_t launch_topk_merge(int M, int tiles, int k, const float* cand_v, const int32_t* cand_i,
                              const float2* cand_lse, int32_t* idx, float* val, float* lse, cudaStream_t s, bool pdl,
                              const int32_t* id_map = nullptr);

// a launch configuration with programmatic dependent launch when pdl (attr: 1 slot)
cudaLaunchConfig_t make_cfg(dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, cudaLaunchAttribute* attr);

// ---------------------------------------------------------------------------
// dynamic draft tree (draft_tree.cu)
// ---------------------------------------------------------------------------
constexpr int kTreeMaxOffers = 1024;  // candidates offered over all steps, per tree
constexpr int kTreeMaxNodes = 128;    // nodes joined over all steps, per tree (root included)

struct TreeOffer {
  float v;      // cumulative log-probability
  int depth;    // the offered node's depth
  int order;    // offer order within the tree (ties)
  int parent;   // offering node (joined node id)
  int token;
  int node;     // joined node id, or -1
};

struct TreeArgs {
  int K;            // top-k per offering node, and nodes joining per step
  int max_nodes;    // stride of the per-tree node arrays
  int write_next;   // 1: write the next step's tree into the parameter block
  int32_t* tok;     // [B][max_nodes] joined nodes
  int32_t* par;
  float* val;
  TreeOffer* offers;  // [B][kTreeMaxOffers]
  int32_t* n_offers;  // [B]
};

cudaError_t launch_tree_save_root(int B, int d, int ld, const __nv_bfloat16* ge, __nv_bfloat16* groot,
                                  const int32_t* tokens, const TreeArgs& a, cudaStream_t s, bool pdl);
cudaError_t launch_tree_feature_rows(int M, int d, int ld, int n, int n_prev, const int32_t* parents,
                                     const __nv_bfloat16* groot, const float* x_prev, __nv_bfloat16* ge,
                                     cudaStream_t s, bool pdl);
cudaError_t launch_tree_expand(const TreeArgs& a, int B, int t, int n, int nf, const int32_t* top_i,
                               const float* top_v, const float* lse, int32_t* tokens_io, int32_t* parents_io,
                               int32_t* node_off_io, cudaStream_t s, bool pdl);
cudaError_t launch_tree_rerank(const TreeArgs& a, int B, int total, int32_t* out_tok, int32_t* out_par,
                               float* out_val, cudaStream_t s, bool pdl);
// x += sum of split partials; xn = RMSNorm(x) * w
cudaError_t launch_residual_norm(int dtype, int M, int d, int S, const float* partial, size_t split_stride, float* x,
                                 void* xn, const void* w, float eps, cudaStream_t s, bool pdl);
// sum partials, rotary on q and k, q -> q_out, k/v -> cache slots P_b + local
cudaError_t launch_qkv_rope_store(int dtype, const StepView& sv, int S, const float* partial, size_t split_stride,
                                  int Hq, int Hkv, int hd, void* q_out, const KvView& kv, int layer, cudaStream_t s,
                                  bool pdl);
// fp32 path: h = silu(gate) * up from a [M][2F] buffer
cudaError_t launch_swiglu_f32(int M, int F, const float* gu, float* h, cudaStream_t s);
// fp32 path SIMT GEMM: C[t][o] = sum_k A[t][k] W[o][k]
cudaError_t launch_gemm_simt_f32(const float* A, int lda, const float* W, int K, float* C, int ldc, int M, int N,
                                 cudaStream_t s);

// attention
struct AttnArgs {
  StepView sv;
  KvView kv;
  int layer;
  int Hq, hd;
  const void* q;            // [M][Hq][hd]
  void* out;                // [M][Hq*hd]
  float* part_o;            // [M*Hq][n_chunks][hd]
  float* part_lse;          // [M*Hq][n_chunks]
  int n_chunks, chunk;      // key chunking of [0, P_b + n_b)
  int max_rows;             // max over batch of n_b * (Hq/Hkv)
  int q_rows;               // bf16 path: q is [Hkv][q_rows][hd], row node * G + g
  float rescale_slack;      // bf16 path: the running max moves only when a block's max exceeds it by this (log2 units)
  int cluster_merge;        // bf16 path: the n_chunks chunk CTAs of a row tile form a cluster and merge through DSMEM
  int* counters;            // bf16 path: [groups][2] chunk arrivals, zero at launch; a layer's own within a step
  uint64_t* trace;          // optional [256 CTAs][16] %globaltimer marks (attention_tc.cu)
};
// fp32 models: one warp per (node, head)
cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s);
// bf16 models: tensor-core kernel; q map over [Hkv * q_rows][128] fp16, kv map
// over the whole cache as [n_layers * 2 * max_batch * Hkv * max_seq][128] fp16,
// both with 64 x 128 boxes and the 128-byte swizzle
struct AttnTcMaps {
  CUtensorMap q, kv;
};
constexpr int kAttnTcRows = 128;   // query rows per CTA
constexpr int kAttnTcKeys = 64;    // keys per block; chunks are multiples of it
constexpr int kAttnPartCtas = 256; // partial slots: chunked launches stay within this many CTAs
constexpr int kAttnMaxChunks = 16; // key chunks per (sequence, kv head, row tile) at most
cudaError_t launch_attention_tc(const AttnArgs& a, const AttnTcMaps& maps, cudaStream_t s, bool pdl);
size_t attention_tc_smem_bytes();
// also max_clusters[cs] (cs = 0 .. kAttnMaxChunks): clusters of cs chunk CTAs the GPU holds at once
cudaError_t attention_tc_configure(int* max_clusters);

// LM head reductions
// with err (optional): when the error word is non-zero (an earlier kernel gave up on a
// wait), every row gets argmax -1 and top1 = top2 = NaN instead
cudaError_t launch_top2_reduce(int M, int tiles, const Top2* part, int top_ld, int32_t* argmax, float* top1,
                               float* top2, cudaStream_t s, bool pdl, const uint32_t* err = nullptr);
// (with inv_temp > 0, the sampled choice of each row as in GemmTcArgs)
cudaError_t launch_rows_top2_f32(int M, int V, const float* logits, int32_t* argmax, float* top1, float* top2,
                                 cudaStream_t s, float inv_temp = 0.f, uint32_t seed_lo = 0, uint32_t seed_hi = 0,
                                 const int32_t* row_sid = nullptr, const int32_t* row_pos = nullptr);

// acceptance walk (or commit-all for prefill chains) + state update
struct WalkArgs {
  StepView sv;
  const int32_t* argmax;    // [M]
  int32_t* acc_len;         // [B]
  int32_t* acc_nodes;       // [B][max_nodes]
  int32_t* acc_tokens;      // [B][max_nodes]
  int32_t* bonus;           // [B]
  int max_nodes;
  int mode;
};
cudaError_t launch_accept_walk(const WalkArgs& w, cudaStream_t s, bool pdl);
cudaError_t kv_compact_configure(size_t smem);
// move accepted nodes' K/V to slots P+1..P+a (all layers, heads)
// draft-head features: the residual stream (fp32 [M][d]) as bf16 rows of out, and the rows of
// each tree's emitted path (root, accepted nodes) from tap [3][Mpad][d] to out [B][max_nodes][3][d]
cudaError_t launch_feature_tap(int M, int d, const float* x, __nv_bfloat16* out, cudaStream_t s, bool pdl);
cudaError_t launch_feature_rows_out(int M, const __nv_bfloat16* tap, int Mpad, int d, __nv_bfloat16* out,
                                    cudaStream_t s, bool pdl);
cudaError_t launch_feature_gather(const StepView& sv, const int32_t* acc_len, const int32_t* acc_nodes,
                                  int max_nodes, const __nv_bfloat16* tap, int Mpad, int d, __nv_bfloat16* out,
                                  cudaStream_t s, bool pdl);
cudaError_t launch_kv_compact(const StepView& sv, const KvView& kv, int n_layers, const int32_t* acc_len,
                              const int32_t* acc_nodes, int max_nodes, cudaStream_t s, bool pdl);

// draft-head pieces
cudaError_t launch_gather_concat(int M, int d, const __nv_bfloat16* g, const int32_t* tokens,
                                 const __nv_bfloat16* embed, __nv_bfloat16* out, cudaStream_t s);

}  // namespace spec
