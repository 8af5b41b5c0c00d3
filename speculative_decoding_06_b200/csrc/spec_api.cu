// C ABI of the tree-verification library: argument validation, workspace
// layout, TMA descriptors, the per-step kernel sequence and CUDA-graph replay.
//
// One verification step (all on the caller's stream):
//   embed_meta      depth / position / ancestor bits per node, embedding, RMSNorm
//   per layer:      QKV GEMM -> rotary + K/V store -> tree attention -> O GEMM ->
//                   residual + RMSNorm -> gate/up GEMM + SwiGLU -> down GEMM ->
//                   residual + RMSNorm
//   LM head GEMM with a fused per-token argmax, then a small cross-tile reduction
//   acceptance walk (one warp per tree) + sequence state update
//   K/V compaction of the accepted path
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/spec.h"
#include "common.cuh"
#include "kernels.h"

using namespace spec;

namespace {

constexpr int kMaxNodesLimit = 128;  // ancestor bitmask is two 64-bit words
constexpr int kMaxSplits = 16;
// split-K arrival counters: one region per (launch, phase) of a step, all zeroed
// when the step starts, so no kernel has to reset them
constexpr int kMaxAttnChunks = kAttnMaxChunks;  // key chunks of one (sequence, kv head, row tile)
constexpr int kDraftTopK = SPEC_DRAFT_TOPK;  // candidates per draft node
constexpr int kCountersPerPhase = 1024;  // two ints per split-K tile (<= 2 x 296 resident CTAs), one per stream-K tile
constexpr int kSkMaxCtas = 320;          // stream-K phases run on at most this many CTAs (their partial slots)

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }

struct WsLayout {
  size_t total = 0;
  int Mmax = 0, Mpad = 0, splits_cap = 1, chunks_cap = 1;
  // parameter block (one host->device copy per step)
  size_t p_tokens, p_parents, p_node_off, p_seq_ids, p_dlen, p_order, p_err, p_end;
  // per-row metadata
  size_t row_seq, row_local, row_slot, row_sid, row_pos, row_anc, rope_cs, P_step;
  // persistent state
  size_t seq_len, pending, hist, err_sticky;
  // activations
  size_t x, xn, q, attn, hmlp, partial, part_o, part_lse, top_part, argmax, top1, top2, inv_freq;
  size_t ss, gemm_ctr, attn_ctr, phase_bar;
  int gemm_ctr_n = 0;  // ints: 4 phases x launches of a step x kCountersPerPhase
  // draft head: split features [2 Mpad][3d], [g|e] operand [2 Mpad][2d], logits, top-k
  size_t fsplit = 0, ge = 0, cand_v = 0, cand_i = 0, cand_lse = 0, dtop_i = 0, dtop_v = 0;
  // feature tap: bf16 residual stream after the three feature layers [3][Mpad][d]
  size_t tap = 0;
  // dynamic draft tree: per-tree nodes and offers, saved root features, per-row top-k and log-sum-exp, output
  size_t tr_tok = 0, tr_par = 0, tr_val = 0, tr_offers = 0, tr_noff = 0, tr_groot = 0, tr_lse = 0, tr_top_i = 0,
         tr_top_v = 0, tr_out_tok = 0, tr_out_par = 0, tr_out_val = 0;
  int n_ss = 1, attn_ctr_n = 0, phase_bar_n = 0;
  size_t partial_bytes;
  // outputs (one device->host copy per step)
  size_t o_acc_len, o_acc_nodes, o_acc_tokens, o_bonus, o_end;
};

WsLayout make_layout(const spec_config& c) {
  WsLayout L;
  const size_t es = c.dtype == SPEC_DTYPE_BF16 ? 2 : 4;
  L.Mmax = c.max_batch * c.max_nodes;
  L.Mpad = (int)align_up(L.Mmax, 128);
  L.splits_cap = L.Mpad <= 256 ? kMaxSplits : 2;
  L.chunks_cap = kMaxAttnChunks;
  const int qd = c.n_q_heads * c.head_dim;
  const int nqkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.p_tokens = take(4 * (size_t)L.Mmax);
  L.p_parents = take(4 * (size_t)L.Mmax);
  L.p_node_off = take(4 * (size_t)(c.max_batch + 1));
  L.p_seq_ids = take(4 * (size_t)c.max_batch);
  L.p_dlen = take(4 * (size_t)c.max_batch);
  L.p_order = take(4 * (size_t)c.max_batch);
  L.p_err = take(16);
  L.p_end = off;
  L.row_seq = take(4 * (size_t)L.Mmax);
  L.row_local = take(4 * (size_t)L.Mmax);
  L.row_slot = take(4 * (size_t)L.Mmax);
  L.row_sid = take(4 * (size_t)L.Mmax);
  L.row_pos = take(4 * (size_t)L.Mmax);
  L.row_anc = take(16 * (size_t)L.Mmax);
  L.rope_cs = take(8 * (size_t)L.Mmax * (c.head_dim / 2));
  L.P_step = take(4 * (size_t)c.max_batch);
  L.seq_len = take(4 * (size_t)c.max_batch);
  L.pending = take(4 * (size_t)c.max_batch);
  L.hist = take(4 * (size_t)c.max_batch * c.max_seq);
  L.err_sticky = take(16);
  L.inv_freq = take(8 * (size_t)(c.head_dim / 2));
  L.x = take(4 * (size_t)L.Mpad * c.hidden);
  // bf16 models keep GEMM activations as split bf16 (hi and lo rows): 2 x Mpad rows of 2 bytes
  const size_t arows = c.dtype == SPEC_DTYPE_BF16 ? 2 * (size_t)L.Mpad : (size_t)L.Mpad;
  L.xn = take(es * arows * c.hidden);
  L.q = take(es * (size_t)L.Mpad * qd * (c.dtype == SPEC_DTYPE_BF16 ? 2 : 1));  // bf16 models: hi and lo parts
  L.attn = take(es * arows * qd);
  L.hmlp = take(es * arows * c.ffn);
  size_t pcols = (size_t)std::max(nqkv, c.hidden) * (c.dtype == SPEC_DTYPE_BF16 ? L.splits_cap : 1);
  if (c.dtype == SPEC_DTYPE_F32) pcols = std::max<size_t>(pcols, std::max<size_t>(2 * (size_t)c.ffn, c.vocab));
  L.partial_bytes = 4 * (size_t)L.Mpad * pcols;
  // stream-K hand-over slots: [resident CTAs][128 rows][BN <= 128 tokens] fp32
  if (c.dtype == SPEC_DTYPE_BF16) L.partial_bytes = std::max(L.partial_bytes, 4 * (size_t)kSkMaxCtas * 128 * 128);
  L.partial = take(L.partial_bytes);
  if (c.dtype == SPEC_DTYPE_BF16) {
    // chunked tensor-core attention: one [128 rows][hd] partial per CTA
    L.part_o = take(4 * (size_t)kAttnPartCtas * kAttnTcRows * c.head_dim);
    L.part_lse = take(4 * (size_t)kAttnPartCtas * kAttnTcRows);
  } else {
    L.part_o = take(4);
    L.part_lse = take(4);
  }
  L.top_part = take(sizeof(Top2) * (size_t)ceil_div(c.vocab, 128) * L.Mpad);
  L.n_ss = std::max(1, c.hidden / 128);
  L.ss = take(4 * (size_t)L.n_ss * L.Mpad);
  // launches of a step: the first QKV and one per layer (verification); three (draft step)
  L.gemm_ctr_n = 4 * std::max(c.n_layers + 1, 3) * kCountersPerPhase;
  L.gemm_ctr = take(4 * (size_t)L.gemm_ctr_n);
  L.phase_bar_n = 4 * (c.n_layers + 2);
  L.phase_bar = take(4 * (size_t)L.phase_bar_n);
  L.attn_ctr_n = 2 * kAttnPartCtas * (c.n_layers + 1);  // per layer, the draft head's last

  L.attn_ctr = take(4 * (size_t)L.attn_ctr_n);
  L.argmax = take(4 * (size_t)L.Mpad);
  L.top1 = take(4 * (size_t)L.Mpad);
  L.top2 = take(4 * (size_t)L.Mpad);
  if (c.feature_layers[0] > 0) L.tap = take(2 * 3 * (size_t)L.Mpad * c.hidden);
  if (c.draft_head) {
    L.fsplit = take(2 * 2 * (size_t)L.Mpad * 3 * c.hidden);
    L.ge = take(2 * 2 * (size_t)L.Mpad * 2 * c.hidden);
    // the draft LM head's top-k candidates: per row and 128-row vocabulary tile,
    // kCandSlots (value, index) holding the tile's k <= 16 best, and (max, sum of exp)
    const size_t vtiles = ((size_t)c.vocab + 127) / 128;
    L.cand_v = take(4 * (size_t)L.Mpad * vtiles * kCandSlots);
    L.cand_i = take(4 * (size_t)L.Mpad * vtiles * kCandSlots);
    L.cand_lse = take(8 * (size_t)L.Mpad * vtiles);
    L.dtop_i = take(4 * (size_t)L.Mpad * kDraftTopK);
    L.dtop_v = take(4 * (size_t)L.Mpad * kDraftTopK);
    const size_t tn = (size_t)c.max_batch * kTreeMaxNodes;
    L.tr_tok = take(4 * tn);
    L.tr_par = take(4 * tn);
    L.tr_val = take(4 * tn);
    L.tr_offers = take(sizeof(TreeOffer) * (size_t)c.max_batch * kTreeMaxOffers);
    L.tr_noff = take(4 * (size_t)c.max_batch);
    L.tr_groot = take(2 * 2 * (size_t)c.max_batch * c.hidden);
    L.tr_lse = take(4 * (size_t)L.Mpad);
    L.tr_top_i = take(4 * (size_t)L.Mpad * kTopKMax);
    L.tr_top_v = take(4 * (size_t)L.Mpad * kTopKMax);
    L.tr_out_tok = take(4 * tn);
    L.tr_out_par = take(4 * tn);
    L.tr_out_val = take(4 * tn);
  }
  const size_t o0 = off;
  L.o_acc_len = take(4 * (size_t)c.max_batch);
  L.o_acc_nodes = take(4 * (size_t)c.max_batch * c.max_nodes);
  L.o_acc_tokens = take(4 * (size_t)c.max_batch * c.max_nodes);
  L.o_bonus = take(4 * (size_t)c.max_batch);
  L.o_end = off;
  (void)o0;
  L.total = off;
  return L;
}

// decoder layers with a K/V cache: the target's, plus the draft head's one layer
int cache_layers(const spec_config& c) { return c.n_layers + (c.draft_head ? 1 : 0); }

// planes per cache layer: K and V; bf16 models add K_lo = fp16(k - fp16(k)) for the attention scores
int cache_planes(const spec_config& c) { return c.dtype == SPEC_DTYPE_BF16 ? 3 : 2; }

size_t kv_bytes_of(const spec_config& c) {
  const size_t es = c.dtype == SPEC_DTYPE_BF16 ? 2 : 4;
  return (size_t)cache_layers(c) * cache_planes(c) * c.max_batch * c.n_kv_heads * (size_t)c.max_seq * c.head_dim * es;
}

std::string check_config(const spec_config* c) {
  if (!c) return "config is NULL";
  if (c->n_layers < 1 || c->hidden < 1 || c->n_q_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 2 || c->ffn < 1 ||
      c->vocab < 2)
    return "all model dimensions must be positive";
  if (c->n_q_heads % c->n_kv_heads) return "n_q_heads must be a multiple of n_kv_heads";
  if (c->dtype != SPEC_DTYPE_F32 && c->dtype != SPEC_DTYPE_BF16) return "dtype must be SPEC_DTYPE_F32 or SPEC_DTYPE_BF16";
  if (c->max_batch < 1 || c->max_seq < 2 || c->max_nodes < 1) return "max_batch, max_seq, max_nodes must be positive";
  if (c->max_nodes > kMaxNodesLimit) return "max_nodes must be <= 128";
  if (c->max_nodes > c->max_seq) return "max_nodes must be <= max_seq";
  if (!(c->rms_eps > 0.f) || !(c->rope_theta > 1.f)) return "rms_eps must be > 0 and rope_theta > 1";
  if (c->dtype == SPEC_DTYPE_BF16) {
    if (c->head_dim != 128) return "bf16 models need head_dim == 128";
    if (c->hidden % 128) return "bf16 models need hidden % 128 == 0";
    if (c->ffn % 64) return "bf16 models need ffn % 64 == 0";
  } else {
    if (c->head_dim > 128 || c->head_dim % 2) return "fp32 models need an even head_dim <= 128";
    if (c->hidden % 4) return "fp32 models need hidden % 4 == 0";
  }
  if (c->draft_head && c->dtype != SPEC_DTYPE_BF16) return "the draft head is bf16 only";
  if (c->draft_vocab < 0 || c->draft_vocab == 1 || c->draft_vocab > c->vocab)
    return "draft_vocab must be 0 or in [2, vocab]";
  if (c->draft_vocab && !c->draft_head) return "draft_vocab needs the draft head";
  const int* fl = c->feature_layers;
  if (fl[0] || fl[1] || fl[2]) {
    for (int f = 0; f < 3; ++f)
      if (fl[f] < 1 || fl[f] > c->n_layers) return "feature_layers must all be 0 or each in [1, n_layers]";
    if (c->hidden % 8) return "feature taps need hidden % 8 == 0";
  }
  return "";
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [rows][cols] bf16, row-major; boxes of 64 columns x box_rows rows, 128-byte swizzle
bool make_tmap(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
               CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct LayerMaps {
  CUtensorMap wq, wk, wv, wo, wg, wu, wd;
};

struct GemmPlan {
  int bn, tiles_o, tiles_t, splits, kbps, grid;
  int sk = 0;  // stream-K over all resident CTAs (GemmTcArgs::streamk)
  int sk_tiles = 0;  // the tiles it shares out (the others go whole, round-robin)
};

struct StepPlan {
  int B, M, max_n, max_lk, n_chunks, chunk, max_rows;
  int cluster_merge = 0;  // attention chunks merge through DSMEM (all groups' clusters co-resident)
  int grid_all;  // co-resident CTAs of the multi-phase GEMM launches
  GemmPlan qkv, o, gu, down, lm;
};

using GraphKey = std::tuple<int, int, int, int, int, int, int, int>;

}  // namespace

struct spec_handle {
  spec_config cfg{};
  WsLayout lay;
  int device = 0;
  int sm_count = 148;
  cudaStream_t stream = nullptr;
  const void* embed = nullptr;
  const void* final_norm = nullptr;
  const void* lm_head = nullptr;
  std::vector<spec_layer_weights> layers;
  KvView kv{};
  uint8_t* ws = nullptr;
  std::vector<LayerMaps> maps;
  CUtensorMap map_lm;
  CUtensorMap map_xn[4], map_attn[4], map_h[4];  // B operands for BN = 64, 128, 96, 80 (bn_slot)
  AttnTcMaps attn_maps;                           // q and the K/V cache (fp16)
  // draft head (cfg.draft_head): its decoder layer is layers[n_layers], maps[n_layers]
  const void* draft_fc_fuse = nullptr;
  const void* draft_fc_in = nullptr;
  const void* draft_final_norm = nullptr;
  const void* draft_lm_head = nullptr;     // reduced draft vocabulary: [draft_vocab][d]
  const int32_t* draft_ids = nullptr;      // its token ids (device)
  CUtensorMap map_lm_draft;
  CUtensorMap map_fc_fuse, map_fc_in, map_fsplit[4], map_ge[4];
  std::vector<int32_t> dlen;        // draft-head prefix length per sequence
  std::vector<uint8_t> dready;
  int resident[4][4] = {};  // co-resident CTAs per SM [bn_slot][epi]
  int occ_api[4][4] = {};   // what the occupancy query reported
  // host mirror of per-sequence state
  std::vector<int32_t> len, pending;
  std::vector<int32_t> len_hi;  // upper bound while device-output steps are in flight
  std::vector<uint8_t> ready;   // prefilled
  bool stale = false;
  // pinned staging
  uint8_t* h_params = nullptr;
  uint8_t* h_out = nullptr;
  float* dbg_logits = nullptr;
  size_t dbg_bytes = 0;
  float temperature = 0.f;  // > 0: tokens are sampled (spec_set_sampling); 0: greedy
  uint64_t seed = 0;
  void* feat_out = nullptr;  // SPEC_FEATURES destination, bf16 [B][max_nodes][3][d]
  size_t feat_bytes = 0;
  void* pf_feat_out = nullptr;  // features of the prefill chunk being run, bf16 [rows][3][d]
  std::map<GraphKey, cudaGraphExec_t> graphs;
  bool use_pdl = true;
  int max_splits = 16;    // split-K cap
  int max_chunks = kMaxAttnChunks;  // attention key-chunk cap
  int resident_cap = 0;   // 0: as many CTAs per SM as fit
  int streamk = -1;       // stream-K when whole tiles leave CTAs idle: 1 for the SWIGLU, ARGMAX and TOPK
                          // phases, 2 for SWIGLU only, 0 off, -1 (default, the measured best) the LM heads'
                          // ARGMAX and TOPK and SWIGLU at 80- to 128-token tiles, where one CTA per SM leaves
                          // the most idle (SPEC_TUNE sk=)
  float rescale_slack = 8.f;  // attention: running-max slack in log2 units (p <= 2^slack)
  int attn_clusters[kAttnMaxChunks + 1] = {};  // co-resident clusters of n chunk CTAs
  bool attn_dsmem = true;     // merge chunk partials through distributed shared memory when they fit a cluster
  bool sk_hybrid = true;      // stream-K shares only the last round's tiles (else every tile)
  int bn64_max = 64;          // largest token count planned with 64-token tiles (several token tiles above 64)
  bool bn80 = true;           // 80-token tiles for 65 .. 80 tokens (6 stages: as many weight bytes in flight as at 64)
  bool bn96 = true;           // 96-token tiles for 65 (81) .. 96 tokens (else 128)
  // L2 prefetch of weights ahead of the GEMM that streams them
  uint64_t* trace = nullptr;  // optional GEMM timeline of one layer's launch
  size_t trace_bytes = 0;
  int trace_layer = 0;
  std::string err;
  // profiler: an event pair per launch
  bool prof = false;
  std::vector<cudaEvent_t> ev_pool;
  std::vector<std::pair<int, int>> prof_marks;  // (class, index of first event of the pair)
  int launches = 0;

  template <typename T>
  T* W(size_t off) const { return reinterpret_cast<T*>(ws + off); }
};

namespace {

int fail(spec_handle* h, int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  return code;
}

#define CUDA_TRY(h, call)                                                                      \
  do {                                                                                         \
    cudaError_t e__ = (call);                                                                  \
    if (e__ != cudaSuccess)                                                                    \
      return fail(h, SPEC_ERR_CUDA, "%s failed: %s (%s)", #call, cudaGetErrorName(e__),        \
                  cudaGetErrorString(e__));                                                    \
  } while (0)

// Launch wrapper: counts launches and, when profiling, brackets each one with events.
template <typename F>
cudaError_t launch_k(spec_handle* h, int cls, int n_kernels, F&& fn) {
  int i0 = -1;
  if (h->prof) {
    i0 = (int)(2 * h->prof_marks.size());
    while ((int)h->ev_pool.size() < i0 + 2) {
      cudaEvent_t e;
      cudaError_t r = cudaEventCreate(&e);
      if (r != cudaSuccess) return r;
      h->ev_pool.push_back(e);
    }
    cudaError_t r = cudaEventRecord(h->ev_pool[i0], h->stream);
    if (r != cudaSuccess) return r;
  }
  cudaError_t e = fn();
  if (e != cudaSuccess) return e;
  h->launches += n_kernels;
  if (h->prof) {
    cudaError_t r = cudaEventRecord(h->ev_pool[i0 + 1], h->stream);
    if (r != cudaSuccess) return r;
    h->prof_marks.emplace_back(cls, i0);
  }
  return cudaSuccess;
}

// index of a token-tile width in the per-width tables (tensor maps, residency)
int bn_slot(int bn) { return bn == 64 ? 0 : bn == 128 ? 1 : bn == 96 ? 2 : 3; }
constexpr int kNumTileWidths = 4;
constexpr int kTileWidths[kNumTileWidths] = {64, 128, 96, 80};

GemmPlan plan_gemm(const spec_handle* h, int rows_per_tile, int n_out, int K, int M, int epi) {
  GemmPlan p;
  p.bn = M <= h->bn64_max ? 64 : (h->bn80 && M <= 80 ? 80 : (h->bn96 && M <= 96 ? 96 : 128));
  const int bi = bn_slot(p.bn);
  int per_sm = std::max(1, h->resident[bi][0]);  // one kernel function for every epilogue
  if (h->resident_cap > 0) per_sm = std::min(per_sm, h->resident_cap);
  const int resident = per_sm * h->sm_count;
  p.tiles_o = ceil_div(n_out, rows_per_tile);
  p.tiles_t = ceil_div(M, p.bn);
  const int KB = K / 64;
  const int base = p.tiles_o * p.tiles_t;
  int S = 1;
  if (epi == GEMM_EPI_QKV || epi == GEMM_EPI_RESID) {
    // split-K only while every tile x split CTA can be resident at once: the
    // splits of a tile wait for one another
    const int cap = std::min(std::min(h->lay.splits_cap, h->max_splits), std::max(1, KB / 4));
    S = std::max(1, std::min(cap, resident / std::max(1, base)));
  }
  p.kbps = ceil_div(KB, S);
  p.splits = ceil_div(KB, p.kbps);  // no empty split
  p.grid = p.splits > 1 ? base * p.splits : std::min(base, resident);
  // Stream-K for the phases without split-K when whole tiles would leave CTAs
  // idle in the last round (more than 2 % of the CTA-rounds): the last round's
  // tiles (all of them when there are fewer tiles than CTAs) are shared out so
  // that every resident CTA streams the same number of weight k-blocks; the
  // earlier rounds' tiles go whole.
  const bool sk_epi = h->streamk == 1   ? (epi == GEMM_EPI_SWIGLU || epi == GEMM_EPI_ARGMAX || epi == GEMM_EPI_TOPK)
                      : h->streamk == 2 ? epi == GEMM_EPI_SWIGLU
                                        : h->streamk < 0 && (epi == GEMM_EPI_ARGMAX || epi == GEMM_EPI_TOPK ||
                                                             (epi == GEMM_EPI_SWIGLU && p.bn > 64));
  const int sk_tiles = (base < resident || !h->sk_hybrid) ? base : base % resident;
  if (sk_epi && p.splits == 1 && sk_tiles > 0 &&
      resident <= kSkMaxCtas && base <= kCountersPerPhase && (long long)sk_tiles * KB >= 2LL * resident &&
      (size_t)resident * 128 * p.bn * 4 <= h->lay.partial_bytes) {
    const long long rounds = ceil_div(base, resident);
    if (rounds * resident * 100 > 102LL * base) {
      p.sk = 1;
      p.sk_tiles = sk_tiles;
      p.grid = resident;
    }
  }
  return p;
}

StepPlan make_plan(const spec_handle* h, int B, int M, int max_n, int max_lk) {
  const spec_config& c = h->cfg;
  StepPlan s;
  s.B = B;
  s.M = M;
  s.max_n = max_n;
  s.max_lk = max_lk;
  const int G = c.n_q_heads / c.n_kv_heads;
  s.max_rows = max_n * G;
  if (c.dtype == SPEC_DTYPE_BF16) {
    // Key chunks only while the (sequence, kv head, row tile) groups leave SMs
    // idle; the chunk CTAs of a group meet, so a chunked grid stays within one
    // CTA per SM (all co-resident) and within the partial slots.
    const int groups = B * c.n_kv_heads * ceil_div(s.max_rows, kAttnTcRows);
    const int blocks = ceil_div(max_lk, kAttnTcKeys);
    const int cap = std::min(h->sm_count, kAttnPartCtas);
    int nc = 1;
    if (2 * groups <= cap) nc = std::max(1, std::min({blocks, cap / groups, h->max_chunks}));
    s.chunk = ceil_div(blocks, nc) * kAttnTcKeys;
    s.n_chunks = ceil_div(max_lk, s.chunk);
    // the chunk CTAs of a group merge through distributed shared memory when
    // every group's cluster fits on the GPU at once (else through global memory)
    s.cluster_merge = (h->attn_dsmem && s.n_chunks > 1 && s.n_chunks <= kAttnMaxChunks &&
                       h->attn_clusters[s.n_chunks] >= groups) ? 1 : 0;
  } else {
    s.chunk = max_lk;
    s.n_chunks = 1;
  }
  const int nqkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  const int qd = c.n_q_heads * c.head_dim;
  s.qkv = plan_gemm(h, 128, nqkv, c.hidden, M, GEMM_EPI_QKV);
  s.o = plan_gemm(h, 128, c.hidden, qd, M, GEMM_EPI_RESID);
  s.gu = plan_gemm(h, 64, c.ffn, c.hidden, M, GEMM_EPI_SWIGLU);
  s.down = plan_gemm(h, 128, c.hidden, c.ffn, M, GEMM_EPI_RESID);
  s.lm = plan_gemm(h, 128, c.vocab, c.hidden, M, GEMM_EPI_ARGMAX);
  {
    const int bi = bn_slot(s.qkv.bn);
    int per_sm = std::max(1, h->resident[bi][0]);
    if (h->resident_cap > 0) per_sm = std::min(per_sm, h->resident_cap);
    s.grid_all = per_sm * h->sm_count;
  }
  return s;
}

StepView make_view(spec_handle* h, int B, int M) {
  const WsLayout& L = h->lay;
  StepView v;
  v.tokens = h->W<int32_t>(L.p_tokens);
  v.parents = h->W<int32_t>(L.p_parents);
  v.node_off = h->W<int32_t>(L.p_node_off);
  v.seq_ids = h->W<int32_t>(L.p_seq_ids);
  v.order = h->W<int32_t>(L.p_order);
  v.B = B;
  v.M = M;
  v.row_seq = h->W<int32_t>(L.row_seq);
  v.row_local = h->W<int32_t>(L.row_local);
  v.row_slot = h->W<int32_t>(L.row_slot);
  v.row_sid = h->W<int32_t>(L.row_sid);
  v.row_pos = h->W<int32_t>(L.row_pos);
  v.row_anc = h->W<uint64_t>(L.row_anc);
  v.rope_cs = h->W<float2>(L.rope_cs);
  v.P_step = h->W<int32_t>(L.P_step);
  v.seq_len = h->W<int32_t>(L.seq_len);
  v.pending = h->W<int32_t>(L.pending);
  v.hist = h->W<int32_t>(L.hist);
  v.max_seq = h->cfg.max_seq;
  v.err = h->W<uint32_t>(L.p_err);
  v.err_sticky = h->W<uint32_t>(L.err_sticky);

  return v;
}

GemmTcLaunch gemm_launch(const GemmPlan& p, int epi, int n_out, int K, int M, const CUtensorMap* a0,
                         const CUtensorMap* a1, const CUtensorMap* a2, const CUtensorMap* b, int s0, int s1, int s2,
                         uint32_t* err) {
  GemmTcLaunch L{};
  L.bn = p.bn;
  L.epi = epi;
  L.grid = p.grid;
  L.mA0 = a0;
  L.mA1 = a1 ? a1 : a0;
  L.mA2 = a2 ? a2 : a0;
  L.mB = b;
  L.args.n_out = n_out;
  L.args.K = K;
  L.args.M = M;
  L.args.tiles_o = p.tiles_o;
  L.args.tiles_t = p.tiles_t;
  L.args.splits = p.splits;
  L.args.kb_per_split = p.kbps;
  L.args.streamk = p.sk;
  L.args.sk_tiles = p.sk_tiles;
  L.args.seg_rows[0] = s0;
  L.args.seg_rows[1] = s1;
  L.args.seg_rows[2] = s2;
  L.args.err = err;
  return L;
}

#define CUDA_RET(expr)                   \
  do {                                   \
    cudaError_t e_ = (expr);             \
    if (e_ != cudaSuccess) return e_;    \
  } while (0)

// Enqueue the whole step (everything after the parameter upload).
#define LK(cls, nk, expr)                                                             \
  do {                                                                                \
    cudaError_t e_ = launch_k(h, cls, nk, [&]() { return (expr); });                  \
    if (e_ != cudaSuccess) return e_;                                                 \
  } while (0)

// The GEMM phases of the bf16 path, for decoder layer l (the draft head's
// layer is index n_layers).  Split-K counters: one region per phase slot.
struct PhaseBuilder {
  spec_handle* h;
  const StepPlan& sp;
  const StepView& sv;
  int bi, d, qd, kvd, nqkv, M;
  PhaseBuilder(spec_handle* h_, const StepPlan& sp_, const StepView& sv_) : h(h_), sp(sp_), sv(sv_) {
    const spec_config& c = h->cfg;
    bi = bn_slot(sp.qkv.bn);
    d = c.hidden;
    qd = c.n_q_heads * c.head_dim;
    kvd = c.n_kv_heads * c.head_dim;
    nqkv = qd + 2 * kvd;
    M = sp.M;
  }
  static GemmPhase as_phase(const GemmTcLaunch& g) {
    GemmPhase q{};
    q.epi = g.epi;
    q.mA0 = g.mA0;
    q.mA1 = g.mA1;
    q.mA2 = g.mA2;
    q.mB = g.mB;
    q.args = g.args;
    return q;
  }
  // counters of phase `slot` of launch `launch` within the step
  int* ctr(int region) const { return h->W<int>(h->lay.gemm_ctr) + region * kCountersPerPhase; }
  GemmPhase qkv(int l, int slot) const {
    const spec_config& c = h->cfg;
    const WsLayout& L = h->lay;
    const LayerMaps& mp = h->maps[l];
    __half* kc = reinterpret_cast<__half*>(h->kv.base) + (size_t)l * h->kv.layer_stride();
    GemmTcLaunch g = gemm_launch(sp.qkv, GEMM_EPI_QKV, nqkv, d, M, &mp.wq, &mp.wk, &mp.wv, &h->map_xn[bi], qd, kvd,
                                 kvd, sv.err);
    g.args.ss_in = h->W<float>(L.ss);
    g.args.n_ss = L.n_ss;
    g.args.ss_ld = L.Mpad;
    g.args.norm_d = d;
    g.args.eps = c.rms_eps;
    g.args.part = h->W<float>(L.partial);
    g.args.split_stride = (size_t)L.Mpad * nqkv;
    g.args.counters = ctr(slot);
    g.args.row_seq = sv.row_seq;
    g.args.row_local = sv.row_local;
    g.args.row_slot = sv.row_slot;
    g.args.row_sid = sv.row_sid;
    g.args.P_step = sv.P_step;
    g.args.seq_ids = sv.seq_ids;
    g.args.rope_cs = sv.rope_cs;
    g.args.q_out = h->W<__half>(L.q);
    g.args.q_rows = L.Mpad * (c.n_q_heads / c.n_kv_heads);
    g.args.k_cache = kc;
    g.args.v_cache = kc + h->kv.kv_stride();
    g.args.klo_cache = kc + 2 * h->kv.kv_stride();
    g.args.kv_seq_stride = h->kv.seq_stride();
    g.args.kv_head_stride = h->kv.head_stride();
    g.args.Hq = c.n_q_heads;
    g.args.Hkv = c.n_kv_heads;
    g.args.max_seq = c.max_seq;
    return as_phase(g);
  }
  // x += A.W^T; xn = split(x * norm_next); ss = per-tile sums of squares
  GemmPhase resid(const GemmPlan& pl, int K, const CUtensorMap* mw, const CUtensorMap* mb, const void* norm_next,
                  int slot) const {
    const WsLayout& L = h->lay;
    GemmTcLaunch g = gemm_launch(pl, GEMM_EPI_RESID, d, K, M, mw, nullptr, nullptr, mb, d, 0, 0, sv.err);
    g.args.part = h->W<float>(L.partial);
    g.args.split_stride = (size_t)L.Mpad * d;
    g.args.counters = ctr(slot);
    g.args.x = h->W<float>(L.x);
    g.args.norm_w_next = reinterpret_cast<const __nv_bfloat16*>(norm_next);
    g.args.xn_out = h->W<__nv_bfloat16>(L.xn);
    g.args.ss_out = h->W<float>(L.ss);
    g.args.ss_ld = L.Mpad;
    return as_phase(g);
  }
  GemmPhase o(int l, int slot) const {
    return resid(sp.o, qd, &h->maps[l].wo, &h->map_attn[bi], h->layers[l].mlp_norm, slot);
  }
  GemmPhase down(int l, int slot, const void* next_norm) const {
    return resid(sp.down, h->cfg.ffn, &h->maps[l].wd, &h->map_h[bi], next_norm, slot);
  }
  GemmPhase gu(int l, int slot) const {
    const spec_config& c = h->cfg;
    const WsLayout& L = h->lay;
    GemmTcLaunch g = gemm_launch(sp.gu, GEMM_EPI_SWIGLU, c.ffn, d, M, &h->maps[l].wg, &h->maps[l].wu, nullptr,
                                 &h->map_xn[bi], 0, 0, 0, sv.err);
    g.args.part = h->W<float>(L.partial);  // stream-K hand-over slots
    g.args.counters = ctr(slot);
    g.args.ss_in = h->W<float>(L.ss);
    g.args.n_ss = L.n_ss;
    g.args.ss_ld = L.Mpad;
    g.args.norm_d = d;
    g.args.eps = c.rms_eps;
    g.args.out_bf16 = h->W<__nv_bfloat16>(L.hmlp);
    g.args.ld_out = c.ffn;
    return as_phase(g);
  }
  // final norm (folded) + LM head with per-tile top-2; logits also stored when given;
  // with `sample`, the top-2 is of the temperature-scaled logits plus the Gumbel noise
  // the draft head's LM head: per row and vocabulary tile, the tile's k best and (max,
  // sum of exp) for launch_topk_merge; logits (optional) get the logits themselves
  GemmPhase lm_topk(float* logits, const GemmPlan& plan, const CUtensorMap* map, int rows, int k, int slot) const {
    const WsLayout& L = h->lay;
    GemmPhase q = lm_rows(logits, false, plan, map, rows, slot);
    q.epi = GEMM_EPI_TOPK;
    q.args.topk = k;
    q.args.cand_ld = plan.tiles_o;
    q.args.cand_v = h->W<float>(L.cand_v);
    q.args.cand_i = h->W<int32_t>(L.cand_i);
    q.args.cand_lse = h->W<float2>(L.cand_lse);
    return q;
  }
  GemmPhase lm(float* logits, bool sample, int slot) const {
    return lm_rows(logits, sample, sp.lm, &h->map_lm, h->cfg.vocab, slot);
  }
  // the same over a given set of LM-head rows (the reduced draft vocabulary)
  GemmPhase lm_rows(float* logits, bool sample, const GemmPlan& plan, const CUtensorMap* map, int rows,
                    int slot) const {
    const spec_config& c = h->cfg;
    const WsLayout& L = h->lay;
    GemmTcLaunch g = gemm_launch(plan, GEMM_EPI_ARGMAX, rows, d, M, map, nullptr, nullptr, &h->map_xn[bi], rows, 0, 0,
                                 sv.err);
    g.args.part = h->W<float>(L.partial);  // stream-K hand-over slots
    g.args.counters = ctr(slot);
    g.args.top_part = h->W<Top2>(L.top_part);
    g.args.top_ld = L.Mpad;
    g.args.dbg_logits = logits;
    if (sample) {
      g.args.inv_temp = 1.f / h->temperature;
      g.args.seed_lo = (uint32_t)h->seed;
      g.args.seed_hi = (uint32_t)(h->seed >> 32);
      g.args.row_sid = sv.row_sid;
      g.args.row_pos = sv.row_pos;
    }
    g.args.ss_in = h->W<float>(L.ss);
    g.args.n_ss = L.n_ss;
    g.args.ss_ld = L.Mpad;
    g.args.norm_d = d;
    g.args.eps = c.rms_eps;
    return as_phase(g);
  }
};

cudaError_t enqueue_step(spec_handle* h, const StepPlan& sp, int mode, bool dbg, bool feat) {
  const spec_config& c = h->cfg;
  const WsLayout& L = h->lay;
  cudaStream_t st = h->stream;
  const bool pdl = h->use_pdl && !h->prof;
  StepView sv = make_view(h, sp.B, sp.M);
  const int dt = c.dtype == SPEC_DTYPE_BF16 ? 1 : 0;
  const int d = c.hidden, qd = c.n_q_heads * c.head_dim, kvd = c.n_kv_heads * c.head_dim;
  const int nqkv = qd + 2 * kvd;
  const int M = sp.M;
  float* x = h->W<float>(L.x);
  void* xn = h->ws + L.xn;
  void* q = h->ws + L.q;
  void* attn = h->ws + L.attn;
  void* hm = h->ws + L.hmlp;
  float* part = h->W<float>(L.partial);
  h->launches = 0;

  float* ss = h->W<float>(L.ss);
  int* gctr = h->W<int>(L.gemm_ctr);
  // feature tap: after the layer that completes the residual stream of feature layer f
  __nv_bfloat16* tap = feat ? h->W<__nv_bfloat16>(L.tap) : nullptr;
  auto tap_after = [&](int layers_done, bool tpdl) -> cudaError_t {
    if (!feat) return cudaSuccess;
    for (int f = 0; f < 3; ++f)
      if (c.feature_layers[f] == layers_done)
        LK(SPEC_PROF_FEATURES, 1, launch_feature_tap(M, d, x, tap + (size_t)f * L.Mpad * d, st, tpdl));
    return cudaSuccess;
  };
  if (dt == 1) {
    // arrival counters start every step at zero, whatever an earlier failed step left behind
    cudaError_t e0 = cudaMemsetAsync(gctr, 0, 4 * (size_t)L.gemm_ctr_n, st);
    if (e0 == cudaSuccess) e0 = cudaMemsetAsync(h->ws + L.attn_ctr, 0, 4 * (size_t)L.attn_ctr_n, st);
    if (e0 == cudaSuccess) e0 = cudaMemsetAsync(h->ws + L.phase_bar, 0, 4 * (size_t)L.phase_bar_n, st);
    if (e0 != cudaSuccess) return e0;
  }
  LK(SPEC_PROF_EMBED_META, 1,
     launch_embed_meta(dt, sv, h->embed, h->layers[0].attn_norm, d, c.rms_eps, x, xn, ss, L.n_ss, L.Mpad,
                       h->W<double>(L.inv_freq), c.head_dim / 2, mode, st, pdl));

  AttnArgs aa{};
  aa.sv = sv;
  aa.kv = h->kv;
  aa.Hq = c.n_q_heads;
  aa.hd = c.head_dim;
  aa.q = q;
  aa.out = attn;
  aa.part_o = h->W<float>(L.part_o);
  aa.part_lse = h->W<float>(L.part_lse);
  aa.n_chunks = sp.n_chunks;
  aa.chunk = sp.chunk;
  aa.max_rows = sp.max_rows;
  aa.counters = h->W<int>(L.attn_ctr);
  aa.q_rows = L.Mpad * (c.n_q_heads / c.n_kv_heads);
  aa.rescale_slack = h->rescale_slack;
  aa.cluster_merge = sp.cluster_merge;

  const PhaseBuilder pb(h, sp, sv);
  if (dt == 1) {
    GemmMultiLaunch m{};
    m.bn = sp.qkv.bn;
    m.grid = sp.grid_all;
    m.err = sv.err;
    m.phase_bar = h->W<int>(L.phase_bar);
    m.n_phases = 1;
    m.ph[0] = pb.qkv(0, 0);
    LK(SPEC_PROF_GEMM_QKV, 1, gemm_multi_launch(m, st, pdl));
  }

  for (int l = 0; l < c.n_layers; ++l) {
    const spec_layer_weights& lw = h->layers[l];
    const void* next_norm = (l + 1 < c.n_layers) ? h->layers[l + 1].attn_norm : h->final_norm;
    aa.layer = l;
    aa.counters = h->W<int>(L.attn_ctr) + (size_t)l * 2 * kAttnPartCtas;  // this layer's own
    if (dt == 1) {
      // attention of layer l (its QKV ran in the previous launch), then one
      // launch: O, gate/up, down, and the next layer's QKV or the LM head
      // the traced layer's attention and the next layer's (which follows the traced GEMM launch)
      aa.trace = (h->trace && (l == h->trace_layer || l == h->trace_layer + 1))
                     ? h->trace + (size_t)2 * h->sm_count * kMaxGemmPhases * kGemmTraceMarks +
                           (size_t)(l - h->trace_layer) * kAttnPartCtas * 16
                     : nullptr;
      LK(SPEC_PROF_ATTENTION, 1, launch_attention_tc(aa, h->attn_maps, st, pdl));
      GemmMultiLaunch m{};
      m.bn = sp.qkv.bn;
      m.grid = sp.grid_all;
      m.err = sv.err;
      m.phase_bar = h->W<int>(L.phase_bar) + 4 * (l + 1);
      m.n_phases = 4;
      // split-K counter regions 4 * (l + 1) + phase (region 0 is the first QKV launch's)
      m.ph[0] = pb.o(l, 4 * (l + 1) + 0);
      m.ph[1] = pb.gu(l, 4 * (l + 1) + 1);
      m.ph[2] = pb.down(l, 4 * (l + 1) + 2, next_norm);
      m.ph[3] = (l + 1 < c.n_layers) ? pb.qkv(l + 1, 4 * (l + 1) + 3)
                                     : pb.lm(dbg ? h->dbg_logits : nullptr, h->temperature > 0.f, 4 * (l + 1) + 3);
      if (h->trace && l == h->trace_layer) m.trace = h->trace;
      LK(SPEC_PROF_GEMM_LAYER, 1, gemm_multi_launch(m, st, pdl));
      CUDA_RET(tap_after(l + 1, pdl));
    } else {
      const float* xf = reinterpret_cast<const float*>(xn);
      LK(SPEC_PROF_GEMM_QKV, 1, launch_gemm_simt_f32(xf, d, (const float*)lw.wq, d, part, nqkv, M, qd, st));
      LK(SPEC_PROF_GEMM_QKV, 1, launch_gemm_simt_f32(xf, d, (const float*)lw.wk, d, part + qd, nqkv, M, kvd, st));
      LK(SPEC_PROF_GEMM_QKV, 1,
         launch_gemm_simt_f32(xf, d, (const float*)lw.wv, d, part + qd + kvd, nqkv, M, kvd, st));
      LK(SPEC_PROF_ROPE_KV, 1,
         launch_qkv_rope_store(dt, sv, 1, part, 0, c.n_q_heads, c.n_kv_heads, c.head_dim, q, h->kv, l, st, false));
      LK(SPEC_PROF_ATTENTION, 1, launch_attention_f32(aa, st));
      LK(SPEC_PROF_GEMM_O, 1, launch_gemm_simt_f32((const float*)attn, qd, (const float*)lw.wo, qd, part, d, M, d, st));
      LK(SPEC_PROF_RESID_NORM, 1, launch_residual_norm(dt, M, d, 1, part, 0, x, xn, lw.mlp_norm, c.rms_eps, st, false));
      LK(SPEC_PROF_GEMM_GATE_UP, 1,
         launch_gemm_simt_f32(xf, d, (const float*)lw.w_gate, d, part, 2 * c.ffn, M, c.ffn, st));
      LK(SPEC_PROF_GEMM_GATE_UP, 1,
         launch_gemm_simt_f32(xf, d, (const float*)lw.w_up, d, part + c.ffn, 2 * c.ffn, M, c.ffn, st));
      LK(SPEC_PROF_GEMM_GATE_UP, 1, launch_swiglu_f32(M, c.ffn, part, (float*)hm, st));
      LK(SPEC_PROF_GEMM_DOWN, 1,
         launch_gemm_simt_f32((const float*)hm, c.ffn, (const float*)lw.w_down, c.ffn, part, d, M, d, st));
      LK(SPEC_PROF_RESID_NORM, 1, launch_residual_norm(dt, M, d, 1, part, 0, x, xn, next_norm, c.rms_eps, st, false));
      CUDA_RET(tap_after(l + 1, false));
    }
  }

  int32_t* amax = h->W<int32_t>(L.argmax);
  if (dt == 1) {
    // the LM head ran as the last phase of the last layer's launch
    LK(SPEC_PROF_LM_REDUCE, 1,
       launch_top2_reduce(M, sp.lm.tiles_o, h->W<Top2>(L.top_part), L.Mpad, amax, h->W<float>(L.top1),
                          h->W<float>(L.top2), st, pdl));
  } else {
    LK(SPEC_PROF_LM_HEAD, 1,
       launch_gemm_simt_f32((const float*)xn, d, (const float*)h->lm_head, d, part, c.vocab, M, c.vocab, st));
    LK(SPEC_PROF_LM_REDUCE, 1,
       launch_rows_top2_f32(M, c.vocab, part, amax, h->W<float>(L.top1), h->W<float>(L.top2), st,
                            h->temperature > 0.f ? 1.f / h->temperature : 0.f, (uint32_t)h->seed,
                            (uint32_t)(h->seed >> 32), sv.row_sid, sv.row_pos));
    if (dbg && h->dbg_logits) {
      cudaError_t e = cudaMemcpyAsync(h->dbg_logits, part, sizeof(float) * (size_t)M * c.vocab,
                                      cudaMemcpyDeviceToDevice, st);
      if (e != cudaSuccess) return e;
    }
  }

  WalkArgs w{};
  w.sv = sv;
  w.argmax = amax;
  w.acc_len = h->W<int32_t>(L.o_acc_len);
  w.acc_nodes = h->W<int32_t>(L.o_acc_nodes);
  w.acc_tokens = h->W<int32_t>(L.o_acc_tokens);
  w.bonus = h->W<int32_t>(L.o_bonus);
  w.max_nodes = c.max_nodes;
  w.mode = mode;
  LK(SPEC_PROF_WALK, 1, launch_accept_walk(w, st, pdl && dt == 1));
  if (mode == STEP_VERIFY)
    LK(SPEC_PROF_COMPACT, 1,
       launch_kv_compact(sv, h->kv, c.n_layers, w.acc_len, w.acc_nodes, c.max_nodes, st, pdl && dt == 1));
  if (feat && mode == STEP_VERIFY)
    LK(SPEC_PROF_FEATURES, 1,
       launch_feature_gather(sv, w.acc_len, w.acc_nodes, c.max_nodes, tap, L.Mpad, d,
                             static_cast<__nv_bfloat16*>(h->feat_out), st, pdl && dt == 1));
  else if (feat && mode == STEP_PREFILL)
    LK(SPEC_PROF_FEATURES, 1,
       launch_feature_rows_out(M, tap, L.Mpad, d, static_cast<__nv_bfloat16*>(h->pf_feat_out), st, pdl && dt == 1));
  return cudaSuccess;
}

// The draft head's step (A: its input rows, then its decoder layer, LM head and
// top-k).  The draft layer is layer n_layers of the cache; prefix lengths come
// with the parameter block.  With `kv_only` (draft prefill) the step stops once
// the layer's K/V are stored: they depend on the layer input alone.
// One step of the dynamic draft tree: step t over trees of n nodes (n_prev at
// step t - 1), top-k K per row, the tree state.
struct TreeStep {
  int t, n, n_prev, K;
  TreeArgs args;
};

cudaError_t enqueue_draft(spec_handle* h, const StepPlan& sp, bool kv_only, bool dbg, const TreeStep* ts = nullptr) {
  const spec_config& c = h->cfg;
  const WsLayout& L = h->lay;
  cudaStream_t st = h->stream;
  const bool pdl = h->use_pdl && !h->prof;
  StepView sv = make_view(h, sp.B, sp.M);
  sv.seq_len = h->W<int32_t>(L.p_dlen);
  const int d = c.hidden, M = sp.M, Ld = c.n_layers;
  const int bi = bn_slot(sp.qkv.bn);
  h->launches = 0;
  CUDA_RET(cudaMemsetAsync(h->ws + L.gemm_ctr, 0, 4 * (size_t)L.gemm_ctr_n, st));
  CUDA_RET(cudaMemsetAsync(h->ws + L.attn_ctr, 0, 4 * (size_t)L.attn_ctr_n, st));
  CUDA_RET(cudaMemsetAsync(h->ws + L.phase_bar, 0, 4 * (size_t)L.phase_bar_n, st));
  __nv_bfloat16* ge = h->W<__nv_bfloat16>(L.ge);
  // metadata on the draft prefixes; e = E[token] into the right half of [g|e]
  LK(SPEC_PROF_EMBED_META, 1,
     launch_embed_meta(1, sv, h->embed, nullptr, d, c.rms_eps, nullptr, nullptr, nullptr, 0, 0,
                       h->W<double>(L.inv_freq), c.head_dim / 2, STEP_SCORE, st, pdl, ge, 2 * d, d));
  const PhaseBuilder pb(h, sp, sv);
  __nv_bfloat16* groot = h->W<__nv_bfloat16>(L.tr_groot);
  if (ts && ts->t > 0) {
    // a later drafting step: the root keeps its fused target feature, every other
    // node takes its parent's draft output a (the previous step's x)
    LK(SPEC_PROF_DRAFT_FC, 1,
       launch_tree_feature_rows(M, d, 2 * d, ts->n, ts->n_prev, h->W<int32_t>(L.p_parents), groot, h->W<float>(L.x),
                                ge, st, pdl));
  } else {
    // g = [l|m|h] . W_fuse^T into the left half of [g|e]
    const GemmPlan pf = plan_gemm(h, 128, d, 3 * d, M, GEMM_EPI_STORE);
    GemmTcLaunch g = gemm_launch(pf, GEMM_EPI_STORE, d, 3 * d, M, &h->map_fc_fuse, nullptr, nullptr,
                                 &h->map_fsplit[bi], d, 0, 0, sv.err);
    g.args.out_bf16 = ge;
    g.args.ld_out = 2 * d;
    LK(SPEC_PROF_DRAFT_FC, 1, gemm_tc_launch(g, st, pdl));
    if (ts)
      LK(SPEC_PROF_TREE, 1,
         launch_tree_save_root(sp.B, d, 2 * d, ge, groot, h->W<int32_t>(L.p_tokens), ts->args, st, pdl));
  }
  // x = [g|e] . W_in^T (a residual GEMM on x = 0), xn = split(x * attn_norm), ss
  CUDA_RET(cudaMemsetAsync(h->ws + L.x, 0, 4 * (size_t)M * d, st));
  {
    const GemmPlan pf = plan_gemm(h, 128, d, 2 * d, M, GEMM_EPI_RESID);
    GemmMultiLaunch m{};
    m.bn = pf.bn;
    m.grid = pf.grid;
    m.err = sv.err;
    m.phase_bar = h->W<int>(L.phase_bar);
    m.n_phases = 1;
    m.ph[0] = pb.resid(pf, 2 * d, &h->map_fc_in, &h->map_ge[bi], h->layers[Ld].attn_norm, 0);
    LK(SPEC_PROF_DRAFT_FC, 1, gemm_multi_launch(m, st, false));
  }
  GemmMultiLaunch m{};
  m.bn = sp.qkv.bn;
  m.grid = sp.grid_all;
  m.err = sv.err;
  m.phase_bar = h->W<int>(L.phase_bar) + 4 * (c.n_layers + 1);
  m.n_phases = 1;
  m.ph[0] = pb.qkv(Ld, 4 + 1);
  LK(SPEC_PROF_GEMM_QKV, 1, gemm_multi_launch(m, st, pdl));
  if (kv_only) return cudaSuccess;

  AttnArgs aa{};
  aa.sv = sv;
  aa.kv = h->kv;
  aa.layer = Ld;
  aa.Hq = c.n_q_heads;
  aa.hd = c.head_dim;
  aa.q = h->ws + L.q;
  aa.out = h->ws + L.attn;
  aa.part_o = h->W<float>(L.part_o);
  aa.part_lse = h->W<float>(L.part_lse);
  aa.n_chunks = sp.n_chunks;
  aa.chunk = sp.chunk;
  aa.max_rows = sp.max_rows;
  aa.counters = h->W<int>(L.attn_ctr) + (size_t)Ld * 2 * kAttnPartCtas;  // the draft layer's own
  aa.q_rows = L.Mpad * (c.n_q_heads / c.n_kv_heads);
  aa.rescale_slack = h->rescale_slack;
  aa.cluster_merge = sp.cluster_merge;
  LK(SPEC_PROF_ATTENTION, 1, launch_attention_tc(aa, h->attn_maps, st, pdl));
  m.n_phases = 4;
  m.ph[0] = pb.o(Ld, 8 + 0);
  m.ph[1] = pb.gu(Ld, 8 + 1);
  m.ph[2] = pb.down(Ld, 8 + 2, h->draft_final_norm);
  // the LM head (over the reduced vocabulary when there is one) keeps, per row and
  // 128-row tile, the tile's k best and (max, sum of exp); the logits are never stored
  // (except into the debug buffer), and a small kernel merges the tiles
  const int Vd = c.draft_vocab ? c.draft_vocab : c.vocab;
  const int K = ts ? ts->K : kDraftTopK;
  const GemmPlan pl = c.draft_vocab ? plan_gemm(h, 128, Vd, d, M, GEMM_EPI_TOPK) : sp.lm;
  m.ph[3] = pb.lm_topk(dbg ? h->dbg_logits : nullptr, pl, c.draft_vocab ? &h->map_lm_draft : &h->map_lm, Vd, K, 8 + 3);
  LK(SPEC_PROF_GEMM_LAYER, 1, gemm_multi_launch(m, st, pdl));
  LK(SPEC_PROF_TOPK, 1,
     launch_topk_merge(M, pl.tiles_o, K, h->W<float>(L.cand_v), h->W<int32_t>(L.cand_i), h->W<float2>(L.cand_lse),
                       h->W<int32_t>(ts ? L.tr_top_i : L.dtop_i), h->W<float>(ts ? L.tr_top_v : L.dtop_v),
                       ts ? h->W<float>(L.tr_lse) : nullptr, st, pdl, h->draft_ids));
  return cudaSuccess;
}

// Batch entries by decreasing key count (cached length + tree nodes): attention
// takes its (sequence, kv head) work in this order, so that the longest
// sequences start first and the shortest fill the tail.  Only the speed depends
// on it; an approximate length (while device-output steps are in flight) is fine.
void key_order(const spec_handle* h, int B, const int32_t* seq_ids, const int32_t* node_off,
               const std::vector<int32_t>& len, int32_t* out) {
  (void)h;
  std::vector<std::pair<int, int>> keys((size_t)B);
  for (int b = 0; b < B; ++b) keys[b] = {-(len[seq_ids[b]] + node_off[b + 1] - node_off[b]), b};
  std::stable_sort(keys.begin(), keys.end());
  for (int b = 0; b < B; ++b) out[b] = keys[b].second;
}

// Validate a batch of trees on the host (before anything is queued).
int validate_batch(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens, const int32_t* parents,
                   const int32_t* node_off, int mode, int* M_out, int* max_n_out, int* max_lk_out) {
  const spec_config& c = h->cfg;
  if (B < 1 || B > c.max_batch) return fail(h, SPEC_ERR_CAPACITY, "batch %d outside [1, %d]", B, c.max_batch);
  if (!seq_ids || !tokens || !parents || !node_off) return fail(h, SPEC_ERR_ARG, "null input pointer");
  if (node_off[0] != 0) return fail(h, SPEC_ERR_ARG, "node_offsets[0] must be 0");
  std::vector<uint8_t> seen(c.max_batch, 0);
  int max_n = 0, max_lk = 0;
  for (int b = 0; b < B; ++b) {
    const int s = seq_ids[b];
    if (s < 0 || s >= c.max_batch) return fail(h, SPEC_ERR_ARG, "seq id %d outside [0, %d)", s, c.max_batch);
    if (seen[s]) return fail(h, SPEC_ERR_ARG, "seq id %d appears twice in one batch", s);
    seen[s] = 1;
    const int n = node_off[b + 1] - node_off[b];
    if (n < 1) return fail(h, SPEC_ERR_ARG, "tree %d is empty", b);
    if (n > c.max_nodes) return fail(h, SPEC_ERR_CAPACITY, "tree %d has %d nodes > max_nodes %d", b, n, c.max_nodes);
    if (mode != STEP_PREFILL && !h->ready[s]) return fail(h, SPEC_ERR_STATE, "sequence %d has not been prefilled", s);
    const int P = h->stale ? h->len_hi[s] : h->len[s];
    if (P + n > c.max_seq)
      return fail(h, SPEC_ERR_CAPACITY, "sequence %d: length %d + %d nodes exceeds max_seq %d", s, P, n, c.max_seq);
    const int32_t* tk = tokens + node_off[b];
    const int32_t* pr = parents + node_off[b];
    const int vr = spec_validate_tree(tk, pr, n, c.vocab, c.max_nodes);
    if (vr == SPEC_ERR_TREE) return fail(h, vr, "tree %d: parents[0] must be -1 and 0 <= parents[i] < i", b);
    if (vr == SPEC_ERR_TOKEN) return fail(h, vr, "tree %d: a token is outside [0, %d)", b, c.vocab);
    if (vr) return fail(h, vr, "tree %d rejected", b);
    if (mode == STEP_VERIFY && !h->stale && tk[0] != h->pending[s])
      return fail(h, SPEC_ERR_ROOT, "sequence %d: tokens[0] = %d is not the pending token %d", s, tk[0], h->pending[s]);
    max_n = std::max(max_n, n);
    max_lk = std::max(max_lk, P + n);
  }
  *M_out = node_off[B];
  *max_n_out = max_n;
  *max_lk_out = max_lk;
  return SPEC_OK;
}

// Upload parameters and run one step; with `sync`, wait and read the outputs.
int run_step(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens, const int32_t* parents,
             const int32_t* node_off, int mode, int flags, bool sync) {
  int M = 0, max_n = 0, max_lk = 0;
  int rc = validate_batch(h, B, seq_ids, tokens, parents, node_off, mode, &M, &max_n, &max_lk);
  if (rc) return rc;
  const WsLayout& L = h->lay;
  const bool dbg = (flags & SPEC_DEBUG_LOGITS) != 0;
  if (dbg && (!h->dbg_logits || h->dbg_bytes < sizeof(float) * (size_t)M * h->cfg.vocab))
    return fail(h, SPEC_ERR_CAPACITY, "SPEC_DEBUG_LOGITS needs a debug buffer of %zu bytes",
                sizeof(float) * (size_t)M * h->cfg.vocab);
  const bool feat = (flags & SPEC_FEATURES) != 0;
  if (feat) {
    if (mode != STEP_VERIFY && !(mode == STEP_PREFILL && h->pf_feat_out))
      return fail(h, SPEC_ERR_ARG, "SPEC_FEATURES applies to verification steps");
    if (h->cfg.feature_layers[0] < 1) return fail(h, SPEC_ERR_STATE, "the handle was created without feature layers");
    const size_t need = 2 * 3 * (size_t)B * h->cfg.max_nodes * h->cfg.hidden;
    if (mode == STEP_VERIFY && (!h->feat_out || h->feat_bytes < need))
      return fail(h, SPEC_ERR_CAPACITY, "SPEC_FEATURES needs a feature buffer of %zu bytes", need);
  }
  // pack the parameter block
  uint8_t* pb = h->h_params;
  std::memcpy(pb + L.p_tokens, tokens, 4 * (size_t)M);
  std::memcpy(pb + L.p_parents, parents, 4 * (size_t)M);
  std::memcpy(pb + L.p_node_off, node_off, 4 * (size_t)(B + 1));
  std::memcpy(pb + L.p_seq_ids, seq_ids, 4 * (size_t)B);
  key_order(h, B, seq_ids, node_off, h->stale ? h->len_hi : h->len, reinterpret_cast<int32_t*>(pb + L.p_order));
  std::memset(pb + L.p_err, 0, 16);
  CUDA_TRY(h, cudaMemcpyAsync(h->ws, pb, L.p_end, cudaMemcpyHostToDevice, h->stream));

  StepPlan sp = make_plan(h, B, M, max_n, max_lk);
  // the legacy default stream cannot be captured: launch directly there
  const bool graph = !(flags & SPEC_NO_GRAPH) && !h->prof && h->stream != nullptr;
  if (graph) {
    GraphKey key{mode, B, M, max_n, sp.n_chunks, sp.chunk, (dbg ? 1 : 0) | (feat ? 2 : 0), h->use_pdl ? 1 : 0};
    auto it = h->graphs.find(key);
    if (it == h->graphs.end()) {
      cudaGraph_t g = nullptr;
      CUDA_TRY(h, cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal));
      cudaError_t e = enqueue_step(h, sp, mode, dbg, feat);
      cudaError_t e2 = cudaStreamEndCapture(h->stream, &g);
      if (e != cudaSuccess || e2 != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        return fail(h, SPEC_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(e != cudaSuccess ? e : e2));
      }
      cudaGraphExec_t ex = nullptr;
      e = cudaGraphInstantiate(&ex, g, 0);
      cudaGraphDestroy(g);
      if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
      it = h->graphs.emplace(key, ex).first;
    }
    CUDA_TRY(h, cudaGraphLaunch(it->second, h->stream));
  } else {
    cudaError_t e = enqueue_step(h, sp, mode, dbg, feat);
    if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
  }

  if (!sync) {
    // device-output step: lengths are known only as upper bounds until spec_sync
    for (int b = 0; b < B; ++b) {
      const int s = seq_ids[b];
      const int n = node_off[b + 1] - node_off[b];
      const int base = h->stale ? h->len_hi[s] : h->len[s];
      if (mode == STEP_VERIFY) h->len_hi[s] = base + n;
      else if (mode == STEP_PREFILL) h->len_hi[s] = base + n;
      else h->len_hi[s] = base;
    }
    if (mode != STEP_SCORE) h->stale = true;
    return SPEC_OK;
  }
  CUDA_TRY(h, cudaMemcpyAsync(h->h_out, h->ws + L.o_acc_len, L.o_end - L.o_acc_len, cudaMemcpyDeviceToHost, h->stream));
  uint32_t errw[2] = {0, 0};
  CUDA_TRY(h, cudaMemcpyAsync(errw, h->ws + L.p_err, 4, cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  if (errw[0] & SPEC_DEVERR_TIMEOUT) return fail(h, SPEC_ERR_TIMEOUT, "a bounded wait expired on the device");
  if (errw[0] & SPEC_DEVERR_ROOT) return fail(h, SPEC_ERR_ROOT, "tokens[0] is not the pending token (device check)");
  if (errw[0] & SPEC_DEVERR_RANGE) return fail(h, SPEC_ERR_RANGE, "a q / K / V value exceeded the fp16 range");
  if (errw[0]) return fail(h, SPEC_ERR_CUDA, "device reported error bits 0x%x", errw[0]);
  // mirror the state update done on the device
  if (mode != STEP_SCORE) {
    const int32_t* acc_len = reinterpret_cast<const int32_t*>(h->h_out);
    const int32_t* bonus = reinterpret_cast<const int32_t*>(h->h_out + (L.o_bonus - L.o_acc_len));
    for (int b = 0; b < B; ++b) {
      const int s = seq_ids[b];
      h->len[s] += 1 + acc_len[b];
      h->len_hi[s] = h->len[s];
      h->pending[s] = bonus[b];
    }
  }
  return SPEC_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Run one draft-head step (or a draft prefill chunk) from host inputs; feats
// is a device pointer to bf16 [M][3][d].
int run_draft(spec_handle* h, int B, const int32_t* seq_ids, const void* feats, const int32_t* tokens,
              const int32_t* parents, const int32_t* node_off, bool kv_only, int flags, int32_t* top_idx,
              float* top_val) {
  const spec_config& c = h->cfg;
  const WsLayout& L = h->lay;
  if (!c.draft_head) return fail(h, SPEC_ERR_STATE, "the handle was created without the draft head");
  if (B < 1 || B > c.max_batch) return fail(h, SPEC_ERR_CAPACITY, "batch %d outside [1, %d]", B, c.max_batch);
  if (!seq_ids || !feats || !tokens || !parents || !node_off) return fail(h, SPEC_ERR_ARG, "null input pointer");
  if (!aligned16(feats)) return fail(h, SPEC_ERR_ARG, "feats must be 16-byte aligned");
  if (node_off[0] != 0) return fail(h, SPEC_ERR_ARG, "node_offsets[0] must be 0");
  std::vector<uint8_t> seen(c.max_batch, 0);
  int max_n = 0, max_lk = 0;
  for (int b = 0; b < B; ++b) {
    const int s = seq_ids[b];
    if (s < 0 || s >= c.max_batch) return fail(h, SPEC_ERR_ARG, "seq id %d outside [0, %d)", s, c.max_batch);
    if (seen[s]) return fail(h, SPEC_ERR_ARG, "seq id %d appears twice in one batch", s);
    seen[s] = 1;
    const int n = node_off[b + 1] - node_off[b];
    if (n < 1) return fail(h, SPEC_ERR_ARG, "tree %d is empty", b);
    if (n > c.max_nodes) return fail(h, SPEC_ERR_CAPACITY, "tree %d has %d nodes > max_nodes %d", b, n, c.max_nodes);
    if (!kv_only && !h->dready[s]) return fail(h, SPEC_ERR_STATE, "sequence %d has no draft prefix", s);
    if (h->dlen[s] + n > c.max_seq)
      return fail(h, SPEC_ERR_CAPACITY, "sequence %d: draft length %d + %d nodes exceeds max_seq %d", s, h->dlen[s], n,
                  c.max_seq);
    const int vr = spec_validate_tree(tokens + node_off[b], parents + node_off[b], n, c.vocab, c.max_nodes);
    if (vr == SPEC_ERR_TREE) return fail(h, vr, "tree %d: parents[0] must be -1 and 0 <= parents[i] < i", b);
    if (vr) return fail(h, vr, "tree %d rejected", b);
    max_n = std::max(max_n, n);
    max_lk = std::max(max_lk, h->dlen[s] + n);
  }
  const int M = node_off[B];
  const bool dbg = (flags & SPEC_DEBUG_LOGITS) != 0 && !kv_only;
  if (dbg && (!h->dbg_logits || h->dbg_bytes < sizeof(float) * (size_t)M * c.vocab))
    return fail(h, SPEC_ERR_CAPACITY, "SPEC_DEBUG_LOGITS needs a debug buffer of %zu bytes",
                sizeof(float) * (size_t)M * c.vocab);
  uint8_t* pb = h->h_params;
  std::memcpy(pb + L.p_tokens, tokens, 4 * (size_t)M);
  std::memcpy(pb + L.p_parents, parents, 4 * (size_t)M);
  std::memcpy(pb + L.p_node_off, node_off, 4 * (size_t)(B + 1));
  std::memcpy(pb + L.p_seq_ids, seq_ids, 4 * (size_t)B);
  std::memcpy(pb + L.p_dlen, h->dlen.data(), 4 * (size_t)c.max_batch);
  key_order(h, B, seq_ids, node_off, h->dlen, reinterpret_cast<int32_t*>(pb + L.p_order));
  std::memset(pb + L.p_err, 0, 16);
  CUDA_TRY(h, cudaMemcpyAsync(h->ws, pb, L.p_end, cudaMemcpyHostToDevice, h->stream));
  // the caller's features become the first GEMM's split operand (outside any graph:
  // the pointer may change from call to call)
  CUDA_TRY(h, launch_split_rows(static_cast<const __nv_bfloat16*>(feats), M, 3 * c.hidden,
                                h->W<__nv_bfloat16>(L.fsplit), h->stream, false));
  StepPlan sp = make_plan(h, B, M, max_n, max_lk);
  const int mode = kv_only ? STEP_DRAFT_KV : STEP_DRAFT;
  const bool graph = !(flags & SPEC_NO_GRAPH) && !h->prof && h->stream != nullptr;
  if (graph) {
    GraphKey key{mode, B, M, max_n, sp.n_chunks, sp.chunk, dbg ? 1 : 0, h->use_pdl ? 1 : 0};
    auto it = h->graphs.find(key);
    if (it == h->graphs.end()) {
      cudaGraph_t g = nullptr;
      CUDA_TRY(h, cudaStreamBeginCapture(h->stream, cudaStreamCaptureModeThreadLocal));
      cudaError_t e = enqueue_draft(h, sp, kv_only, dbg);
      cudaError_t e2 = cudaStreamEndCapture(h->stream, &g);
      if (e != cudaSuccess || e2 != cudaSuccess) {
        if (g) cudaGraphDestroy(g);
        return fail(h, SPEC_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(e != cudaSuccess ? e : e2));
      }
      cudaGraphExec_t ex = nullptr;
      e = cudaGraphInstantiate(&ex, g, 0);
      cudaGraphDestroy(g);
      if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
      it = h->graphs.emplace(key, ex).first;
    }
    CUDA_TRY(h, cudaGraphLaunch(it->second, h->stream));
  } else {
    cudaError_t e = enqueue_draft(h, sp, kv_only, dbg);
    if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
  }
  if (!kv_only && (flags & SPEC_DEVICE_OUTPUTS)) {
    if (top_idx)
      CUDA_TRY(h, cudaMemcpyAsync(top_idx, h->ws + L.dtop_i, 4 * (size_t)M * kDraftTopK, cudaMemcpyDeviceToDevice,
                                  h->stream));
    if (top_val)
      CUDA_TRY(h, cudaMemcpyAsync(top_val, h->ws + L.dtop_v, 4 * (size_t)M * kDraftTopK, cudaMemcpyDeviceToDevice,
                                  h->stream));
    return SPEC_OK;
  }
  if (!kv_only) {
    if (top_idx)
      CUDA_TRY(h, cudaMemcpyAsync(top_idx, h->ws + L.dtop_i, 4 * (size_t)M * kDraftTopK, cudaMemcpyDeviceToHost,
                                  h->stream));
    if (top_val)
      CUDA_TRY(h, cudaMemcpyAsync(top_val, h->ws + L.dtop_v, 4 * (size_t)M * kDraftTopK, cudaMemcpyDeviceToHost,
                                  h->stream));
  }
  uint32_t errw[2] = {0, 0};
  CUDA_TRY(h, cudaMemcpyAsync(errw, h->ws + L.p_err, 4, cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  if (errw[0] & SPEC_DEVERR_TIMEOUT) return fail(h, SPEC_ERR_TIMEOUT, "a bounded wait expired on the device");
  if (errw[0] & SPEC_DEVERR_RANGE) return fail(h, SPEC_ERR_RANGE, "a q / K / V value exceeded the fp16 range");
  if (errw[0]) return fail(h, SPEC_ERR_CUDA, "device reported error bits 0x%x", errw[0]);
  return SPEC_OK;
}

int refresh_state(spec_handle* h) {
  const WsLayout& L = h->lay;
  const int nb = h->cfg.max_batch;
  std::vector<int32_t> buf(2 * (size_t)nb);
  uint32_t sticky = 0;
  CUDA_TRY(h, cudaMemcpyAsync(buf.data(), h->ws + L.seq_len, 4 * (size_t)nb, cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaMemcpyAsync(buf.data() + nb, h->ws + L.pending, 4 * (size_t)nb, cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaMemcpyAsync(&sticky, h->ws + L.err_sticky, 4, cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaMemsetAsync(h->ws + L.err_sticky, 0, 4, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  for (int s = 0; s < nb; ++s) {
    h->len[s] = buf[s];
    h->len_hi[s] = buf[s];
    h->pending[s] = buf[nb + s];
  }
  h->stale = false;
  if (sticky & SPEC_DEVERR_TIMEOUT) return fail(h, SPEC_ERR_TIMEOUT, "a bounded wait expired on the device");
  if (sticky & SPEC_DEVERR_ROOT) return fail(h, SPEC_ERR_ROOT, "a queued step had tokens[0] != pending token");
  if (sticky & SPEC_DEVERR_RANGE) return fail(h, SPEC_ERR_RANGE, "a queued step exceeded the fp16 range of q / K / V");
  if (sticky) return fail(h, SPEC_ERR_CUDA, "device reported error bits 0x%x", sticky);
  return SPEC_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

int spec_validate_tree(const int32_t* tokens, const int32_t* parents, int n, int vocab, int max_nodes) {
  if (!tokens || !parents) return SPEC_ERR_ARG;
  if (n < 1 || n > max_nodes || max_nodes > kMaxNodesLimit) return SPEC_ERR_CAPACITY;
  if (parents[0] != -1) return SPEC_ERR_TREE;
  for (int i = 1; i < n; ++i)
    if (parents[i] < 0 || parents[i] >= i) return SPEC_ERR_TREE;
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= vocab) return SPEC_ERR_TOKEN;
  return SPEC_OK;
}

size_t spec_kv_bytes(const spec_config* cfg) {
  if (!check_config(cfg).empty()) return 0;
  return kv_bytes_of(*cfg);
}

size_t spec_workspace_bytes(const spec_config* cfg) {
  if (!check_config(cfg).empty()) return 0;
  return make_layout(*cfg).total;
}

int spec_init(const spec_config* cfg, const spec_weights* w, void* kv_cache, size_t kv_bytes, void* workspace,
              size_t ws_bytes, void* cuda_stream, spec_handle** out) {
  if (!out) return SPEC_ERR_ARG;
  *out = nullptr;
  std::string why = check_config(cfg);
  static std::string init_err;
  if (!why.empty()) return SPEC_ERR_ARG;
  if (!w || !w->embed || !w->final_norm || !w->lm_head || !w->layers || !kv_cache || !workspace) return SPEC_ERR_ARG;
  const spec_config& c = *cfg;
  if (kv_bytes < kv_bytes_of(c)) return SPEC_ERR_CAPACITY;
  WsLayout lay = make_layout(c);
  if (ws_bytes < lay.total) return SPEC_ERR_CAPACITY;
  if (!aligned16(kv_cache) || !aligned16(workspace) || !aligned16(w->embed) || !aligned16(w->lm_head) ||
      !aligned16(w->final_norm))
    return SPEC_ERR_ARG;
  for (int l = 0; l < cache_layers(c); ++l) {
    if (l == c.n_layers && !w->draft_layer) return SPEC_ERR_ARG;
    const spec_layer_weights& lw = l < c.n_layers ? w->layers[l] : *w->draft_layer;
    const void* ps[9] = {lw.wq, lw.wk, lw.wv, lw.wo, lw.w_gate, lw.w_up, lw.w_down, lw.attn_norm, lw.mlp_norm};
    for (const void* p : ps)
      if (!p || !aligned16(p)) return SPEC_ERR_ARG;
  }
  if (c.draft_head && (!w->draft_fc_fuse || !w->draft_fc_in || !w->draft_final_norm || !aligned16(w->draft_fc_fuse) ||
                       !aligned16(w->draft_fc_in) || !aligned16(w->draft_final_norm)))
    return SPEC_ERR_ARG;
  if (c.draft_vocab) {
    if (!w->draft_lm_head || !aligned16(w->draft_lm_head) || !w->draft_vocab_ids) return SPEC_ERR_ARG;
    // the token ids must be strictly increasing in [0, vocab): the top-k's tie order follows them
    std::vector<int32_t> ids((size_t)c.draft_vocab);
    if (cudaMemcpy(ids.data(), w->draft_vocab_ids, 4 * ids.size(), cudaMemcpyDeviceToHost) != cudaSuccess)
      return SPEC_ERR_CUDA;
    for (size_t i = 0; i < ids.size(); ++i)
      if (ids[i] < 0 || ids[i] >= c.vocab || (i && ids[i] <= ids[i - 1])) return SPEC_ERR_ARG;
  }

  spec_handle* h = new spec_handle();
  h->cfg = c;
  h->lay = lay;
  h->stream = reinterpret_cast<cudaStream_t>(cuda_stream);
  h->embed = w->embed;
  h->final_norm = w->final_norm;
  h->lm_head = w->lm_head;
  h->layers.assign(w->layers, w->layers + c.n_layers);
  if (c.draft_head) {
    h->layers.push_back(*w->draft_layer);
    h->draft_fc_fuse = w->draft_fc_fuse;
    h->draft_fc_in = w->draft_fc_in;
    h->draft_final_norm = w->draft_final_norm;
    if (c.draft_vocab) {
      h->draft_lm_head = w->draft_lm_head;
      h->draft_ids = w->draft_vocab_ids;
    }
  }
  h->dlen.assign(c.max_batch, 0);
  h->dready.assign(c.max_batch, 0);
  h->ws = reinterpret_cast<uint8_t*>(workspace);
  h->kv.base = kv_cache;
  h->kv.max_batch = c.max_batch;
  h->kv.Hkv = c.n_kv_heads;
  h->kv.max_seq = c.max_seq;
  h->kv.hd = c.head_dim;
  h->kv.elem = c.dtype == SPEC_DTYPE_BF16 ? 2 : 4;
  h->kv.planes = cache_planes(c);
  h->len.assign(c.max_batch, 0);
  h->pending.assign(c.max_batch, -1);
  h->len_hi.assign(c.max_batch, 0);
  h->ready.assign(c.max_batch, 0);

  auto bail = [&](int code, const char* msg) {
    spec_free(h);
    (void)msg;
    return code;
  };
  // Optional tuning knobs, e.g. SPEC_TUNE="splits=4,chunks=8,pdl=0,per_sm=1"
  if (const char* t = getenv("SPEC_TUNE")) {
    int v = 0;
    if (const char* q = strstr(t, "splits=")) if (sscanf(q + 7, "%d", &v) == 1 && v >= 1 && v <= kMaxSplits) h->max_splits = v;
    if (const char* q = strstr(t, "chunks=")) if (sscanf(q + 7, "%d", &v) == 1 && v >= 1 && v <= kMaxAttnChunks) h->max_chunks = v;
    if (const char* q = strstr(t, "pdl=")) if (sscanf(q + 4, "%d", &v) == 1) h->use_pdl = v != 0;
    if (const char* q = strstr(t, "dsmem=")) if (sscanf(q + 6, "%d", &v) == 1) h->attn_dsmem = v != 0;
    if (const char* q = strstr(t, "bn64max=")) if (sscanf(q + 8, "%d", &v) == 1 && v >= 64) h->bn64_max = v;
    if (const char* q = strstr(t, "bn96=")) if (sscanf(q + 5, "%d", &v) == 1) h->bn96 = v != 0;
    if (const char* q = strstr(t, "bn80=")) if (sscanf(q + 5, "%d", &v) == 1) h->bn80 = v != 0;
    if (const char* q = strstr(t, "per_sm=")) if (sscanf(q + 7, "%d", &v) == 1 && v >= 0) h->resident_cap = v;
    if (const char* q = strstr(t, "sk=")) if (sscanf(q + 3, "%d", &v) == 1 && v >= -1 && v <= 2) h->streamk = v;
    if (const char* q = strstr(t, "skh=")) if (sscanf(q + 4, "%d", &v) == 1) h->sk_hybrid = v != 0;
    float fv = 0.f;
    if (const char* q = strstr(t, "rescale=")) if (sscanf(q + 8, "%f", &fv) == 1 && fv >= 0.f && fv <= 15.f) h->rescale_slack = fv;
  }
  if (cudaGetDevice(&h->device) != cudaSuccess) return bail(SPEC_ERR_CUDA, "cudaGetDevice");
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, h->device) != cudaSuccess) return bail(SPEC_ERR_CUDA, "props");
  h->sm_count = prop.multiProcessorCount;
  if (cudaMallocHost(&h->h_params, lay.p_end) != cudaSuccess) return bail(SPEC_ERR_CUDA, "pinned");
  if (cudaMallocHost(&h->h_out, lay.o_end - lay.o_acc_len) != cudaSuccess) return bail(SPEC_ERR_CUDA, "pinned");

  // per-sequence state starts empty; rotary frequencies theta^(-2j/hd) in double
  std::vector<double> inv(c.head_dim / 2);
  for (int j = 0; j < c.head_dim / 2; ++j) inv[j] = std::pow((double)c.rope_theta, -2.0 * j / c.head_dim);
  if (cudaMemsetAsync(h->ws + lay.seq_len, 0, 4 * (size_t)c.max_batch, h->stream) != cudaSuccess ||
      cudaMemsetAsync(h->ws + lay.pending, 0xff, 4 * (size_t)c.max_batch, h->stream) != cudaSuccess ||
      cudaMemsetAsync(h->ws + lay.err_sticky, 0, 16, h->stream) != cudaSuccess ||
      cudaMemsetAsync(h->ws + lay.gemm_ctr, 0, 4 * (size_t)lay.gemm_ctr_n, h->stream) != cudaSuccess ||
      cudaMemsetAsync(h->ws + lay.attn_ctr, 0, 4 * (size_t)lay.attn_ctr_n, h->stream) != cudaSuccess ||

      cudaMemcpyAsync(h->ws + lay.inv_freq, inv.data(), 8 * inv.size(), cudaMemcpyHostToDevice, h->stream) !=
          cudaSuccess ||
      cudaStreamSynchronize(h->stream) != cudaSuccess)
    return bail(SPEC_ERR_CUDA, "state init");

  if (kv_compact_configure((size_t)(c.max_nodes - 1) * c.head_dim * h->kv.elem + 16) != cudaSuccess)
    return bail(SPEC_ERR_CUDA, "smem attribute");
  if (c.dtype == SPEC_DTYPE_BF16) {
    if (!get_encode_fn()) return bail(SPEC_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    if (attention_tc_configure(h->attn_clusters) != cudaSuccess) return bail(SPEC_ERR_CUDA, "smem attribute");
    const int qd = c.n_q_heads * c.head_dim, kvd = c.n_kv_heads * c.head_dim;
    {
      // q as [2 * Hkv * q_rows][128] (hi part, then lo part) and the cache as
      // [layers * planes * batch * Hkv * max_seq][128], fp16; TMA row coordinates are 32-bit
      const uint64_t cache_rows = (uint64_t)cache_layers(c) * cache_planes(c) * c.max_batch * c.n_kv_heads * c.max_seq;
      if (cache_rows + 128 >= (1ull << 31)) return bail(SPEC_ERR_CAPACITY, "cache too large for 32-bit rows");
      const uint64_t q_rows = (uint64_t)c.n_kv_heads * lay.Mpad * (c.n_q_heads / c.n_kv_heads);
      if (!make_tmap(&h->attn_maps.q, h->ws + lay.q, 2 * q_rows, 128, 128, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
          !make_tmap(&h->attn_maps.kv, kv_cache, cache_rows, 128, kAttnTcKeys, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
        return bail(SPEC_ERR_CUDA, "tensor map");
      // attention reads whole key blocks (P = 0 beyond a sequence's keys): every
      // slot must hold a finite value from the start, and q rows too
      if (cudaMemsetAsync(kv_cache, 0, kv_bytes_of(c), h->stream) != cudaSuccess ||
          cudaMemsetAsync(h->ws + lay.q, 0, 2 * 2 * (size_t)lay.Mpad * qd, h->stream) != cudaSuccess ||
          cudaStreamSynchronize(h->stream) != cudaSuccess)
        return bail(SPEC_ERR_CUDA, "cache init");
    }
    h->maps.resize(h->layers.size());
    for (int l = 0; l < (int)h->layers.size(); ++l) {
      const spec_layer_weights& lw = h->layers[l];
      LayerMaps& m = h->maps[l];
      bool ok = make_tmap(&m.wq, lw.wq, qd, c.hidden, 128) && make_tmap(&m.wk, lw.wk, kvd, c.hidden, 128) &&
                make_tmap(&m.wv, lw.wv, kvd, c.hidden, 128) && make_tmap(&m.wo, lw.wo, c.hidden, qd, 128) &&
                make_tmap(&m.wg, lw.w_gate, c.ffn, c.hidden, 64) && make_tmap(&m.wu, lw.w_up, c.ffn, c.hidden, 64) &&
                make_tmap(&m.wd, lw.w_down, c.hidden, c.ffn, 128);
      if (!ok) return bail(SPEC_ERR_CUDA, "tensor map");
    }
    if (!make_tmap(&h->map_lm, h->lm_head, c.vocab, c.hidden, 128)) return bail(SPEC_ERR_CUDA, "tensor map");
    if (c.draft_head &&
        (!make_tmap(&h->map_fc_fuse, h->draft_fc_fuse, c.hidden, 3 * (uint64_t)c.hidden, 128) ||
         !make_tmap(&h->map_fc_in, h->draft_fc_in, c.hidden, 2 * (uint64_t)c.hidden, 128)))
      return bail(SPEC_ERR_CUDA, "tensor map");
    if (c.draft_vocab && !make_tmap(&h->map_lm_draft, h->draft_lm_head, c.draft_vocab, c.hidden, 128))
      return bail(SPEC_ERR_CUDA, "tensor map");
    const int* bns = kTileWidths;
    for (int i = 0; i < kNumTileWidths; ++i) {
      // split activations: a tile of BN tokens is 2*BN rows (hi and lo)
      if (!make_tmap(&h->map_xn[i], h->ws + lay.xn, 2 * (uint64_t)lay.Mpad, c.hidden, 2 * bns[i]) ||
          !make_tmap(&h->map_attn[i], h->ws + lay.attn, 2 * (uint64_t)lay.Mpad, qd, 2 * bns[i]) ||
          !make_tmap(&h->map_h[i], h->ws + lay.hmlp, 2 * (uint64_t)lay.Mpad, c.ffn, 2 * bns[i]))
        return bail(SPEC_ERR_CUDA, "tensor map");
      if (c.draft_head &&
          (!make_tmap(&h->map_fsplit[i], h->ws + lay.fsplit, 2 * (uint64_t)lay.Mpad, 3 * (uint64_t)c.hidden,
                      2 * bns[i]) ||
           !make_tmap(&h->map_ge[i], h->ws + lay.ge, 2 * (uint64_t)lay.Mpad, 2 * (uint64_t)c.hidden, 2 * bns[i])))
        return bail(SPEC_ERR_CUDA, "tensor map");
    }
    for (int i = 0; i < kNumTileWidths; ++i)
      for (int e = 0; e < 4; ++e) {
        const void* fn = gemm_tc_function(bns[i]);
        const int smem = (int)gemm_tc_smem_bytes(bns[i]);
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared) != cudaSuccess)
          return bail(SPEC_ERR_CUDA, "smem attribute");
        int nb = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, 192, smem) != cudaSuccess || nb < 1)
          return bail(SPEC_ERR_CUDA, "occupancy");
        // shared memory per SM (1 KB per CTA is reserved by the system)
        const int by_smem = prop.sharedMemPerMultiprocessor / (smem + (int)prop.reservedSharedMemPerBlock);
        // registers: allocated per warp in units of 256 (8 per thread)
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) return bail(SPEC_ERR_CUDA, "function attributes");
        const int regs_cta = ((fa.numRegs + 7) / 8) * 8 * 192;
        const int by_regs = regs_cta > 0 ? prop.regsPerMultiprocessor / regs_cta : 1;
        h->occ_api[i][e] = nb;
        nb = std::min(std::max(nb, by_smem), by_regs);
        // tensor memory: two accumulators of 2*BN columns (hi and lo) per CTA, 512 columns per SM
        h->resident[i][e] = std::max(1, std::min(nb, 512 / (4 * bns[i])));
      }
  }
  *out = h;
  return SPEC_OK;
}

static int prefill_impl(spec_handle* h, int seq, const int32_t* tokens, int n, int32_t* pending_token,
                        void* feats_out) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  const spec_config& c = h->cfg;
  if (feats_out && c.feature_layers[0] < 1)
    return fail(h, SPEC_ERR_STATE, "the handle was created without feature layers");
  if (feats_out && !aligned16(feats_out)) return fail(h, SPEC_ERR_ARG, "feats_out must be 16-byte aligned");
  if (!tokens || n < 1) return fail(h, SPEC_ERR_ARG, "prefill needs n >= 1 tokens");
  if (seq < 0 || seq >= c.max_batch) return fail(h, SPEC_ERR_ARG, "seq %d outside [0, %d)", seq, c.max_batch);
  if (n > c.max_seq) return fail(h, SPEC_ERR_CAPACITY, "prompt of %d tokens exceeds max_seq %d", n, c.max_seq);
  for (int i = 0; i < n; ++i)
    if (tokens[i] < 0 || tokens[i] >= c.vocab) return fail(h, SPEC_ERR_TOKEN, "token %d outside [0, %d)", tokens[i], c.vocab);
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  // reset the sequence
  const int zero = 0;
  CUDA_TRY(h, cudaMemcpyAsync(h->ws + h->lay.seq_len + 4 * (size_t)seq, &zero, 4, cudaMemcpyHostToDevice, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  h->len[seq] = 0;
  h->len_hi[seq] = 0;
  h->ready[seq] = 0;
  std::vector<int32_t> parents(c.max_nodes);
  for (int i = 0; i < c.max_nodes; ++i) parents[i] = i - 1;
  const int32_t ids[1] = {seq};
  for (int s0 = 0; s0 < n; s0 += c.max_nodes) {
    const int m = std::min(c.max_nodes, n - s0);
    const int32_t off[2] = {0, m};
    // with features: this chunk's rows go to feats_out at its offset (no graph: the
    // destination changes from chunk to chunk)
    h->pf_feat_out = feats_out ? static_cast<uint8_t*>(feats_out) + (size_t)s0 * 3 * c.hidden * 2 : nullptr;
    int rc = run_step(h, 1, ids, tokens + s0, parents.data(), off, STEP_PREFILL,
                      feats_out ? (SPEC_FEATURES | SPEC_NO_GRAPH) : 0, true);
    h->pf_feat_out = nullptr;
    if (rc) return rc;
  }
  h->ready[seq] = 1;
  if (pending_token) *pending_token = h->pending[seq];
  return SPEC_OK;
}

int spec_prefill(spec_handle* h, int seq, const int32_t* tokens, int n, int32_t* pending_token) {
  return prefill_impl(h, seq, tokens, n, pending_token, nullptr);
}

int spec_prefill_features(spec_handle* h, int seq, const int32_t* tokens, int n, int32_t* pending_token,
                          void* feats_out) {
  if (!feats_out) return h ? fail(h, SPEC_ERR_ARG, "feats_out is NULL") : SPEC_ERR_ARG;
  return prefill_impl(h, seq, tokens, n, pending_token, feats_out);
}

int spec_verify_tree_batch(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens,
                           const int32_t* parents, const int32_t* node_offsets, int32_t* accepted_len,
                           int32_t* accepted_nodes, int32_t* accepted_tokens, int32_t* bonus, int flags) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  const bool dev = (flags & SPEC_DEVICE_OUTPUTS) != 0;
  int rc = run_step(h, B, seq_ids, tokens, parents, node_offsets, STEP_VERIFY, flags, !dev);
  if (rc) return rc;
  const WsLayout& L = h->lay;
  const size_t nn = (size_t)B * h->cfg.max_nodes;
  if (dev) {
    if (accepted_len)
      CUDA_TRY(h, cudaMemcpyAsync(accepted_len, h->ws + L.o_acc_len, 4 * (size_t)B, cudaMemcpyDeviceToDevice, h->stream));
    if (accepted_nodes)
      CUDA_TRY(h, cudaMemcpyAsync(accepted_nodes, h->ws + L.o_acc_nodes, 4 * nn, cudaMemcpyDeviceToDevice, h->stream));
    if (accepted_tokens)
      CUDA_TRY(h, cudaMemcpyAsync(accepted_tokens, h->ws + L.o_acc_tokens, 4 * nn, cudaMemcpyDeviceToDevice, h->stream));
    if (bonus) CUDA_TRY(h, cudaMemcpyAsync(bonus, h->ws + L.o_bonus, 4 * (size_t)B, cudaMemcpyDeviceToDevice, h->stream));
    return SPEC_OK;
  }
  const uint8_t* ho = h->h_out;
  if (accepted_len) std::memcpy(accepted_len, ho + (L.o_acc_len - L.o_acc_len), 4 * (size_t)B);
  if (accepted_nodes) std::memcpy(accepted_nodes, ho + (L.o_acc_nodes - L.o_acc_len), 4 * nn);
  if (accepted_tokens) std::memcpy(accepted_tokens, ho + (L.o_acc_tokens - L.o_acc_len), 4 * nn);
  if (bonus) std::memcpy(bonus, ho + (L.o_bonus - L.o_acc_len), 4 * (size_t)B);
  return SPEC_OK;
}

int spec_verify_tree(spec_handle* h, int seq, const int32_t* tokens, const int32_t* parents, int n_nodes,
                     int32_t* accepted_len, int32_t* accepted_tokens, int32_t* bonus_token) {
  if (!h) return SPEC_ERR_ARG;
  if (n_nodes < 1) return fail(h, SPEC_ERR_ARG, "n_nodes must be >= 1");
  if (n_nodes > h->cfg.max_nodes)
    return fail(h, SPEC_ERR_CAPACITY, "%d nodes > max_nodes %d", n_nodes, h->cfg.max_nodes);
  const int32_t ids[1] = {seq};
  const int32_t off[2] = {0, n_nodes};
  int32_t len = 0, bon = 0;
  std::vector<int32_t> toks(h->cfg.max_nodes);
  int rc = spec_verify_tree_batch(h, 1, ids, tokens, parents, off, &len, nullptr, toks.data(), &bon, 0);
  if (rc) return rc;
  if (accepted_len) *accepted_len = len;
  if (accepted_tokens) std::memcpy(accepted_tokens, toks.data(), 4 * (size_t)std::max(0, len));
  if (bonus_token) *bonus_token = bon;
  return SPEC_OK;
}

int spec_score_trees(spec_handle* h, int B, const int32_t* seq_ids, const int32_t* tokens, const int32_t* parents,
                     const int32_t* node_offsets, int32_t* argmax, float* top1, float* top2, int flags) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  int rc = run_step(h, B, seq_ids, tokens, parents, node_offsets, STEP_SCORE, flags & ~SPEC_DEVICE_OUTPUTS, true);
  if (rc) return rc;
  const int M = node_offsets[B];
  const WsLayout& L = h->lay;
  if (argmax) CUDA_TRY(h, cudaMemcpy(argmax, h->ws + L.argmax, 4 * (size_t)M, cudaMemcpyDeviceToHost));
  if (top1) CUDA_TRY(h, cudaMemcpy(top1, h->ws + L.top1, 4 * (size_t)M, cudaMemcpyDeviceToHost));
  if (top2) CUDA_TRY(h, cudaMemcpy(top2, h->ws + L.top2, 4 * (size_t)M, cudaMemcpyDeviceToHost));
  return SPEC_OK;
}

static int draft_rows_impl(spec_handle* h, int seq, const void* feats, const int32_t* tokens, int n, bool reset) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  const spec_config& c = h->cfg;
  if (!c.draft_head) return fail(h, SPEC_ERR_STATE, "the handle was created without the draft head");
  if (!feats || !tokens || n < 1) return fail(h, SPEC_ERR_ARG, "draft prefill needs n >= 1 rows");
  if (seq < 0 || seq >= c.max_batch) return fail(h, SPEC_ERR_ARG, "seq %d outside [0, %d)", seq, c.max_batch);
  const int start = reset ? 0 : h->dlen[seq];
  if (!reset && !h->dready[seq]) return fail(h, SPEC_ERR_STATE, "sequence %d has no draft prefix", seq);
  if (start + n > c.max_seq)
    return fail(h, SPEC_ERR_CAPACITY, "draft prefix of %d rows exceeds max_seq %d", start + n, c.max_seq);
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  // chunks of max_nodes rows as chains: each row's K/V at its own position, after the rows before it
  h->dlen[seq] = start;
  h->dready[seq] = 0;
  const size_t row_bytes = 2 * 3 * (size_t)c.hidden;
  std::vector<int32_t> par(c.max_nodes);
  for (int i = 0; i < c.max_nodes; ++i) par[i] = i - 1;
  for (int i0 = 0; i0 < n; i0 += c.max_nodes) {
    const int m = std::min(c.max_nodes, n - i0);
    const int32_t off[2] = {0, m};
    const int rc = run_draft(h, 1, &seq, static_cast<const uint8_t*>(feats) + (size_t)i0 * row_bytes, tokens + i0,
                             par.data(), off, true, 0, nullptr, nullptr);
    if (rc) return rc;
    h->dlen[seq] += m;
  }
  h->dready[seq] = 1;
  return SPEC_OK;
}

int spec_draft_prefill(spec_handle* h, int seq, const void* feats, const int32_t* tokens, int n) {
  return draft_rows_impl(h, seq, feats, tokens, n, true);
}

int spec_draft_append(spec_handle* h, int seq, const void* feats, const int32_t* tokens, int n) {
  return draft_rows_impl(h, seq, feats, tokens, n, false);
}

int spec_draft_step(spec_handle* h, int B, const int32_t* seq_ids, const void* feats, const int32_t* tokens,
                    const int32_t* parents, const int32_t* node_offsets, int32_t* top_idx, float* top_val,
                    int flags) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  return run_draft(h, B, seq_ids, feats, tokens, parents, node_offsets, false, flags, top_idx, top_val);
}

int spec_draft_tree(spec_handle* h, int B, const int32_t* seq_ids, const void* root_feats, const int32_t* root_tokens,
                    int steps, int topk, int total, int32_t* out_tokens, int32_t* out_parents, float* out_values) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  const spec_config& c = h->cfg;
  const WsLayout& L = h->lay;
  cudaStream_t st = h->stream;
  if (!c.draft_head) return fail(h, SPEC_ERR_STATE, "the handle was created without the draft head");
  if (B < 1 || B > c.max_batch) return fail(h, SPEC_ERR_CAPACITY, "batch %d outside [1, %d]", B, c.max_batch);
  if (!seq_ids || !root_feats || !root_tokens || !out_tokens || !out_parents)
    return fail(h, SPEC_ERR_ARG, "null pointer");
  if (!aligned16(root_feats)) return fail(h, SPEC_ERR_ARG, "root_feats must be 16-byte aligned");
  if (topk != 4 && topk != 8 && topk != 10 && topk != 16) return fail(h, SPEC_ERR_ARG, "topk must be 4, 8, 10 or 16");
  if (steps < 1 || total < 1) return fail(h, SPEC_ERR_ARG, "steps and total must be positive");
  const int n_last = 1 + (steps - 1) * topk;       // rows per tree in the last step
  const int joined = 1 + steps * topk;             // nodes joined over all steps
  const int n_offers = topk + (steps - 1) * topk * topk;
  if (n_last > c.max_nodes || joined > kTreeMaxNodes || n_offers > kTreeMaxOffers)
    return fail(h, SPEC_ERR_CAPACITY, "%d steps of top-%d exceed the tree limits (max_nodes %d)", steps, topk,
                c.max_nodes);
  if (total > n_offers || total + 1 > c.max_nodes)
    return fail(h, SPEC_ERR_CAPACITY, "total %d exceeds the offers (%d) or max_nodes - 1", total, n_offers);
  std::vector<uint8_t> seen(c.max_batch, 0);
  int max_dlen = 0;
  for (int b = 0; b < B; ++b) {
    const int s = seq_ids[b];
    if (s < 0 || s >= c.max_batch) return fail(h, SPEC_ERR_ARG, "seq id %d outside [0, %d)", s, c.max_batch);
    if (seen[s]) return fail(h, SPEC_ERR_ARG, "seq id %d appears twice in one batch", s);
    seen[s] = 1;
    if (!h->dready[s]) return fail(h, SPEC_ERR_STATE, "sequence %d has no draft prefix", s);
    if (h->dlen[s] + n_last > c.max_seq)
      return fail(h, SPEC_ERR_CAPACITY, "sequence %d: draft length %d + %d nodes exceeds max_seq %d", s, h->dlen[s],
                  n_last, c.max_seq);
    if (root_tokens[b] < 0 || root_tokens[b] >= c.vocab) return fail(h, SPEC_ERR_TOKEN, "root token outside [0, vocab)");
    max_dlen = std::max(max_dlen, h->dlen[s]);
  }
  TreeArgs ta{};
  ta.K = topk;
  ta.max_nodes = kTreeMaxNodes;
  ta.tok = h->W<int32_t>(L.tr_tok);
  ta.par = h->W<int32_t>(L.tr_par);
  ta.val = h->W<float>(L.tr_val);
  ta.offers = h->W<TreeOffer>(L.tr_offers);
  ta.n_offers = h->W<int32_t>(L.tr_noff);
  // the parameter block is uploaded once: each expansion writes the next step's
  // trees and node offsets on the device, so the steps queue back to back
  {
    uint8_t* pb = h->h_params;
    int32_t* tk = reinterpret_cast<int32_t*>(pb + L.p_tokens);
    int32_t* pr = reinterpret_cast<int32_t*>(pb + L.p_parents);
    int32_t* no = reinterpret_cast<int32_t*>(pb + L.p_node_off);
    for (int b = 0; b < B; ++b) {
      tk[b] = root_tokens[b];
      pr[b] = -1;
    }
    for (int b = 0; b <= B; ++b) no[b] = b;
    std::memcpy(pb + L.p_seq_ids, seq_ids, 4 * (size_t)B);
    std::memcpy(pb + L.p_dlen, h->dlen.data(), 4 * (size_t)c.max_batch);
    // every tree has the same node count at every step: the draft prefixes decide the order
    key_order(h, B, seq_ids, no, h->dlen, reinterpret_cast<int32_t*>(pb + L.p_order));
    std::memset(pb + L.p_err, 0, 16);
    CUDA_TRY(h, cudaMemcpyAsync(h->ws, pb, L.p_end, cudaMemcpyHostToDevice, st));
    CUDA_TRY(h, launch_split_rows(static_cast<const __nv_bfloat16*>(root_feats), B, 3 * c.hidden,
                                  h->W<__nv_bfloat16>(L.fsplit), st, false));
  }
  for (int t = 0; t < steps; ++t) {
    const int n = 1 + t * topk, M = B * n;
    const StepPlan sp = make_plan(h, B, M, n, max_dlen + n);
    TreeStep ts{t, n, t ? 1 + (t - 1) * topk : 0, topk, ta};
    ts.args.write_next = t + 1 < steps ? 1 : 0;
    cudaError_t e = enqueue_draft(h, sp, false, false, &ts);
    if (e == cudaSuccess)
      e = launch_k(h, SPEC_PROF_TREE, 1, [&]() {
        return launch_tree_expand(ts.args, B, t, n, t == 0 ? 1 : topk, h->W<int32_t>(L.tr_top_i),
                                  h->W<float>(L.tr_top_v), h->W<float>(L.tr_lse), h->W<int32_t>(L.p_tokens),
                                  h->W<int32_t>(L.p_parents), h->W<int32_t>(L.p_node_off), st, false);
      });
    if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
  }
  const size_t no_ = (size_t)B * (total + 1);
  cudaError_t e = launch_k(h, SPEC_PROF_TREE, 1, [&]() {
    return launch_tree_rerank(ta, B, total, h->W<int32_t>(L.tr_out_tok), h->W<int32_t>(L.tr_out_par),
                              h->W<float>(L.tr_out_val), st, false);
  });
  if (e != cudaSuccess) return fail(h, SPEC_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
  CUDA_TRY(h, cudaMemcpyAsync(out_tokens, h->ws + L.tr_out_tok, 4 * no_, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(h, cudaMemcpyAsync(out_parents, h->ws + L.tr_out_par, 4 * no_, cudaMemcpyDeviceToHost, st));
  if (out_values) CUDA_TRY(h, cudaMemcpyAsync(out_values, h->ws + L.tr_out_val, 4 * no_, cudaMemcpyDeviceToHost, st));
  uint32_t errw[2] = {0, 0};
  CUDA_TRY(h, cudaMemcpyAsync(errw, h->ws + L.p_err, 4, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(h, cudaStreamSynchronize(st));
  if (errw[0] & SPEC_DEVERR_TIMEOUT) return fail(h, SPEC_ERR_TIMEOUT, "a bounded wait expired on the device");
  if (errw[0] & SPEC_DEVERR_RANGE) return fail(h, SPEC_ERR_RANGE, "a q / K / V value exceeded the fp16 range");
  if (errw[0]) return fail(h, SPEC_ERR_CUDA, "device reported error bits 0x%x", errw[0]);
  for (int b = 0; b < B; ++b)
    if (spec_validate_tree(out_tokens + (size_t)b * (total + 1), out_parents + (size_t)b * (total + 1), total + 1,
                           c.vocab, c.max_nodes) != SPEC_OK)
      return fail(h, SPEC_ERR_CUDA, "tree %d came out malformed", b);
  return SPEC_OK;
}

int spec_draft_len(spec_handle* h, int seq, int32_t* len) {
  if (!h || !len) return SPEC_ERR_ARG;
  if (seq < 0 || seq >= h->cfg.max_batch) return fail(h, SPEC_ERR_ARG, "seq %d outside [0, %d)", seq, h->cfg.max_batch);
  *len = h->dlen[seq];
  return SPEC_OK;
}

int spec_set_feature_out(spec_handle* h, void* device_buf, size_t bytes) {
  if (!h) return SPEC_ERR_ARG;
  if (h->cfg.feature_layers[0] < 1) return fail(h, SPEC_ERR_STATE, "the handle was created without feature layers");
  if (device_buf && !aligned16(device_buf)) return fail(h, SPEC_ERR_ARG, "the feature buffer must be 16-byte aligned");
  h->feat_out = device_buf;
  h->feat_bytes = device_buf ? bytes : 0;
  // graphs bake the pointer in
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  h->graphs.clear();
  return SPEC_OK;
}

int spec_set_sampling(spec_handle* h, float temperature, uint64_t seed) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  if (!(temperature >= 0.f) || !std::isfinite(temperature))
    return fail(h, SPEC_ERR_ARG, "temperature %g must be finite and >= 0", (double)temperature);
  if (temperature > 0.f && !std::isfinite(1.f / temperature))
    return fail(h, SPEC_ERR_ARG, "temperature %g is too small (1/T overflows)", (double)temperature);
  h->temperature = temperature;
  h->seed = seed;
  // graphs bake the launch arguments in
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  h->graphs.clear();
  return SPEC_OK;
}

int spec_set_debug_logits(spec_handle* h, float* device_buf, size_t bytes) {
  if (!h) return SPEC_ERR_ARG;
  h->dbg_logits = device_buf;
  h->dbg_bytes = device_buf ? bytes : 0;
  // graphs bake the pointer in
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  h->graphs.clear();
  return SPEC_OK;
}

int spec_truncate(spec_handle* h, int seq, int new_len) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  if (seq < 0 || seq >= h->cfg.max_batch) return fail(h, SPEC_ERR_ARG, "seq %d outside [0, %d)", seq, h->cfg.max_batch);
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  if (!h->ready[seq]) return fail(h, SPEC_ERR_STATE, "sequence %d has not been prefilled", seq);
  if (new_len == h->len[seq]) return SPEC_OK;
  if (new_len < 1 || new_len > h->len[seq])
    return fail(h, SPEC_ERR_STATE, "cannot truncate sequence %d from %d to %d", seq, h->len[seq], new_len);
  int32_t tok = 0;
  CUDA_TRY(h, cudaMemcpyAsync(&tok, h->ws + h->lay.hist + 4 * ((size_t)seq * h->cfg.max_seq + new_len), 4,
                              cudaMemcpyDeviceToHost, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  const int32_t vals[1] = {new_len};
  CUDA_TRY(h, cudaMemcpyAsync(h->ws + h->lay.seq_len + 4 * (size_t)seq, vals, 4, cudaMemcpyHostToDevice, h->stream));
  CUDA_TRY(h, cudaMemcpyAsync(h->ws + h->lay.pending + 4 * (size_t)seq, &tok, 4, cudaMemcpyHostToDevice, h->stream));
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  h->len[seq] = new_len;
  h->len_hi[seq] = new_len;
  h->pending[seq] = tok;
  return SPEC_OK;
}

int spec_seq_len(spec_handle* h, int seq, int32_t* len, int32_t* pending) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  if (seq < 0 || seq >= h->cfg.max_batch) return fail(h, SPEC_ERR_ARG, "seq %d outside [0, %d)", seq, h->cfg.max_batch);
  if (h->stale) {
    int rc = refresh_state(h);
    if (rc) return rc;
  }
  if (len) *len = h->len[seq];
  if (pending) *pending = h->pending[seq];
  return SPEC_OK;
}

int spec_sync(spec_handle* h) {
  if (!h) return SPEC_ERR_ARG;
  h->err.clear();
  return refresh_state(h);
}

int spec_profile(spec_handle* h, int enable) {
  if (!h) return SPEC_ERR_ARG;
  h->prof = enable != 0;
  h->prof_marks.clear();
  return SPEC_OK;
}

int spec_profile_read(spec_handle* h, double* ms, int64_t* launches) {
  if (!h) return SPEC_ERR_ARG;
  CUDA_TRY(h, cudaStreamSynchronize(h->stream));
  for (const auto& m : h->prof_marks) {
    float t = 0.f;
    CUDA_TRY(h, cudaEventElapsedTime(&t, h->ev_pool[m.second], h->ev_pool[m.second + 1]));
    if (ms) ms[m.first] += t;
    if (launches) launches[m.first] += 1;
  }
  h->prof_marks.clear();
  return SPEC_OK;
}

int spec_step_launches(spec_handle* h) { return h ? h->launches : 0; }

// GEMM marks [2 * SMs][phases][16], then attention marks [2 layers][kAttnPartCtas][16]
static size_t trace_words(const spec_handle* h) {
  return (size_t)2 * h->sm_count * kMaxGemmPhases * kGemmTraceMarks + (size_t)2 * kAttnPartCtas * 16;
}

int spec_set_trace(spec_handle* h, uint64_t* device_buf, size_t bytes, int layer) {
  if (!h) return SPEC_ERR_ARG;
  if (device_buf && bytes < trace_words(h) * sizeof(uint64_t))
    return fail(h, SPEC_ERR_CAPACITY, "trace buffer too small");
  h->trace = device_buf;
  h->trace_bytes = bytes;
  h->trace_layer = layer;
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);  // graphs bake the pointer in
  h->graphs.clear();
  return SPEC_OK;
}

int spec_info(spec_handle* h, int B, int n_nodes, int prefix, char* buf, size_t n) {
  if (!h || !buf || n == 0) return SPEC_ERR_ARG;
  const StepPlan sp = make_plan(h, B, B * n_nodes, n_nodes, prefix + n_nodes);
  auto g = [](const GemmPlan& p) {
    char t[96];
    snprintf(t, sizeof(t), "bn%d tiles%dx%d splits%d kb/split%d grid%d%s", p.bn, p.tiles_o, p.tiles_t, p.splits,
             p.kbps, p.grid, p.sk ? " stream-K" : "");
    return std::string(t);
  };
  std::string s = "sms " + std::to_string(h->sm_count) + "; attention clusters held [size:count]";
  for (int cs = 2; cs <= kAttnMaxChunks; ++cs) s += " " + std::to_string(cs) + ":" + std::to_string(h->attn_clusters[cs]);
  s += "; resident/SM [bn64|bn128|bn96|bn80][qkv,swiglu,argmax,resid] = ";
  for (int i = 0; i < kNumTileWidths; ++i)
    for (int e = 0; e < 4; ++e)
      s += std::to_string(h->resident[i][e]) + "(" + std::to_string(h->occ_api[i][e]) + ")" + (e < 3 ? "," : "|");
  s += "; qkv " + g(sp.qkv) + "; o " + g(sp.o) + "; gate_up " + g(sp.gu) + "; down " + g(sp.down) + "; lm " +
       g(sp.lm) + "; attention chunks " + std::to_string(sp.n_chunks) + " x " + std::to_string(sp.chunk) +
        (sp.cluster_merge ? " (cluster merge)" : " (global merge)");
  snprintf(buf, n, "%s", s.c_str());
  return SPEC_OK;
}

int spec_io_bytes(spec_handle* h, size_t* h2d, size_t* d2h) {
  if (!h) return SPEC_ERR_ARG;
  if (h2d) *h2d = h->lay.p_end;
  if (d2h) *d2h = (h->lay.o_end - h->lay.o_acc_len) + 4;
  return SPEC_OK;
}

const char* spec_last_error(spec_handle* h) { return h ? h->err.c_str() : "null handle"; }

void spec_free(spec_handle* h) {
  if (!h) return;
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  if (h->h_params) cudaFreeHost(h->h_params);
  if (h->h_out) cudaFreeHost(h->h_out);
  delete h;
}

}  // extern "C"
