// Dynamic draft tree of the EAGLE-3 draft head: multi-step drafting shaped by
// the draft's own confidence.
//
// The pages ("EAGLE-3: Scaling up Inference Acceleration of Large Language
// Models via Training-Time Test", draft-stage description, and its overview of
// EAGLE-2): the draft model's confidence stands in for the acceptance rate and
// shapes the tree; from the second drafting step on, the draft's own output a
// replaces the target feature.  Reading where the pages leave steps open: a
// node's value is the sum of log-probabilities (full-vocabulary softmax of the
// draft logits at its parent) along its root path; every step runs the draft
// head over the tree built so far; the nodes that joined last offer their
// top-k tokens; the k best offers join; after the last step the `total` best
// offers, joined or not, form the tree (ties: lower depth, then earlier offer).
//
// Kernels here: the feature rows of a step (root: the fused target feature
// saved at step 0; other nodes: the parent's draft output from the previous
// step), the expansion (offers, selection, the next step's tree written into
// the device parameter block) and the final rerank.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace spec {

// ---------------------------------------------------------------------------
// feature rows
// ---------------------------------------------------------------------------

// Root rows of step 0: keep their fused feature (split bf16 hi and lo rows of
// the [g|e] operand, columns [0, d)) for the later steps, and start tree b's
// state with its root token (row b of step 0's parameter block).
__global__ void tree_save_root_kernel(int d, int ld, const __nv_bfloat16* __restrict__ ge,
                                      __nv_bfloat16* __restrict__ groot, const int32_t* __restrict__ tokens,
                                      TreeArgs a) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;  // step 0: row b is the root of tree b
  if (threadIdx.x == 0) {
    a.tok[(size_t)b * a.max_nodes] = tokens[b];
    a.par[(size_t)b * a.max_nodes] = -1;
    a.val[(size_t)b * a.max_nodes] = 0.f;
    a.n_offers[b] = 0;
  }
  for (int part = 0; part < 2; ++part) {
    const uint4* src = reinterpret_cast<const uint4*>(ge + (size_t)split_row(b, part) * ld);
    uint4* dst = reinterpret_cast<uint4*>(groot + ((size_t)b * 2 + part) * d);
    for (int i = threadIdx.x; i < d / 8; i += blockDim.x) dst[i] = src[i];
  }
}

// Row r = tree b's node i (uniform trees of n nodes): the feature half of its
// [g|e] row is the root's saved feature (i = 0) or split(a) of its parent, a
// being row b * n_prev + parent of the previous step's draft-layer output x.
__global__ void tree_feature_rows_kernel(int d, int ld, int n, int n_prev, const int32_t* __restrict__ parents,
                                         const __nv_bfloat16* __restrict__ groot, const float* __restrict__ x_prev,
                                         __nv_bfloat16* __restrict__ ge) {
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  const int b = r / n, i = r % n;
  if (i == 0) {
    for (int part = 0; part < 2; ++part) {
      const uint4* src = reinterpret_cast<const uint4*>(groot + ((size_t)b * 2 + part) * d);
      uint4* dst = reinterpret_cast<uint4*>(ge + (size_t)split_row(r, part) * ld);
      for (int c = threadIdx.x; c < d / 8; c += blockDim.x) dst[c] = src[c];
    }
    return;
  }
  const int p = parents[r];
  if ((unsigned)p >= (unsigned)n_prev) return;  // every parent is a node of the previous step's tree
  const float* a = x_prev + ((size_t)b * n_prev + p) * d;
  for (int c = 4 * threadIdx.x; c < d; c += 4 * blockDim.x)
    split_store4(ge, r, ld, c, *reinterpret_cast<const float4*>(a + c));
}

cudaError_t launch_tree_save_root(int B, int d, int ld, const __nv_bfloat16* ge, __nv_bfloat16* groot,
                                  const int32_t* tokens, const TreeArgs& a, cudaStream_t s, bool pdl) {
  if (d % 8) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(B), dim3(128), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, tree_save_root_kernel, d, ld, ge, groot, tokens, a);
}

cudaError_t launch_tree_feature_rows(int M, int d, int ld, int n, int n_prev, const int32_t* parents,
                                     const __nv_bfloat16* groot, const float* x_prev, __nv_bfloat16* ge,
                                     cudaStream_t s, bool pdl) {
  if (d % 8 || n < 1 || M % n) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(M), dim3(128), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, tree_feature_rows_kernel, d, ld, n, n_prev, parents, groot, x_prev, ge);
}

// ---------------------------------------------------------------------------
// expansion
// ---------------------------------------------------------------------------

__device__ __forceinline__ bool offer_before(float va, int oa, float vb, int ob) {
  return va > vb || (va == vb && oa < ob);
}

// One CTA per tree.  Step t: tree b has n nodes (rows b * n .. b * n + n - 1 of
// this step); the nodes n - nf .. n - 1 joined last and offer their K best
// tokens; the K best offers join as nodes n .. n + K - 1; the next step's trees
// (n + K nodes each) go to the parameter block: tokens and parents at rows
// b * (n + K), node offsets b * (n + K).
__global__ void tree_expand_kernel(TreeArgs a, int t, int n, int nf, const int32_t* __restrict__ top_i,
                                   const float* __restrict__ top_v, const float* __restrict__ lse,
                                   int32_t* __restrict__ tokens_io, int32_t* __restrict__ parents_io,
                                   int32_t* __restrict__ node_off_io) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int K = a.K;
  int32_t* tok = a.tok + (size_t)b * a.max_nodes;
  int32_t* par = a.par + (size_t)b * a.max_nodes;
  float* val = a.val + (size_t)b * a.max_nodes;
  TreeOffer* off = a.offers + (size_t)b * kTreeMaxOffers;
  const int base = a.n_offers[b];
  const int no = nf * K;  // offers of this step (<= blockDim.x)
  __shared__ float sv[256];
  __shared__ int so[256];
  __shared__ int taken[kTopKMax];
  const int q = threadIdx.x;
  float v = -INFINITY;
  int order = 0x7fffffff;
  if (q < no) {
    const int f = n - nf + q / K;  // offering node
    const size_t row = (size_t)b * n + f;
    const int j = q % K;
    v = val[f] + fminf(top_v[row * K + j] - lse[row], 0.f);  // a log-probability is <= 0
    order = base + q;
    TreeOffer o;
    o.v = v;
    o.depth = t + 1;
    o.order = order;
    o.parent = f;
    o.token = top_i[row * K + j];
    o.node = -1;
    off[base + q] = o;
  }
  // K block-wide selections of the best offer (value desc, order asc)
  for (int k = 0; k < K; ++k) {
    sv[q] = v;
    so[q] = order;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
      if (q < s && offer_before(sv[q + s], so[q + s], sv[q], so[q])) {
        sv[q] = sv[q + s];
        so[q] = so[q + s];
      }
      __syncthreads();
    }
    if (q == 0) taken[k] = so[0];
    __syncthreads();
    if (order == taken[k]) {
      v = -INFINITY;  // out of the remaining selections
      order = 0x7fffffff;
    }
    __syncthreads();
  }
  if (q < K) {
    const int idx = taken[q] - base;  // offer index of rank q (all K exist: no >= K)
    TreeOffer& o = off[base + idx];
    const int node = n + q;
    tok[node] = o.token;
    par[node] = o.parent;
    val[node] = o.v;
    o.node = node;
  }
  __syncthreads();
  if (q == 0) a.n_offers[b] = base + no;
  // the next step's tree, in its own row layout
  if (a.write_next) {
    const int nn = n + K;
    for (int i = q; i < nn; i += blockDim.x) {
      tokens_io[(size_t)b * nn + i] = tok[i];
      parents_io[(size_t)b * nn + i] = par[i];
    }
    if (b == 0)
      for (int i = q; i <= (int)gridDim.x; i += blockDim.x) node_off_io[i] = i * nn;
  }
}

cudaError_t launch_tree_expand(const TreeArgs& a, int B, int t, int n, int nf, const int32_t* top_i,
                               const float* top_v, const float* lse, int32_t* tokens_io, int32_t* parents_io,
                               int32_t* node_off_io, cudaStream_t s, bool pdl) {
  if (nf * a.K > 256 || a.K > kTopKMax || n + a.K > a.max_nodes) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(B), dim3(256), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, tree_expand_kernel, a, t, n, nf, top_i, top_v, lse, tokens_io, parents_io,
                            node_off_io);
}

// ---------------------------------------------------------------------------
// final rerank
// ---------------------------------------------------------------------------

// key order: value desc, depth asc, order asc
__device__ __forceinline__ bool rank_before(const TreeOffer& x, const TreeOffer& y) {
  if (x.v != y.v) return x.v > y.v;
  if (x.depth != y.depth) return x.depth < y.depth;
  return x.order < y.order;
}

// One CTA of kTreeMaxOffers threads per tree: bitonic sort of the offers, the
// `total` best kept and laid out by (depth, value desc, order) with parents mapped.
__global__ void __launch_bounds__(kTreeMaxOffers) tree_rerank_kernel(TreeArgs a, int total,
                                                                     int32_t* __restrict__ out_tok,
                                                                     int32_t* __restrict__ out_par,
                                                                     float* __restrict__ out_val) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const int q = threadIdx.x;
  __shared__ TreeOffer s[kTreeMaxOffers];
  __shared__ int pos_of[kTreeMaxNodes];
  const int no = a.n_offers[b];
  const TreeOffer* off = a.offers + (size_t)b * kTreeMaxOffers;
  if (q < no) {
    s[q] = off[q];
  } else {
    TreeOffer e;
    e.v = -INFINITY;
    e.depth = 0x7fffffff;
    e.order = 0x7fffffff;
    e.parent = 0;
    e.token = 0;
    e.node = -1;
    s[q] = e;
  }
  if (q < kTreeMaxNodes) pos_of[q] = -1;
  __syncthreads();
  for (int k = 2; k <= kTreeMaxOffers; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int p = q ^ j;
      if (p > q) {
        const bool up = (q & k) == 0;  // ascending in rank order
        const bool swap = up ? rank_before(s[p], s[q]) : rank_before(s[q], s[p]);
        if (swap) {
          const TreeOffer tmp = s[q];
          s[q] = s[p];
          s[p] = tmp;
        }
      }
      __syncthreads();
    }
  }
  // the kept offers are s[0 .. total); output slot 1 + (how many kept offers come
  // before this one by depth, value desc, order)
  int slot = -1;
  if (q < total) {
    const TreeOffer me = s[q];
    int before = 0;
    for (int i = 0; i < total; ++i) {
      const TreeOffer o = s[i];
      const bool b4 = o.depth < me.depth || (o.depth == me.depth && (o.v > me.v || (o.v == me.v && o.order < me.order)));
      before += b4 ? 1 : 0;
    }
    slot = 1 + before;
    if (me.node >= 0) pos_of[me.node] = slot;
  }
  if (q == 0) pos_of[0] = 0;
  __syncthreads();
  int32_t* ot = out_tok + (size_t)b * (total + 1);
  int32_t* op = out_par + (size_t)b * (total + 1);
  float* ov = out_val + (size_t)b * (total + 1);
  if (q == 0) {
    ot[0] = a.tok[(size_t)b * a.max_nodes];
    op[0] = -1;
    ov[0] = 0.f;
  }
  if (slot > 0) {
    const TreeOffer me = s[q];
    ot[slot] = me.token;
    op[slot] = pos_of[me.parent];  // a chosen offer's parent was chosen first (-1 would mark a bug)
    ov[slot] = me.v;
  }
}

cudaError_t launch_tree_rerank(const TreeArgs& a, int B, int total, int32_t* out_tok, int32_t* out_par,
                               float* out_val, cudaStream_t s, bool pdl) {
  if (total < 1 || total >= kTreeMaxOffers || a.max_nodes > kTreeMaxNodes) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(B), dim3(kTreeMaxOffers), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, tree_rerank_kernel, a, total, out_tok, out_par, out_val);
}

}  // namespace spec
