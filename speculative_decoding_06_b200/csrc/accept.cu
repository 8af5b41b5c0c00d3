// Greedy acceptance walk and K/V compaction.
//
// Acceptance ("EAGLE-3投机解码：树验证器方法", section 验证-接受语义): a draft
// token is accepted iff it equals the target's argmax at its parent; scanning
// from the root stops at the first mismatch, and the target's own token at
// the last accepted node is emitted as the bonus.  In a tree the scan moves to
// the lowest-index child whose token matches.  One warp walks one tree: each
// step tests up to 32 candidate children per ballot.
//
// Compaction: the root's K/V already sits at slot P; accepted node d (1-based
// along the path, local index node_d >= d) moves from slot P + node_d to slot
// P + d, for every layer, K and V, and kv head.  All sources are read before
// any destination is written, so the order of the moves does not matter.
#include "common.cuh"
#include "kernels.h"

namespace spec {

__global__ void accept_walk_kernel(WalkArgs w) {
  pdl_wait();
  pdl_launch_dependents();
  const StepView& sv = w.sv;
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  if (b >= sv.B) return;
  const int base = sv.node_off[b];
  const int n = sv.node_off[b + 1] - base;
  const int seq = sv.seq_ids[b];
  const int P = sv.P_step[b];
  const uint32_t step_err = *sv.err;
  if (step_err != 0) {
    // a failed step leaves the cache state untouched
    if (lane == 0) {
      w.acc_len[b] = -1;
      w.bonus[b] = -1;
      atomicOr(sv.err_sticky, step_err);
    }
    return;
  }
  int count = 0;
  int cur = 0;
  if (w.mode == STEP_PREFILL) {
    // a prompt chunk is a chain whose every node is committed
    for (int i = 1 + lane; i < n; i += 32) {
      w.acc_nodes[(size_t)b * w.max_nodes + i - 1] = i;
      w.acc_tokens[(size_t)b * w.max_nodes + i - 1] = sv.tokens[base + i];
    }
    count = n - 1;
    cur = n - 1;
  } else {
    while (true) {
      const int target = w.argmax[base + cur];
      int found = -1;
      for (int c0 = cur + 1; c0 < n; c0 += 32) {  // children have larger indices than their parent
        const int c = c0 + lane;
        const bool hit = c < n && sv.parents[base + c] == cur && sv.tokens[base + c] == target;
        const unsigned m = __ballot_sync(0xffffffffu, hit);
        if (m) {
          found = c0 + __ffs(m) - 1;
          break;
        }
      }
      if (found < 0) break;
      if (lane == 0) {
        w.acc_nodes[(size_t)b * w.max_nodes + count] = found;
        w.acc_tokens[(size_t)b * w.max_nodes + count] = sv.tokens[base + found];
      }
      ++count;
      cur = found;
    }
  }
  const int bonus = w.argmax[base + cur];
  __syncwarp();
  if (w.mode != STEP_SCORE) {
    // commit: slot P holds the root, P + d the d-th accepted node
    int32_t* hist = sv.hist + (size_t)seq * sv.max_seq;
    if (lane == 0) hist[P] = sv.tokens[base];
    for (int d = lane; d < count; d += 32) hist[P + 1 + d] = w.acc_tokens[(size_t)b * w.max_nodes + d];
    if (lane == 0) {
      sv.seq_len[seq] = P + 1 + count;
      sv.pending[seq] = bonus;
    }
  }
  if (lane == 0) {
    w.acc_len[b] = count;
    w.bonus[b] = bonus;
  }
}

cudaError_t launch_accept_walk(const WalkArgs& w, cudaStream_t s, bool pdl) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(w.sv.B);
  cfg.blockDim = dim3(32);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, accept_walk_kernel, w);
}

// grid (n_layers * 2 * Hkv, B); one CTA moves one (layer, K|V, kv head) of one sequence
__global__ void __launch_bounds__(256) kv_compact_kernel(StepView sv, KvView kv, const int32_t* __restrict__ acc_len,
                                                         const int32_t* __restrict__ acc_nodes, int max_nodes) {
  extern __shared__ __align__(16) uint8_t stage[];
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  const int a = acc_len[b];
  if (a <= 0) return;
  const int lk = blockIdx.x;  // (layer * planes + plane) * Hkv + head
  const int head = lk % kv.Hkv;
  const int kvsel = (lk / kv.Hkv) % kv.planes;
  const int layer = lk / (kv.planes * kv.Hkv);
  const int P = sv.P_step[b];
  const int seq = sv.seq_ids[b];
  uint8_t* base = reinterpret_cast<uint8_t*>(kv.base) +
                  (layer * kv.layer_stride() + kvsel * kv.kv_stride() + seq * kv.seq_stride() + head * kv.head_stride()) *
                      kv.elem;
  const int row_bytes = kv.hd * (int)kv.elem;
  const int vec_per_row = row_bytes / 16;
  const int total = a * vec_per_row;
  const int32_t* nodes = acc_nodes + (size_t)b * max_nodes;
  for (int v = threadIdx.x; v < total; v += blockDim.x) {
    const int d = v / vec_per_row, c = v - d * vec_per_row;
    const int src = P + nodes[d];
    *reinterpret_cast<uint4*>(stage + (size_t)v * 16) =
        *reinterpret_cast<const uint4*>(base + (size_t)src * row_bytes + c * 16);
  }
  __syncthreads();
  for (int v = threadIdx.x; v < total; v += blockDim.x) {
    const int d = v / vec_per_row, c = v - d * vec_per_row;
    const int dst = P + 1 + d;
    *reinterpret_cast<uint4*>(base + (size_t)dst * row_bytes + c * 16) = *reinterpret_cast<const uint4*>(stage + (size_t)v * 16);
  }
}

cudaError_t kv_compact_configure(size_t smem) {
  return cudaFuncSetAttribute(kv_compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t launch_kv_compact(const StepView& sv, const KvView& kv, int n_layers, const int32_t* acc_len,
                              const int32_t* acc_nodes, int max_nodes, cudaStream_t s, bool pdl) {
  const size_t smem = (size_t)(max_nodes - 1) * kv.hd * kv.elem;  // <= 127 rows x 512 B, attribute set by spec_init
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_layers * kv.planes * kv.Hkv, sv.B);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kv_compact_kernel, sv, kv, acc_len, acc_nodes, max_nodes);
}

// ---------------------------------------------------------------------------
// draft-head features ("EAGLE-3: Scaling up Inference Acceleration of Large
// Language Models via Training-Time Test", draft-stage description: the draft
// head takes the target's low-, mid- and high-level hidden states of each
// position, recorded during prefill and verification)
// ---------------------------------------------------------------------------

// the residual stream x (fp32 [M][d], d % 4 == 0) after a tap layer, as bf16 rows
__global__ void feature_tap_kernel(int d, const float* __restrict__ x, __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t t = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(x + t * d);
  uint2* o = reinterpret_cast<uint2*>(out + t * d);
  for (int c = threadIdx.x; c < d / 4; c += blockDim.x) {
    const float4 v = xr[c];
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&a);
    u.y = *reinterpret_cast<const uint32_t*>(&b);
    o[c] = u;
  }
}

cudaError_t launch_feature_tap(int M, int d, const float* x, __nv_bfloat16* out, cudaStream_t s, bool pdl) {
  if (M < 1 || d % 4) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M);
  cfg.blockDim = dim3(128);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, feature_tap_kernel, d, x, out);
}

// Block (k, b): the k-th node of tree b's emitted path (the root, then the
// accepted nodes) -> out[b][k][f][:] = tap[f][row of that node][:], f = 0..2.
// Nothing for k > acc_len[b].  d % 8 == 0; 16-byte copies.
__global__ void feature_gather_kernel(StepView sv, const int32_t* __restrict__ acc_len,
                                      const int32_t* __restrict__ acc_nodes, int max_nodes,
                                      const __nv_bfloat16* __restrict__ tap, int Mpad, int d,
                                      __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y, k = blockIdx.x;
  const int a = acc_len[b];
  if (k > a) return;
  const int node = k == 0 ? 0 : acc_nodes[(size_t)b * max_nodes + k - 1];
  const size_t row = (size_t)sv.node_off[b] + node;
  const int nv = d / 8;
  for (int f = 0; f < 3; ++f) {
    const uint4* src = reinterpret_cast<const uint4*>(tap + ((size_t)f * Mpad + row) * d);
    uint4* dst = reinterpret_cast<uint4*>(out + (((size_t)b * max_nodes + k) * 3 + f) * d);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) dst[i] = src[i];
  }
}

// Prefill: every row in order, out[r][f][:] = tap[f][r][:].
__global__ void feature_rows_out_kernel(const __nv_bfloat16* __restrict__ tap, int Mpad, int d,
                                        __nv_bfloat16* __restrict__ out) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t r = blockIdx.x;
  const int nv = d / 8;
  for (int f = 0; f < 3; ++f) {
    const uint4* src = reinterpret_cast<const uint4*>(tap + ((size_t)f * Mpad + r) * d);
    uint4* dst = reinterpret_cast<uint4*>(out + (r * 3 + f) * d);
    for (int i = threadIdx.x; i < nv; i += blockDim.x) dst[i] = src[i];
  }
}

cudaError_t launch_feature_rows_out(int M, const __nv_bfloat16* tap, int Mpad, int d, __nv_bfloat16* out,
                                    cudaStream_t s, bool pdl) {
  if (d % 8 || M < 1) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M);
  cfg.blockDim = dim3(128);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, feature_rows_out_kernel, tap, Mpad, d, out);
}

cudaError_t launch_feature_gather(const StepView& sv, const int32_t* acc_len, const int32_t* acc_nodes,
                                  int max_nodes, const __nv_bfloat16* tap, int Mpad, int d, __nv_bfloat16* out,
                                  cudaStream_t s, bool pdl) {
  if (d % 8 || max_nodes < 1) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(max_nodes, sv.B);
  cfg.blockDim = dim3(128);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, feature_gather_kernel, sv, acc_len, acc_nodes, max_nodes, tap, Mpad, d, out);
}

// draft head: out[r] = [g[r] | E[tokens[r]]]  (bf16, 2d wide)
__global__ void gather_concat_kernel(int d, const __nv_bfloat16* __restrict__ g, const int32_t* __restrict__ tokens,
                                     const __nv_bfloat16* __restrict__ embed, __nv_bfloat16* __restrict__ out) {
  const int r = blockIdx.x;
  const uint4* gs = reinterpret_cast<const uint4*>(g + (size_t)r * d);
  const uint4* es = reinterpret_cast<const uint4*>(embed + (size_t)tokens[r] * d);
  uint4* o = reinterpret_cast<uint4*>(out + (size_t)r * 2 * d);
  const int nv = d / 8;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    o[i] = gs[i];
    o[nv + i] = es[i];
  }
}

cudaError_t launch_gather_concat(int M, int d, const __nv_bfloat16* g, const int32_t* tokens,
                                 const __nv_bfloat16* embed, __nv_bfloat16* out, cudaStream_t s) {
  gather_concat_kernel<<<M, 128, 0, s>>>(d, g, tokens, embed, out);
  return cudaGetLastError();
}

}  // namespace spec
