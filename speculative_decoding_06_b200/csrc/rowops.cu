// Row-wise kernels of the verification forward: tree metadata with the
// embedding gather and first RMSNorm, split-K reduction fused with the
// residual add and the next RMSNorm, rotary embedding fused with the K/V cache
// store, the LM-head argmax reductions, and the fp32 (SIMT) GEMM used by the
// fp32 model path.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (threadIdx.x < 32) {
    t = threadIdx.x < NT / 32 ? red[threadIdx.x] : 0.f;
    t = warp_sum(t);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  t = red[0];
  __syncthreads();
  return t;
}


}  // namespace

cudaLaunchConfig_t make_cfg(dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cfg;
}

// ---------------------------------------------------------------------------
// tree metadata + embedding + RMSNorm
// ---------------------------------------------------------------------------
// One CTA per node.  A node's depth and ancestor set come from walking its
// parent links up to the root ("EAGLE-3投机解码：树验证器方法", section 树draft vs
// 链draft: every token sees only its ancestors); its position is P_b + depth.
// SPLIT: write the normalised row as split bf16 (bf16 models); else as T (fp32 models)
// bf16 models leave the normalisation to the next GEMM: xn = split(x*w) and
// ss[0][r] = sum x^2 (the other n_ss-1 partial slots are zero).
template <typename T, bool SPLIT>
__global__ void __launch_bounds__(256) embed_meta_kernel(StepView sv, const T* __restrict__ embed,
                                                         const T* __restrict__ norm_w, int d, float eps,
                                                         float* __restrict__ x, void* __restrict__ xn,
                                                         float* __restrict__ ss_out, int n_ss, int ss_ld,
                                                         const double* __restrict__ inv_freq, int half, int mode,
                                                         __nv_bfloat16* __restrict__ e_out, int e_ld, int e_col) {
  __shared__ int s_pos;
  __shared__ float red[8];
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  if (threadIdx.x == 0) {
    int b = 0;
    while (b + 1 < sv.B && sv.node_off[b + 1] <= r) ++b;
    const int base = sv.node_off[b];
    const int n = sv.node_off[b + 1] - base;
    const int i = r - base;
    const int seq = sv.seq_ids[b];
    const int P = sv.seq_len[seq];
    uint64_t a0 = 0, a1 = 0;
    int depth = -1;
    int j = i;
    int guard = 0;
    while (j >= 0 && guard <= n) {
      if (j < 64) a0 |= 1ull << j; else a1 |= 1ull << (j - 64);
      const int pj = sv.parents[base + j];
      if (pj >= j) {  // malformed links are rejected on the host; never follow one here
        set_error(sv.err, SPEC_DEVERR_BOUNDS);
        break;
      }
      j = pj;
      ++depth;
      ++guard;
    }
    sv.row_seq[r] = b;
    sv.row_local[r] = i;
    sv.row_slot[r] = P + i < sv.max_seq ? P + i : -1;
    sv.row_sid[r] = seq;
    sv.row_pos[r] = P + depth;
    sv.row_anc[2 * r] = a0;
    sv.row_anc[2 * r + 1] = a1;
    if (i == 0) {
      sv.P_step[b] = P;
      if (mode == STEP_VERIFY && sv.tokens[r] != sv.pending[seq]) set_error(sv.err, SPEC_DEVERR_ROOT);
    }
    s_pos = P + depth;
  }
  __syncthreads();
  const int pos = s_pos;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    double sn, cs;
    sincos((double)pos * inv_freq[j], &sn, &cs);
    sv.rope_cs[(size_t)r * half + j] = make_float2((float)cs, (float)sn);
  }
  const int tok = sv.tokens[r];
  const T* e = embed + (size_t)tok * d;
  if (SPLIT && e_out) {  // draft head: the embedding is half of the next GEMM's operand
    for (int k = threadIdx.x; k < d; k += blockDim.x) split_store(e_out, r, e_ld, e_col + k, to_f32(e[k]));
    return;
  }
  float* xr = x + (size_t)r * d;
  float ss = 0.f;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    const float v = to_f32(e[k]);
    xr[k] = v;
    ss += v * v;
  }
  ss = block_sum<256>(ss, red);
  if (SPLIT) {
    for (int k = threadIdx.x; k < d; k += blockDim.x)
      split_store(reinterpret_cast<__nv_bfloat16*>(xn), r, d, k, xr[k] * to_f32(norm_w[k]));
    for (int i = threadIdx.x; i < n_ss; i += blockDim.x) ss_out[(size_t)i * ss_ld + r] = i == 0 ? ss : 0.f;
  } else {
    const float inv = rsqrtf(ss / (float)d + eps);
    for (int k = threadIdx.x; k < d; k += blockDim.x)
      reinterpret_cast<T*>(xn)[(size_t)r * d + k] = from_f32<T>(xr[k] * inv * to_f32(norm_w[k]));
  }
}

cudaError_t launch_embed_meta(int dtype, const StepView& sv, const void* embed, const void* norm_w, int d, float eps,
                              float* x, void* xn, float* ss, int n_ss, int ss_ld, const double* inv_freq, int half,
                              int mode, cudaStream_t s, bool pdl, __nv_bfloat16* e_out, int e_ld, int e_col) {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(sv.M), dim3(256), 0, s, pdl, attr);
  if (dtype == 0)
    return cudaLaunchKernelEx(&cfg, embed_meta_kernel<float, false>, sv, (const float*)embed, (const float*)norm_w, d,
                              eps, x, xn, ss, n_ss, ss_ld, inv_freq, half, mode, (__nv_bfloat16*)nullptr, 0, 0);
  return cudaLaunchKernelEx(&cfg, embed_meta_kernel<__nv_bfloat16, true>, sv, (const __nv_bfloat16*)embed,
                            (const __nv_bfloat16*)norm_w, d, eps, x, xn, ss, n_ss, ss_ld, inv_freq, half, mode, e_out,
                            e_ld, e_col);
}

// ---------------------------------------------------------------------------
// split-K reduction + residual + RMSNorm
// ---------------------------------------------------------------------------
// x[r] += sum_s partial[s][r] (fixed order, deterministic); xn[r] = x[r] * rsqrt(mean x^2 + eps) * w.
// A row is shared by a cluster of CL CTAs, each owning d/CL columns; the CTAs
// exchange their partial sums of squares through distributed shared memory and
// add them in rank order, so every CTA applies the same normaliser.
template <typename T, bool SPLIT>
__global__ void __launch_bounds__(256) residual_norm_kernel(int d, int S, const float* __restrict__ partial,
                                                            size_t split_stride, float* __restrict__ x,
                                                            void* __restrict__ xn, const T* __restrict__ w, float eps) {
  __shared__ float red[8];
  __shared__ float cta_ss;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x / CL;
  const int cols = d / CL;
  const int c0 = rank * cols;
  float* xr = x + (size_t)r * d;
  const float* pr = partial + (size_t)r * d;
  float ss = 0.f;
  for (int k = c0 + threadIdx.x * 4; k < c0 + cols; k += blockDim.x * 4) {
    float4 acc = *reinterpret_cast<const float4*>(xr + k);
    for (int sp = 0; sp < S; ++sp) {
      const float4 p = *reinterpret_cast<const float4*>(pr + sp * split_stride + k);
      acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
    }
    *reinterpret_cast<float4*>(xr + k) = acc;
    ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
  }
  ss = block_sum<256>(ss, red);
  if (threadIdx.x == 0) cta_ss = ss;
  cluster.sync();
  float total = 0.f;
  for (int q = 0; q < CL; ++q) total += *cluster.map_shared_rank(&cta_ss, q);
  cluster.sync();  // keep every CTA's cta_ss alive until all have read it
  const float inv = rsqrtf(total / (float)d + eps);
  for (int k = c0 + threadIdx.x; k < c0 + cols; k += blockDim.x) {
    const float v = xr[k] * inv * to_f32(w[k]);
    if (SPLIT) split_store(reinterpret_cast<__nv_bfloat16*>(xn), r, d, k, v);
    else reinterpret_cast<T*>(xn)[(size_t)r * d + k] = from_f32<T>(v);
  }
}

int residual_norm_cluster(int d) {
  // 4 KB-wide slices (one float4 per thread) when the row is wide enough
  if (d % 4096 == 0 && d >= 4096) return 4;
  if (d % 2048 == 0 && d >= 2048) return 2;
  return 1;
}

cudaError_t launch_residual_norm(int dtype, int M, int d, int S, const float* partial, size_t split_stride, float* x,
                                 void* xn, const void* w, float eps, cudaStream_t s, bool pdl) {
  const int CL = residual_norm_cluster(d);
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = make_cfg(dim3(M * CL), dim3(256), 0, s, pdl, attr);
  attr[cfg.numAttrs].id = cudaLaunchAttributeClusterDimension;
  attr[cfg.numAttrs].val.clusterDim.x = CL;
  attr[cfg.numAttrs].val.clusterDim.y = 1;
  attr[cfg.numAttrs].val.clusterDim.z = 1;
  cfg.numAttrs += 1;
  if (dtype == 0)
    return cudaLaunchKernelEx(&cfg, residual_norm_kernel<float, false>, d, S, partial, split_stride, x, xn,
                              (const float*)w, eps);
  return cudaLaunchKernelEx(&cfg, residual_norm_kernel<__nv_bfloat16, true>, d, S, partial, split_stride, x, xn,
                            (const __nv_bfloat16*)w, eps);
}

// ---------------------------------------------------------------------------
// split-K reduction + rotary embedding + K/V cache store
// ---------------------------------------------------------------------------
// grid (node, group of 8 heads of q|k|v)
constexpr int kRopeHeadsPerCta = 8;
// Rotate-half pairing: element j and element j + hd/2 of a head form one pair,
// rotated by pos * theta^(-2j/hd) (table computed in double per step).
// T is the attention operand type: fp32 for fp32 models, fp16 for bf16 models
// (q and the K/V cache; 10 mantissa bits at 2 bytes).
template <typename T>
__global__ void __launch_bounds__(256) qkv_rope_store_kernel(StepView sv, int S, const float* __restrict__ partial,
                                                             size_t split_stride, int Hq, int Hkv, int hd,
                                                             T* __restrict__ q_out, KvView kv, int layer) {
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  const int half = hd / 2;
  const int n_cols = (Hq + 2 * Hkv) * hd;
  const int h_begin = blockIdx.y * kRopeHeadsPerCta;
  const int h_end = min(Hq + 2 * Hkv, h_begin + kRopeHeadsPerCta);
  const float* pr = partial + (size_t)r * n_cols;
  const int b = sv.row_seq[r];
  const int slot = sv.P_step[b] + sv.row_local[r];
  const int seq = sv.seq_ids[b];
  const bool slot_ok = slot < kv.max_seq;
  if (!slot_ok && threadIdx.x == 0 && blockIdx.y == 0) set_error(sv.err, SPEC_DEVERR_BOUNDS);
  T* kbase = reinterpret_cast<T*>(kv.base) + layer * kv.layer_stride() + seq * kv.seq_stride() + (size_t)slot * hd;
  T* vbase = kbase + kv.kv_stride();
  const float2* cs = sv.rope_cs + (size_t)r * half;
  const int pairs = (h_end - h_begin) * half;
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const int h = h_begin + p / half;
    const int j = p % half;
    const int c1 = h * hd + j;
    const int c2 = c1 + half;
    float v1 = 0.f, v2 = 0.f;
    for (int sp = 0; sp < S; ++sp) {
      v1 += pr[sp * split_stride + c1];
      v2 += pr[sp * split_stride + c2];
    }
    if (h < Hq + Hkv) {
      const float2 c = cs[j];
      const float o1 = v1 * c.x - v2 * c.y;
      const float o2 = v2 * c.x + v1 * c.y;
      v1 = o1;
      v2 = o2;
    }
    if (h < Hq) {
      T* q = q_out + (size_t)r * Hq * hd;
      q[c1] = from_f32<T>(v1);
      q[c2] = from_f32<T>(v2);
    } else if (slot_ok) {
      const int kh = (h < Hq + Hkv) ? h - Hq : h - Hq - Hkv;
      T* dst = ((h < Hq + Hkv) ? kbase : vbase) + kh * kv.head_stride();
      dst[j] = from_f32<T>(v1);
      dst[j + half] = from_f32<T>(v2);
    }
  }
}

cudaError_t launch_qkv_rope_store(int dtype, const StepView& sv, int S, const float* partial, size_t split_stride,
                                  int Hq, int Hkv, int hd, void* q_out, const KvView& kv, int layer, cudaStream_t s,
                                  bool pdl) {
  cudaLaunchAttribute attr[1];
  const int groups = (Hq + 2 * Hkv + kRopeHeadsPerCta - 1) / kRopeHeadsPerCta;
  cudaLaunchConfig_t cfg = make_cfg(dim3(sv.M, groups), dim3(256), 0, s, pdl, attr);
  if (dtype == 0)
    return cudaLaunchKernelEx(&cfg, qkv_rope_store_kernel<float>, sv, S, partial, split_stride, Hq, Hkv, hd,
                              (float*)q_out, kv, layer);
  return cudaLaunchKernelEx(&cfg, qkv_rope_store_kernel<__half>, sv, S, partial, split_stride, Hq, Hkv, hd,
                            (__half*)q_out, kv, layer);
}

// ---------------------------------------------------------------------------
// fp32 path: SwiGLU and a plain tiled SIMT GEMM (FFMA, no TF32)
// ---------------------------------------------------------------------------
__global__ void swiglu_f32_kernel(int M, int F, const float* __restrict__ gu, float* __restrict__ h) {
  const size_t total = (size_t)M * F;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / F, f = i - r * F;
    const float g = gu[r * 2 * F + f];
    const float u = gu[r * 2 * F + F + f];
    h[i] = g / (1.0f + expf(-g)) * u;
  }
}

cudaError_t launch_swiglu_f32(int M, int F, const float* gu, float* h, cudaStream_t s) {
  const int blocks = (int)(((size_t)M * F + 255) / 256);
  swiglu_f32_kernel<<<blocks < 4096 ? blocks : 4096, 256, 0, s>>>(M, F, gu, h);
  return cudaGetLastError();
}

// C[t][o] = sum_k A[t][k] * W[o][k]; 16 tokens x 64 outputs per block, k ascending.
__global__ void __launch_bounds__(256) gemm_simt_f32_kernel(const float* __restrict__ A, int lda,
                                                            const float* __restrict__ W, int K,
                                                            float* __restrict__ C, int ldc, int M, int N) {
  __shared__ float sA[16][33];
  __shared__ float sW[64][33];
  const int t0 = blockIdx.y * 16, o0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15;   // output column group
  const int ty = threadIdx.x >> 4;   // token row
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k0 = 0; k0 < K; k0 += 32) {
    for (int i = threadIdx.x; i < 16 * 32; i += 256) {
      const int rr = i / 32, kk = i % 32;
      const int t = t0 + rr, k = k0 + kk;
      sA[rr][kk] = (t < M && k < K) ? A[(size_t)t * lda + k] : 0.f;
    }
    for (int i = threadIdx.x; i < 64 * 32; i += 256) {
      const int rr = i / 32, kk = i % 32;
      const int o = o0 + rr, k = k0 + kk;
      sW[rr][kk] = (o < N && k < K) ? W[(size_t)o * K + k] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float a = sA[ty][kk];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = fmaf(a, sW[tx + 16 * j][kk], acc[j]);
    }
    __syncthreads();
  }
  const int t = t0 + ty;
  if (t < M) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int o = o0 + tx + 16 * j;
      if (o < N) C[(size_t)t * ldc + o] = acc[j];
    }
  }
}

cudaError_t launch_gemm_simt_f32(const float* A, int lda, const float* W, int K, float* C, int ldc, int M, int N,
                                 cudaStream_t s) {
  dim3 grid((N + 63) / 64, (M + 15) / 16);
  gemm_simt_f32_kernel<<<grid, 256, 0, s>>>(A, lda, W, K, C, ldc, M, N);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// LM-head reductions
// ---------------------------------------------------------------------------
// one warp per token: merge the per-tile (best, index, runner-up) in tile order
// One CTA per token: every thread merges a strided set of the vocabulary
// tiles' (best, index, runner-up) with its loads issued together, then the
// warps and the CTA merge (lowest index on equal values).
__global__ void __launch_bounds__(256) top2_reduce_kernel(int M, int tiles, const Top2* __restrict__ part,
                                                         int top_ld, int32_t* __restrict__ argmax,
                                                         float* __restrict__ top1, float* __restrict__ top2,
                                                         const uint32_t* __restrict__ err) {
  __shared__ Top2 wbest[8];
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  if (t >= M) return;
  if (err && *err) {  // the partials may be stale: say so instead of reducing them
    if (threadIdx.x == 0) {
      argmax[t] = -1;
      top1[t] = __int_as_float(0x7fc00000);
      top2[t] = __int_as_float(0x7fc00000);
    }
    return;
  }
  constexpr int kU = 4;
  Top2 best;
  best.v1 = -INFINITY; best.i1 = 0x7fffffff; best.v2 = -INFINITY;
  for (int i0 = threadIdx.x; i0 < tiles; i0 += kU * blockDim.x) {
    Top2 x[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < tiles) {
        x[u] = part[(size_t)i * top_ld + t];
      } else {
        x[u].v1 = -INFINITY; x[u].i1 = 0x7fffffff; x[u].v2 = -INFINITY;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) best = top2_merge(best, x[u]);
  }
  best = warp_top2(best);
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) wbest[warp] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    Top2 r = wbest[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = top2_merge(r, wbest[w]);
    argmax[t] = r.i1;
    top1[t] = r.v1;
    top2[t] = r.v2;
  }
}

cudaError_t launch_top2_reduce(int M, int tiles, const Top2* part, int top_ld, int32_t* argmax, float* top1,
                               float* top2, cudaStream_t s, bool pdl, const uint32_t* err) {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(M), dim3(256), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, top2_reduce_kernel, M, tiles, part, top_ld, argmax, top1, top2, err);
}

__global__ void rows_top2_f32_kernel(int M, int V, const float* __restrict__ logits, int32_t* __restrict__ argmax,
                                     float* __restrict__ top1, float* __restrict__ top2, float inv_temp,
                                     uint32_t seed_lo, uint32_t seed_hi, const int32_t* __restrict__ row_sid,
                                     const int32_t* __restrict__ row_pos) {
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= M) return;
  const bool sample = inv_temp > 0.f;
  const int sid = sample ? row_sid[t] : 0;
  const int pos = sample ? row_pos[t] : 0;
  Top2 best;
  best.v1 = -INFINITY; best.i1 = 0x7fffffff; best.v2 = -INFINITY;
  for (int v = lane; v < V; v += 32) {
    Top2 x;
    const float l = logits[(size_t)t * V + v];
    x.v1 = sample ? fmaf(l, inv_temp, gumbel_noise(seed_lo, seed_hi, sid, pos, v)) : l;
    x.i1 = v; x.v2 = -INFINITY;
    best = top2_merge(best, x);
  }
  best = warp_top2(best);
  if (lane == 0) {
    argmax[t] = best.i1;
    top1[t] = best.v1;
    top2[t] = best.v2;
  }
}

cudaError_t launch_rows_top2_f32(int M, int V, const float* logits, int32_t* argmax, float* top1, float* top2,
                                 cudaStream_t s, float inv_temp, uint32_t seed_lo, uint32_t seed_hi,
                                 const int32_t* row_sid, const int32_t* row_pos) {
  if (inv_temp > 0.f && (!row_sid || !row_pos)) return cudaErrorInvalidValue;
  rows_top2_f32_kernel<<<(M + 7) / 8, 256, 0, s>>>(M, V, logits, argmax, top1, top2, inv_temp, seed_lo, seed_hi,
                                                   row_sid, row_pos);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// bf16 rows -> split-bf16 GEMM operand
// ---------------------------------------------------------------------------
// Rows that are already bf16 (the draft head's input features) have a zero lo
// part.  16 bytes per thread.
__global__ void __launch_bounds__(256) split_rows_kernel(const uint4* __restrict__ src, int rows, int cols8,
                                                        uint4* __restrict__ dst) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n = (size_t)rows * cols8;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / cols8);
    const int c = (int)(i - (size_t)t * cols8);
    dst[(size_t)split_row(t, 0) * cols8 + c] = src[i];
    dst[(size_t)split_row(t, 1) * cols8 + c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

cudaError_t launch_split_rows(const __nv_bfloat16* src, int rows, int cols, __nv_bfloat16* dst, cudaStream_t s,
                              bool pdl) {
  if (cols % 8) return cudaErrorInvalidValue;
  const int cols8 = cols / 8;
  const size_t n = (size_t)rows * cols8;
  const int grid = (int)std::min<size_t>((n + 255) / 256, 148 * 8);
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(grid), dim3(256), 0, s, pdl, attr);
  return cudaLaunchKernelEx(&cfg, split_rows_kernel, reinterpret_cast<const uint4*>(src), rows, cols8,
                            reinterpret_cast<uint4*>(dst));
}

// ---------------------------------------------------------------------------
// top-k per row (the draft head's candidate list)
// ---------------------------------------------------------------------------
// One CTA per row.  Each thread keeps a sorted list of its best K values (in
// registers: K is a compile-time constant) over a strided slice of the row;
// each warp then merges its lanes' lists by K rounds of a warp-wide best-of,
// and warp 0 merges the eight warp lists the same way.  Order: value
// descending, index ascending.
namespace {
__device__ __forceinline__ bool topk_better(float a, int ai, float b, int bi) {
  return a > b || (a == b && ai < bi);
}
// K rounds: each round the best head among the lanes' lists is taken
template <int K>
__device__ __forceinline__ void warp_merge_topk(const float (&lv)[K], const int (&li)[K], float* out_v, int* out_i) {
  const int lane = threadIdx.x & 31;
  int head = 0;
#pragma unroll
  for (int r = 0; r < K; ++r) {
    // this lane's current head, selected without dynamic register indexing
    float v = -INFINITY;
    int i = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < K; ++j)
      if (j == head) {
        v = lv[j];
        i = li[j];
      }
    int src = lane;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float v2 = __shfl_xor_sync(0xffffffffu, v, o);
      const int i2 = __shfl_xor_sync(0xffffffffu, i, o);
      const int s2 = __shfl_xor_sync(0xffffffffu, src, o);
      if (topk_better(v2, i2, v, i) || (v2 == v && i2 == i && s2 < src)) {
        v = v2;
        i = i2;
        src = s2;
      }
    }
    if (lane == src) ++head;
    if (lane == 0) {
      out_v[r] = v;
      out_i[r] = i;
    }
  }
}
}  // namespace

// Top-k of a row from the per-tile candidates of the LM head's TOPK epilogue: each
// 128-row vocabulary tile gave kCandSlots candidates holding its k best (in no
// particular order; unused slots -inf) and its (max, sum of exp(l - max)).  The
// row's k best are among the tiles' k best; its log-sum-exp combines the tiles'
// pairs.  One CTA per row; thread j takes tiles j, j + 256, ...
template <int K, bool LSE>
__global__ void __launch_bounds__(256) topk_merge_kernel(int tiles, const float* __restrict__ cand_v,
                                                        const int32_t* __restrict__ cand_i,
                                                        const float2* __restrict__ cand_lse,
                                                        int32_t* __restrict__ out_i, float* __restrict__ out_v,
                                                        float* __restrict__ out_lse,
                                                        const int32_t* __restrict__ id_map) {
  __shared__ float wv[8][K];
  __shared__ int wi[8][K];
  __shared__ float lse_m[8], lse_s[8];
  pdl_wait();
  pdl_launch_dependents();
  const int r = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr float kLog2e = 1.4426950408889634f;
  float lv[K];
  int li[K];
#pragma unroll
  for (int j = 0; j < K; ++j) {
    lv[j] = -INFINITY;
    li[j] = 0x7fffffff;
  }
  float lm = -INFINITY, ls = 0.f;
  for (int t = threadIdx.x; t < tiles; t += blockDim.x) {
    const size_t b = (size_t)r * tiles + t;
    const float* cv = cand_v + b * kCandSlots;
    const int32_t* ci = cand_i + b * kCandSlots;
    for (int j = 0; j < kCandSlots; ++j) {
      float x = __ldcs(cv + j);
      int c = __ldcs(ci + j);
      if (!topk_better(x, c, lv[K - 1], li[K - 1])) continue;
#pragma unroll
      for (int q = 0; q < K; ++q) {
        if (topk_better(x, c, lv[q], li[q])) {
          const float tv = lv[q];
          const int ti = li[q];
          lv[q] = x;
          li[q] = c;
          x = tv;
          c = ti;
        }
      }
    }
    if (LSE) {
      const float2 pr = __ldcs(cand_lse + b);
      if (pr.x > -INFINITY) {
        if (pr.x > lm) {
          ls = (lm == -INFINITY ? 0.f : ls * fast_exp2((lm - pr.x) * kLog2e));
          lm = pr.x;
        }
        ls += pr.y * fast_exp2((pr.x - lm) * kLog2e);
      }
    }
  }
  if (LSE) {
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, lm, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, ls, o);
      const float mm = fmaxf(lm, m2);
      if (mm > -INFINITY) {
        ls = (lm == -INFINITY ? 0.f : ls * fast_exp2((lm - mm) * kLog2e)) +
             (m2 == -INFINITY ? 0.f : s2 * fast_exp2((m2 - mm) * kLog2e));
        lm = mm;
      }
    }
    if (lane == 0) {
      lse_m[warp] = lm;
      lse_s[warp] = ls;
    }
  }
  warp_merge_topk<K>(lv, li, wv[warp], wi[warp]);
  __syncthreads();
  if (warp == 0) {
    float mv[K];
    int mi[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      mv[j] = lane < 8 ? wv[lane][j] : -INFINITY;
      mi[j] = lane < 8 ? wi[lane][j] : 0x7fffffff;
    }
    __syncwarp();
    warp_merge_topk<K>(mv, mi, wv[0], wi[0]);
    __syncwarp();
    if (lane < K) {
      out_v[(size_t)r * K + lane] = wv[0][lane];
      out_i[(size_t)r * K + lane] = id_map ? id_map[wi[0][lane]] : wi[0][lane];
    }
    if (LSE && lane == 0) {
      float M0 = -INFINITY;
      for (int w = 0; w < 8; ++w) M0 = fmaxf(M0, lse_m[w]);
      float S0 = 0.f;
      for (int w = 0; w < 8; ++w)
        if (lse_m[w] > -INFINITY) S0 += lse_s[w] * fast_exp2((lse_m[w] - M0) * kLog2e);
      out_lse[r] = M0 + __logf(S0);
    }
  }
}

cudaError_t launch_topk_merge(int M, int tiles, int k, const float* cand_v, const int32_t* cand_i,
                              const float2* cand_lse, int32_t* idx, float* val, float* lse, cudaStream_t s, bool pdl,
                              const int32_t* id_map) {
  if (M < 1 || tiles < 1 || k < 1 || k > kTopKMax) return cudaErrorInvalidValue;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = make_cfg(dim3(M), dim3(256), 0, s, pdl, attr);
  const bool l = lse != nullptr;
  switch (k) {
#define SPEC_TOPK_MERGE(KK)                                                                                         \
  case KK:                                                                                                          \
    return l ? cudaLaunchKernelEx(&cfg, topk_merge_kernel<KK, true>, tiles, cand_v, cand_i, cand_lse, idx, val, lse, \
                                  id_map)                                                                           \
             : cudaLaunchKernelEx(&cfg, topk_merge_kernel<KK, false>, tiles, cand_v, cand_i, cand_lse, idx, val, lse, \
                                  id_map);
    SPEC_TOPK_MERGE(4)
    SPEC_TOPK_MERGE(8)
    SPEC_TOPK_MERGE(10)
    SPEC_TOPK_MERGE(16)
#undef SPEC_TOPK_MERGE
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace spec
