// Tree attention of fp32 models: one warp per (node, head), keys visited in
// slot order with an exact fp32 online softmax.
//
// Node i of a tree (local index) sits at cache slot P_b + i and at position
// P_b + depth(i).  A query row sees every prefix key (slots 0 .. P_b-1) and the
// tree keys of its own ancestors, itself included ("EAGLE-3投机解码：
// 树验证器方法", section 树draft vs 链draft).  Grouped-query attention: query
// head h reads key/value head h / (Hq/Hkv).  (bf16 models use the tensor-core
// kernel of attention_tc.cu.)
#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

__device__ __forceinline__ bool anc_has(uint64_t a0, uint64_t a1, int j) {
  return j < 64 ? ((a0 >> j) & 1ull) : ((a1 >> (j - 64)) & 1ull);
}

}  // namespace

__global__ void attn_f32_kernel(AttnArgs a) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const StepView& sv = a.sv;
  if (w >= sv.M * a.Hq) return;
  const int hd = a.hd;
  const int r = w / a.Hq;
  const int h = w - r * a.Hq;
  const int G = a.Hq / a.kv.Hkv;
  const int kvh = h / G;
  const int b = sv.row_seq[r];
  const int P = sv.P_step[b];
  const int n_b = sv.node_off[b + 1] - sv.node_off[b];
  const int seq = sv.seq_ids[b];
  const uint64_t a0 = sv.row_anc[2 * r], a1 = sv.row_anc[2 * r + 1];
  const float* kb = reinterpret_cast<const float*>(a.kv.base) + a.layer * a.kv.layer_stride() +
                    seq * a.kv.seq_stride() + kvh * a.kv.head_stride();
  const float* vb = kb + a.kv.kv_stride();
  const float* qv = reinterpret_cast<const float*>(a.q) + ((size_t)r * a.Hq + h) * hd;
  const float scale = 1.f / sqrtf((float)hd);
  constexpr int kMaxPerLane = 4;  // head_dim <= 128
  float qr[kMaxPerLane], acc[kMaxPerLane];
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int d = lane + 32 * i;
    qr[i] = d < hd ? qv[d] : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int key = 0; key < P + n_b; ++key) {
    if (key >= P && !anc_has(a0, a1, key - P)) continue;
    const float* kr = kb + (size_t)key * hd;
    float dot = 0.f;
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int d = lane + 32 * i;
      if (d < hd) dot = fmaf(qr[i], kr[d], dot);
    }
    dot = warp_sum(dot) * scale;
    const float m_new = fmaxf(m, dot);
    const float c = expf(m - m_new);
    const float p = expf(dot - m_new);
    l = l * c + p;
    const float* vr = vb + (size_t)key * hd;
    for (int i = 0; i < kMaxPerLane; ++i) {
      const int d = lane + 32 * i;
      if (d < hd) acc[i] = acc[i] * c + p * vr[d];
    }
    m = m_new;
  }
  float* out = reinterpret_cast<float*>(a.out) + ((size_t)r * a.Hq + h) * hd;
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int d = lane + 32 * i;
    if (d < hd) out[d] = acc[i] / l;
  }
}

cudaError_t launch_attention_f32(const AttnArgs& a, cudaStream_t s) {
  const int warps = a.sv.M * a.Hq;
  attn_f32_kernel<<<(warps + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace spec
