// Tree attention over the K/V cache.
//
// Node i of a tree (local index) sits at cache slot P_b + i and at position
// P_b + depth(i).  Query rows see every prefix key (slots 0 .. P_b-1) and the
// tree keys of their own ancestors, themselves included ("EAGLE-3投机解码：
// 树验证器方法", section 树draft vs 链draft).  Grouped-query attention: query head
// h reads key/value head h / (Hq/Hkv).
//
// bf16-model path (flash-decoding): the keys [0, P_b + n_b) are cut into chunks;
// one CTA handles one (sequence, kv head, chunk, block of 64 query rows).  The
// query rows of a kv head are its G = Hq/Hkv heads for every tree node, so a
// K/V chunk loaded once serves all of them.  q, the K/V cache and the
// probabilities are fp16 (10 mantissa bits at 2 bytes); scores and P.V run on
// fp16 mma.sync tiles with fp32 accumulation and an fp32 online softmax (quad
// shuffles); the ancestor
// mask applies only to keys at or beyond P_b.  Each CTA writes an fp32 partial
// (normalised output + log-sum-exp); the last CTA of each (sequence, kv head,
// row block) to finish combines the chunks and writes the output as split bf16
// for the O-projection GEMM.
//
// fp32 path: one warp per (node, head), exact fp32 scalar arithmetic.
#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

constexpr int kRowsPerCta = 64;
constexpr int kKeyBlock = 64;
constexpr int kStride = 136;  // bf16 elements per smem row (128 + 8 pad: conflict-free ldmatrix)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_f16_16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ bool anc_has(uint64_t a0, uint64_t a1, int j) {
  return j < 64 ? ((a0 >> j) & 1ull) : ((a1 >> (j - 64)) & 1ull);
}

}  // namespace

__global__ void __launch_bounds__(128) attn_chunk_f16_kernel(AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  __half* sQ = reinterpret_cast<__half*>(smem_raw);
  __half* sK = sQ + kRowsPerCta * kStride;          // [2][64][kStride]
  __half* sV = sK + 2 * kKeyBlock * kStride;        // [2][64][kStride]

  // The chunks of one (sequence, kv head, row block) form a thread-block
  // cluster along x: each writes its partial, signals every peer, and the
  // peers then merge disjoint row slices.
  __shared__ __align__(8) uint64_t donebar;
  __shared__ int s_ok;
  pdl_wait();
  pdl_launch_dependents();
  const StepView& sv = a.sv;
  const int hd = 128;
  const int Hkv = a.kv.Hkv;
  const int G = a.Hq / Hkv;
  const int bk = blockIdx.z;
  const int b = bk / Hkv;
  const int kvh = bk - b * Hkv;
  const bool b_ok = b < sv.B;
  const int base = b_ok ? sv.node_off[b] : 0;
  const int n_b = b_ok ? sv.node_off[b + 1] - base : 0;
  const int rows = n_b * G;
  const int row0 = blockIdx.y * kRowsPerCta;
  const int P = b_ok ? sv.P_step[b] : 0;
  const int Lk = P + n_b;
  const int nc = (Lk + a.chunk - 1) / a.chunk;  // chunks this sequence needs (<= cluster size)
  if (threadIdx.x == 0) {
    mbar_init(&donebar, nc > 0 ? nc : 1);
    fence_barrier_init();
  }
  cluster_sync_all();  // every barrier is initialised before any peer arrives
  if (!b_ok || row0 >= rows) return;
  const int c0 = blockIdx.x * a.chunk;
  if (c0 >= Lk) return;  // this chunk lies beyond the sequence: no partial, no signal
  const int c1 = min(c0 + a.chunk, Lk);
  const int seq = sv.seq_ids[b];

  const __half* kbase = reinterpret_cast<const __half*>(a.kv.base) + a.layer * a.kv.layer_stride() +
                        seq * a.kv.seq_stride() + kvh * a.kv.head_stride();
  const __half* vbase = kbase + a.kv.kv_stride();
  const __half* q = reinterpret_cast<const __half*>(a.q);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- Q tile (64 rows x 128 dims), zero rows beyond this tree's rows
  for (int c = tid; c < kRowsPerCta * 16; c += 128) {
    const int rr = c >> 4, ch = c & 15;
    const int qr = row0 + rr;
    const bool ok = qr < rows;
    const int node = ok ? qr / G : 0;
    const int h = kvh * G + (ok ? qr - node * G : 0);
    const __half* src = q + ((size_t)(base + node) * a.Hq + h) * hd + ch * 8;
    cp_async16(sQ + rr * kStride + ch * 8, src, ok);
  }
  auto load_kv = [&](int buf, int kstart) {
    for (int c = tid; c < kKeyBlock * 16; c += 128) {
      const int kr = c >> 4, ch = c & 15;
      const int key = kstart + kr;
      const bool ok = key < c1;
      const size_t off = (size_t)(ok ? key : 0) * hd + ch * 8;
      cp_async16(sK + (buf * kKeyBlock + kr) * kStride + ch * 8, kbase + off, ok);
      cp_async16(sV + (buf * kKeyBlock + kr) * kStride + ch * 8, vbase + off, ok);
    }
  };
  load_kv(0, c0);
  cp_async_commit();

  // ---- per-thread row bookkeeping: rows g and g+8 of this warp's 16
  const int g = lane >> 2, t4 = lane & 3;
  uint64_t anc[2][2];
  bool row_ok[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int qr = row0 + warp * 16 + g + hr * 8;
    row_ok[hr] = qr < rows;
    const int node = row_ok[hr] ? qr / G : 0;
    anc[hr][0] = sv.row_anc[2 * (base + node)];
    anc[hr][1] = sv.row_anc[2 * (base + node) + 1];
  }

  const float sl2 = 1.4426950408889634f / sqrtf((float)hd);  // softmax scale in log2 units
  float m_run[2] = {-INFINITY, -INFINITY};
  float l_run[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

  uint32_t qf[8][4];
  const int nblk = (c1 - c0 + kKeyBlock - 1) / kKeyBlock;
  for (int blk = 0; blk < nblk; ++blk) {
    const int buf = blk & 1;
    if (blk + 1 < nblk) {
      load_kv(buf ^ 1, c0 + (blk + 1) * kKeyBlock);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (blk == 0) {
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t addr = smem_u32(sQ + (warp * 16 + (lane & 15)) * kStride + ks * 16 + (lane >> 4) * 8);
        ldsm_x4(addr, qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
      }
    }
    const __half* K_ = sK + buf * kKeyBlock * kStride;
    const __half* V_ = sV + buf * kKeyBlock * kStride;
    const int kstart = c0 + blk * kKeyBlock;

    // S = Q K^T  (16 rows x 64 keys per warp)
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        uint32_t b0, b1, b2, b3;
        const uint32_t addr = smem_u32(K_ + (nt * 8 + (lane & 7)) * kStride + ks * 16 + (lane >> 3) * 8);
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_f16_16816(s[nt], qf[ks], b0, b1);
        mma_f16_16816(s[nt], qf[ks + 1], b2, b3);
      }
    }
    // mask, scale, online softmax
    float mblk[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const int key = kstart + nt * 8 + 2 * t4 + (e & 1);
        bool vis = row_ok[hr] && key < c1;
        if (vis && key >= P) vis = anc_has(anc[hr][0], anc[hr][1], key - P);
        const float v = vis ? s[nt][e] * sl2 : -INFINITY;
        s[nt][e] = v;
        mblk[hr] = fmaxf(mblk[hr], v);
      }
    }
    float corr[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      mblk[hr] = fmaxf(mblk[hr], __shfl_xor_sync(0xffffffffu, mblk[hr], 1));
      mblk[hr] = fmaxf(mblk[hr], __shfl_xor_sync(0xffffffffu, mblk[hr], 2));
      const float m_new = fmaxf(m_run[hr], mblk[hr]);
      corr[hr] = (m_run[hr] == -INFINITY) ? 0.f : exp2f(m_run[hr] - m_new);
      m_run[hr] = m_new;
    }
    float lsum[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1;
        const float p = (s[nt][e] == -INFINITY) ? 0.f : exp2f(s[nt][e] - m_run[hr]);
        s[nt][e] = p;
        lsum[hr] += p;
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      lsum[hr] += __shfl_xor_sync(0xffffffffu, lsum[hr], 1);
      lsum[hr] += __shfl_xor_sync(0xffffffffu, lsum[hr], 2);
      l_run[hr] = l_run[hr] * corr[hr] + lsum[hr];
    }
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      o[nd][0] *= corr[0]; o[nd][1] *= corr[0];
      o[nd][2] *= corr[1]; o[nd][3] *= corr[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nd = 0; nd < 16; nd += 2) {
        uint32_t b0, b1, b2, b3;
        const int m = lane >> 3;
        const uint32_t addr =
            smem_u32(V_ + (kk * 16 + (m & 1) * 8 + (lane & 7)) * kStride + (nd + (m >> 1)) * 8);
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_f16_16816(o[nd], pa, b0, b1);
        mma_f16_16816(o[nd + 1], pa, b2, b3);
      }
    }
    __syncthreads();
  }

  // ---- partial output: normalised O and log2-sum-exp per row
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    if (!row_ok[hr]) continue;
    const int qr = row0 + warp * 16 + g + hr * 8;
    const int node = qr / G;
    const int h = kvh * G + (qr - node * G);
    const size_t prow = (size_t)(base + node) * a.Hq + h;
    const bool any = l_run[hr] > 0.f;
    const float inv = any ? 1.f / l_run[hr] : 0.f;
    float* po = a.part_o + (prow * a.n_chunks + blockIdx.x) * hd;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      float2 v = make_float2(o[nd][2 * hr] * inv, o[nd][2 * hr + 1] * inv);
      *reinterpret_cast<float2*>(po + nd * 8 + 2 * t4) = v;
    }
    if (t4 == 0) a.part_lse[prow * a.n_chunks + blockIdx.x] = any ? m_run[hr] + log2f(l_run[hr]) : -INFINITY;
  }

  // ---- signal the nc chunk CTAs of this row block, wait for theirs, then merge
  // this CTA's slice of the rows over all chunks, in chunk order:
  // weights 2^(lse_c - max), output written as split bf16 for the O projection
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    for (int r = 0; r < nc; ++r) mbar_arrive_remote(&donebar, (uint32_t)r);
    s_ok = mbar_wait_cluster(&donebar, 0, sv.err) ? 1 : 0;
  }
  __syncthreads();
  if (!s_ok) return;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
  const int ld = a.Hq * hd;
  const int rows_here = min(kRowsPerCta, rows - row0);
  const int per = (rows_here + nc - 1) / nc;
  const int r_begin = blockIdx.x * per;
  const int r_end = min(rows_here, r_begin + per);
  for (int rr = r_begin + warp; rr < r_end; rr += 4) {
    const int qr = row0 + rr;
    const int node = qr / G;
    const int h = kvh * G + (qr - node * G);
    const size_t prow = (size_t)(base + node) * a.Hq + h;
    const float* lse = a.part_lse + prow * a.n_chunks;
    float mx = -INFINITY;
    for (int c = lane; c < nc; c += 32) mx = fmaxf(mx, __ldcg(lse + c));  // written by peer CTAs
    mx = warp_max(mx);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    for (int c = 0; c < nc; ++c) {
      const float l = __ldcg(lse + c);
      if (l == -INFINITY) continue;
      const float wt = exp2f(l - mx);
      wsum += wt;
      const float4 v = __ldcg(reinterpret_cast<const float4*>(a.part_o + (prow * a.n_chunks + c) * hd + lane * 4));
      acc.x += wt * v.x; acc.y += wt * v.y; acc.z += wt * v.z; acc.w += wt * v.w;
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    const int col = h * hd + lane * 4;
    split_store(out, base + node, ld, col + 0, acc.x * inv);
    split_store(out, base + node, ld, col + 1, acc.y * inv);
    split_store(out, base + node, ld, col + 2, acc.z * inv);
    split_store(out, base + node, ld, col + 3, acc.w * inv);
  }
}

// fp32 path: one warp per (node, head); keys visited in slot order with an
// exact fp32 online softmax.
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

size_t attention_smem_bytes() { return (size_t)(kRowsPerCta + 4 * kKeyBlock) * kStride * sizeof(__half); }

cudaError_t attention_configure() {
  cudaError_t e = cudaFuncSetAttribute(attn_chunk_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)attention_smem_bytes());
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(attn_chunk_f16_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              (int)cudaSharedmemCarveoutMaxShared);
}

cudaError_t launch_attention(int dtype, const AttnArgs& a, cudaStream_t s, bool pdl) {
  if (dtype == 0) {
    const int warps = a.sv.M * a.Hq;
    attn_f32_kernel<<<(warps + 7) / 8, 256, 0, s>>>(a);
    return cudaGetLastError();
  }
  const size_t smem = attention_smem_bytes();
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_chunks, (a.max_rows + kRowsPerCta - 1) / kRowsPerCta, a.sv.B * a.kv.Hkv);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  int na = pdl ? 1 : 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = a.n_chunks;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_chunk_f16_kernel, a);
}

}  // namespace spec
