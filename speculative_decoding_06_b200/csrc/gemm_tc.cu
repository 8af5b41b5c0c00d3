// Small-M bf16 GEMMs of the verification forward on the 5th-generation tensor
// cores (tcgen05 + tensor memory), fed by TMA.
//
//   Y[t][o] = sum_k X[t][k] * W[o][k]     X: activations [tokens][K], W: weights [out][K]
//
// At tree-verification sizes the token count (tree nodes x batch) is small,
// so the weights are put on the MMA's M = 128 side and the tokens on its N
// side: one CTA streams 128 weight rows per tile while the few token rows come
// from L2.  The activations arrive as split bf16 (hi and lo parts, see
// split_row): a tile of BN tokens is a box of 2*BN rows and one MMA of
// N = 2*BN; the epilogue adds the hi and lo columns, so the product carries
// ~16 mantissa bits of the activation instead of 8.  The step is bound by streaming the
// weights once from HBM ("EAGLE-3投机解码：树验证器方法", section 问题: decode
// is memory-bandwidth bound), so the kernel is a persistent, warp-specialised
// weight streamer:
//
//   warp 0      TMA producer: weight tile (128 x 64) + token tile (2*BN x 64) per stage
//   warp 1      MMA issuer: 4 x tcgen05.mma (K = 16 each) per stage into a TMEM
//               accumulator; owns the tensor-memory allocation
//   warps 2-5   epilogue: tcgen05.ld of their 32 accumulator lanes, then one of
//               - PARTIAL: fp32 split-K partial sums  [split][tokens][out]
//               - SWIGLU : tile rows 0-63 are gate rows, 64-127 the matching up rows;
//                          writes silu(gate) * up as split bf16 [tokens][ffn]
//               - ARGMAX : per token, best / index / runner-up over the tile's
//                          128 vocabulary rows (logits never reach HBM)
//
// Two TMEM accumulators alternate so the epilogue of one work unit overlaps
// the main loop of the next.  Work units are (row tile, k split, token tile),
// token tile fastest, handed out round-robin over a grid sized to the number
// of co-resident CTAs.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

constexpr int kThreads = 192;
constexpr int kTileO = 128;   // weight rows per tile (MMA M)
constexpr int kTileK = 64;    // K elements per stage (128 bytes of bf16)
constexpr uint32_t kABytes = kTileO * kTileK * 2;

template <int BN, int STAGES, int EPI>
struct SmemLayout {
  static constexpr uint32_t kBBytes = 2 * BN * kTileK * 2;  // hi and lo rows
  static constexpr uint32_t a_off = 0;
  static constexpr uint32_t b_off = a_off + STAGES * kABytes;
  static constexpr uint32_t epi_off = b_off + STAGES * kBBytes;
  // SWIGLU stages up values [64][17] (padded row: conflict-free); ARGMAX keeps per-warp results [4][BN]
  static constexpr uint32_t epi_bytes =
      EPI == GEMM_EPI_SWIGLU ? 64 * 17 * 4 : (EPI == GEMM_EPI_ARGMAX ? 4 * BN * sizeof(Top2) : 0);
  static constexpr uint32_t bar_off = (epi_off + epi_bytes + 7) & ~7u;
  static constexpr uint32_t n_bars = 2 * STAGES + 4;
  static constexpr uint32_t misc_off = bar_off + n_bars * 8;
  static constexpr uint32_t total = misc_off + 16;
  static constexpr uint32_t dyn_bytes = total + 1024;  // slack to align the base to 1024
  static constexpr uint32_t acc_cols = 2 * BN;             // one accumulator: hi and lo columns
  static constexpr uint32_t tmem_cols = 2 * acc_cols;       // two accumulators
};

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

}  // namespace

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mA0, const __grid_constant__ CUtensorMap mA1,
                   const __grid_constant__ CUtensorMap mA2, const __grid_constant__ CUtensorMap mB,
                   GemmTcArgs args) {
  using L = SmemLayout<BN, STAGES, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = bars + 2 * STAGES + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::misc_off + 4);
  volatile int* ep_ok = reinterpret_cast<volatile int*>(smem + L::misc_off + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int KB = args.K / kTileK;
  const int units = args.tiles_o * args.splits * args.tiles_t;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&mA0);
    tma_prefetch_desc(&mB);
    if (EPI == GEMM_EPI_SWIGLU || args.seg_rows[1] > 0) tma_prefetch_desc(&mA1);
    if (args.seg_rows[2] > 0) tma_prefetch_desc(&mA2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // everything above touched only this CTA's own state; activations written by
  // the previous kernel are read only after this point
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (elect_one()) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int tt = u % args.tiles_t;
        const int rest = u / args.tiles_t;
        const int sp = rest % args.splits;
        const int to = rest / args.splits;
        const int kb0 = sp * args.kb_per_split;
        const int kb1 = min(kb0 + args.kb_per_split, KB);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, args.err, abort_flag)) break;
          uint8_t* sa = smem + L::a_off + stage * kABytes;
          uint8_t* sb = smem + L::b_off + stage * L::kBBytes;
          mbar_arrive_expect_tx(&full[stage], kABytes + L::kBBytes);
          const int kx = kb * kTileK;
          if (EPI == GEMM_EPI_SWIGLU) {
            tma_load_2d(sa, &mA0, &full[stage], kx, to * 64, pol_w);
            tma_load_2d(sa + kABytes / 2, &mA1, &full[stage], kx, to * 64, pol_w);
          } else {
            int row = to * kTileO;
            if (row < args.seg_rows[0]) {
              tma_load_2d(sa, &mA0, &full[stage], kx, row, pol_w);
            } else if (row < args.seg_rows[0] + args.seg_rows[1]) {
              tma_load_2d(sa, &mA1, &full[stage], kx, row - args.seg_rows[0], pol_w);
            } else {
              tma_load_2d(sa, &mA2, &full[stage], kx, row - args.seg_rows[0] - args.seg_rows[1], pol_w);
            }
          }
          tma_load_2d(sb, &mB, &full[stage], kx, tt * 2 * BN, pol_x);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // let copies already issued land before this CTA's shared memory is released
        for (int s = 0; s < STAGES; ++s) {
          int st = (stage + s) % STAGES;
          uint32_t ph = (st < stage) ? phase : (phase ^ 1);
          mbar_wait(&full[st], ph, nullptr, nullptr);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTileO, 2 * BN);
      int stage = 0;
      uint32_t phase = 0;
      int j = 0;
      int last_acc = -1;
      uint32_t last_phase = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x, ++j) {
        const int rest = u / args.tiles_t;
        const int sp = rest % args.splits;
        const int kb0 = sp * args.kb_per_split;
        const int kb1 = min(kb0 + args.kb_per_split, KB);
        const int acc = j & 1;
        const uint32_t acc_phase = (j >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, args.err, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * L::acc_cols;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, args.err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + L::a_off + stage * kABytes);
          const uint32_t b_addr = smem_u32(smem + L::b_off + stage * L::kBBytes);
          const uint64_t adesc = sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sw128_kmajor_desc(b_addr);
#pragma unroll
          for (int k = 0; k < kTileK / 16; ++k) {
            // advance 16 bf16 (32 bytes) along K inside the swizzled rows
            tc_mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
        last_acc = acc;
        last_phase = acc_phase;
      }
      if (*abort_flag && last_acc >= 0) mbar_wait(&tfull[last_acc], last_phase, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int row_in_tile = quarter * 32 + lane;
    const int ep_tid = threadIdx.x - 64;  // 0..127
    int j = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++j) {
      const int tt = u % args.tiles_t;
      const int rest = u / args.tiles_t;
      const int sp = rest % args.splits;
      const int to = rest / args.splits;
      const int acc = j & 1;
      const uint32_t acc_phase = (j >> 1) & 1;
      // one thread waits, the four epilogue warps then agree on the outcome, so
      // that no warp can be left alone at a named barrier
      if (ep_tid == 0) *ep_ok = mbar_wait(&tfull[acc], acc_phase, args.err, abort_flag) ? 1 : 0;
      named_sync(2, 128);
      if (!*ep_ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * L::acc_cols;
      const int t_base = tt * BN;

      if (EPI == GEMM_EPI_PARTIAL) {
        const int o = to * kTileO + row_in_tile;
        float* out = args.out_f32 + (size_t)sp * args.split_stride + o;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16], vl[16];
          const uint32_t col = (c0 / 64) * 128 + (c0 % 64);
          tmem_ld16x2(taddr + col, taddr + col + 64, v, vl);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int t = t_base + c0 + i;
            if (t < args.M) out[(size_t)t * args.n_out] = v[i] + vl[i];
          }
        }
      } else if (EPI == GEMM_EPI_SWIGLU) {
        float* stage_up = reinterpret_cast<float*>(smem + L::epi_off);  // [64][17]
        const int f = to * 64 + (row_in_tile & 63);
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16], vl[16];
          const uint32_t col = (c0 / 64) * 128 + (c0 % 64);
          tmem_ld16x2(taddr + col, taddr + col + 64, v, vl);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += vl[i];
          if (quarter >= 2) {
#pragma unroll
            for (int i = 0; i < 16; ++i) stage_up[(row_in_tile - 64) * 17 + i] = v[i];
          }
          named_sync(1, 128);
          if (quarter < 2) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int t = t_base + c0 + i;
              const float g = v[i];
              const float up = stage_up[row_in_tile * 17 + i];
              const float h = g / (1.0f + expf(-g)) * up;
              if (t < args.M) split_store(args.out_bf16, t, args.ld_out, f, h);
            }
          }
          named_sync(1, 128);
        }
      } else {  // GEMM_EPI_ARGMAX
        Top2* wres = reinterpret_cast<Top2*>(smem + L::epi_off);  // [4][BN]
        const int o = to * kTileO + row_in_tile;
        const bool row_ok = o < args.n_out;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          float v[16], vl[16];
          const uint32_t col = (c0 / 64) * 128 + (c0 % 64);
          tmem_ld16x2(taddr + col, taddr + col + 64, v, vl);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += vl[i];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int t = t_base + c0 + i;
            if (args.dbg_logits && row_ok && t < args.M) args.dbg_logits[(size_t)t * args.n_out + o] = v[i];
            Top2 x;
            x.v1 = row_ok ? v[i] : -INFINITY;
            x.i1 = row_ok ? o : 0x7fffffff;
            x.v2 = -INFINITY;
            x = warp_top2(x);
            if (lane == i) wres[quarter * BN + c0 + i] = x;
          }
        }
        named_sync(1, 128);
        for (int c = ep_tid; c < BN; c += 128) {
          Top2 r = wres[c];
#pragma unroll
          for (int q = 1; q < 4; ++q) r = top2_merge(r, wres[q * BN + c]);
          const int t = t_base + c;
          if (t < args.M) args.top_part[(size_t)to * args.top_ld + t] = r;
        }
        named_sync(1, 128);
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  // let the next kernel in the stream begin its prologue
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// host-side launch helpers
// ---------------------------------------------------------------------------

template <int BN, int STAGES, int EPI>
static cudaError_t launch_impl(const GemmTcLaunch& L_, cudaStream_t stream, bool pdl) {
  using L = SmemLayout<BN, STAGES, EPI>;
  auto kern = gemm_tc_kernel<BN, STAGES, EPI>;  // shared-memory attribute set once by spec_init
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(L_.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L::dyn_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, *L_.mA0, *L_.mA1, *L_.mA2, *L_.mB, L_.args);
}

// BN = 64 tokens: 3 stages of 32 KB (two CTAs per SM); BN = 128: 4 stages of 48 KB (one per SM)

uint32_t gemm_tc_smem_bytes(int bn, int epi) {
  switch (epi) {
    case GEMM_EPI_PARTIAL: return bn == 64 ? SmemLayout<64, 3, GEMM_EPI_PARTIAL>::dyn_bytes : SmemLayout<128, 4, GEMM_EPI_PARTIAL>::dyn_bytes;
    case GEMM_EPI_SWIGLU: return bn == 64 ? SmemLayout<64, 3, GEMM_EPI_SWIGLU>::dyn_bytes : SmemLayout<128, 4, GEMM_EPI_SWIGLU>::dyn_bytes;
    default: return bn == 64 ? SmemLayout<64, 3, GEMM_EPI_ARGMAX>::dyn_bytes : SmemLayout<128, 4, GEMM_EPI_ARGMAX>::dyn_bytes;
  }
}

const void* gemm_tc_function(int bn, int epi) {
  switch (epi) {
    case GEMM_EPI_PARTIAL:
      return bn == 64 ? (const void*)gemm_tc_kernel<64, 3, GEMM_EPI_PARTIAL> : (const void*)gemm_tc_kernel<128, 4, GEMM_EPI_PARTIAL>;
    case GEMM_EPI_SWIGLU:
      return bn == 64 ? (const void*)gemm_tc_kernel<64, 3, GEMM_EPI_SWIGLU> : (const void*)gemm_tc_kernel<128, 4, GEMM_EPI_SWIGLU>;
    default:
      return bn == 64 ? (const void*)gemm_tc_kernel<64, 3, GEMM_EPI_ARGMAX> : (const void*)gemm_tc_kernel<128, 4, GEMM_EPI_ARGMAX>;
  }
}

cudaError_t gemm_tc_launch(const GemmTcLaunch& L, cudaStream_t stream, bool pdl) {
  if (L.bn == 64) {
    switch (L.epi) {
      case GEMM_EPI_PARTIAL: return launch_impl<64, 3, GEMM_EPI_PARTIAL>(L, stream, pdl);
      case GEMM_EPI_SWIGLU: return launch_impl<64, 3, GEMM_EPI_SWIGLU>(L, stream, pdl);
      case GEMM_EPI_ARGMAX: return launch_impl<64, 3, GEMM_EPI_ARGMAX>(L, stream, pdl);
    }
  } else if (L.bn == 128) {
    switch (L.epi) {
      case GEMM_EPI_PARTIAL: return launch_impl<128, 4, GEMM_EPI_PARTIAL>(L, stream, pdl);
      case GEMM_EPI_SWIGLU: return launch_impl<128, 4, GEMM_EPI_SWIGLU>(L, stream, pdl);
      case GEMM_EPI_ARGMAX: return launch_impl<128, 4, GEMM_EPI_ARGMAX>(L, stream, pdl);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace spec
