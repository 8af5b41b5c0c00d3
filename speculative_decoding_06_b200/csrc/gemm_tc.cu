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
// ~16 mantissa bits of the activation instead of 8.  The step is bound by
// streaming the weights once from HBM ("EAGLE-3投机解码：树验证器方法", section
// 问题: decode is memory-bandwidth bound), so the kernel is a persistent,
// warp-specialised weight streamer:
//
//   warp 0      TMA producer: weight tile (128 x 64) + token tile (2*BN x 64) per stage
//   warp 1      MMA issuer: 4 x tcgen05.mma (K = 16 each) per stage into a TMEM
//               accumulator; owns the tensor-memory allocation
//   warps 2-5   epilogue: tcgen05.ld of their 32 accumulator lanes, then the
//               phase's epilogue (QKV, RESID, SWIGLU or ARGMAX, see kernels.h)
//
// One launch runs a list of GEMM phases (for instance O, gate/up, down and the
// next layer's QKV).  Between two phases every CTA of the grid meets at a
// counter (the grid is sized to be co-resident in full).  The producer does not
// stop at that barrier: it keeps streaming the next phase's weight tiles into
// free stages and only holds back their activation tiles until the previous
// phase has completed, so HBM stays busy across phase boundaries.
//
// Two TMEM accumulators alternate so the epilogue of one work unit overlaps
// the main loop of the next.  Split-K phases give every tile S CTAs (one unit
// each, S consecutive CTAs); the S CTAs meet at the tile's arrival counter and
// share its finishing work.  Other phases hand tiles out round-robin.
#include <cuda.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

constexpr int kThreads = 192;
constexpr int kTileO = 128;   // weight rows per tile (MMA M)
constexpr int kTileK = 64;    // K elements per stage (128 bytes of bf16)
constexpr uint32_t kABytes = kTileO * kTileK * 2;

constexpr uint32_t cmax(uint32_t a, uint32_t b) { return a > b ? a : b; }

template <int BN, int STAGES>
struct SmemLayout {
  static constexpr uint32_t kBBytes = 2 * BN * kTileK * 2;  // hi and lo rows
  static constexpr uint32_t a_off = 0;
  static constexpr uint32_t b_off = a_off + STAGES * kABytes;
  static constexpr uint32_t epi_off = b_off + STAGES * kBBytes;
  // per-token norm scale r[BN], then the largest of: SWIGLU gate and up values
  // [128][17] (padded rows: conflict-free), the ARGMAX and TOPK token-major staging
  // [16][136] / [16][129], RESID per-warp sums of squares [4][BN]
  static constexpr uint32_t epi_extra = cmax(cmax(128 * 17 * 4, 16 * 136 * 4), 4 * BN * 4);
  static constexpr uint32_t epi_bytes = BN * 4 + epi_extra;
  static constexpr uint32_t bar_off = (epi_off + epi_bytes + 7) & ~7u;
  static constexpr uint32_t n_bars = 2 * STAGES + 4;
  static constexpr uint32_t misc_off = bar_off + n_bars * 8;
  static constexpr uint32_t total = misc_off + 16;
  static constexpr uint32_t dyn_bytes = total + 1024;  // slack to align the base to 1024
  static constexpr uint32_t acc_cols = 2 * BN;             // one accumulator: hi and lo columns
  // two accumulators, allocated as a power of two of at least 32 columns
  static constexpr uint32_t tmem_cols = 2 * acc_cols <= 256 ? 256u : 512u;
};

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Units of a phase done by CTA b: with split-K one unit (b / S, b % S) if
// b < tiles * S; otherwise tiles b, b + grid, ... (WorkIter walks them)
struct UnitIter {
  int tiles, S, grid, b;
  __device__ int first() const { return S > 1 ? (b < tiles * S ? b / S : tiles) : b; }
  __device__ int split() const { return S > 1 ? b % S : 0; }
};

__device__ __forceinline__ UnitIter units_of(const GemmTcArgs& a) {
  UnitIter it;
  it.tiles = a.tiles_o * a.tiles_t;
  it.S = a.splits;
  it.grid = (int)gridDim.x;
  it.b = (int)blockIdx.x;
  return it;
}

// The work units of a phase that a CTA takes, in order: tile `ut` over k-blocks
// [kb0, kb1).  Plain and split-K phases: UnitIter's tiles over this CTA's split
// range.  Stream-K phases (GemmTcArgs::streamk): the shared tiles' sk_tiles x
// KB k-blocks in tile-major order, cut into one contiguous share per CTA,
// [W b / grid, W (b + 1) / grid) with W = sk_tiles x KB, whose pieces (one per
// tile it touches) are the first units; the CTA holding a tile's first k-block
// finishes the tile, the CTAs whose shares start inside the tile hand it fp32
// partial sums.  Then the remaining tiles, whole, round-robin from sk_tiles + b:
// every CTA streams the same number of weight k-blocks, whatever the tile count.
struct WorkIter {
  int KB, kb0s, kb1s, tiles, grid, S, ut;
  long long g, w1;  // stream-K cursor and end (over the shared tiles' k-blocks)
  bool sk;
  __device__ bool next(int& t, int& k0, int& k1) {
    if (sk) {
      if (g < w1) {
        t = (int)(g / KB);
        k0 = (int)(g - (long long)t * KB);
        k1 = (int)min((long long)KB, k0 + (w1 - g));
        g += k1 - k0;
        return true;
      }
      if (ut >= tiles) return false;  // then whole tiles, round-robin
      t = ut;
      k0 = 0;
      k1 = KB;
      ut += grid;
      return true;
    }
    if (ut >= tiles) return false;
    t = ut;
    k0 = kb0s;
    k1 = kb1s;
    ut = S > 1 ? tiles : ut + grid;
    return true;
  }
};

__device__ __forceinline__ WorkIter work_of(const GemmTcArgs& a) {
  const UnitIter it = units_of(a);
  WorkIter w;
  w.KB = a.K / kTileK;
  w.tiles = it.tiles;
  w.grid = it.grid;
  w.S = it.S;
  w.ut = it.first();
  w.kb0s = it.split() * a.kb_per_split;
  w.kb1s = min(w.kb0s + a.kb_per_split, w.KB);
  w.sk = a.streamk != 0;
  const long long W = (long long)a.sk_tiles * w.KB;
  w.g = W * it.b / it.grid;
  w.w1 = W * (it.b + 1) / it.grid;
  if (w.sk) w.ut = a.sk_tiles + it.b;
  return w;
}

// float -> unsigned key with the same order (for integer warp reductions)
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// (value desc, index asc)
__device__ __forceinline__ bool topk_better(float a, int ai, float b, int bi) {
  return a > b || (a == b && ai < bi);
}

// stream-K: the CTA whose share holds k-block index g of the phase (W in all, over grid CTAs)
__device__ __forceinline__ int sk_cta_of(long long W, long long g, int grid) {
  return (int)(((g + 1) * grid - 1) / W);
}

// Optional timeline: stamp k of phase p of this CTA.  Stamps: 0 producer
// starts the phase, 1 producer may load the phase's activations, 2 producer
// has issued the phase's last load, 3 epilogue starts the phase, 4 first
// accumulator of the phase complete, 5 split-K rendezvous passed, 6 epilogue
// done with the phase's units, 7 phase counted at the grid barrier.
__device__ __forceinline__ void stamp(uint64_t* trace, int p, int k) {
  if (trace) trace[((size_t)blockIdx.x * kMaxGemmPhases + p) * kGemmTraceMarks + k] = global_ns();
}

// hi + lo of the accumulator's tokens c0 .. c0 + 31 (c0 % 32 == 0): split groups
// of 16 tokens (16 hi columns, then 16 lo columns), so the 32 tokens are the 64
// columns from 2 * c0; `two` is false when only tokens c0 .. c0 + 15 exist (the
// last chunk of an 80-token tile)
__device__ __forceinline__ void acc_sums32(uint32_t taddr, int c0, bool two, float* s) {
  static_assert(kSplitGroup == 16, "accumulator column layout");
  uint32_t a[32], b[32];
  tmem_ld32_async(taddr + 2 * c0, a);
  if (two) {
    tmem_ld32_async(taddr + 2 * c0 + 32, b);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) b[i] = 0u;
  }
  tmem_wait_ld();
  tmem_reg_fence32(a);
  tmem_reg_fence32(b);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    s[i] = __uint_as_float(a[i]) + __uint_as_float(a[16 + i]);
    s[16 + i] = __uint_as_float(b[i]) + __uint_as_float(b[16 + i]);
  }
}

__device__ __forceinline__ bool phase_done(const int* bar, int need) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
  return v >= need;
}

}  // namespace

// BN = 64: two CTAs per SM (registers capped accordingly); BN = 128: one
template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, BN == 64 ? 2 : 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmPhases P) {
  using L = SmemLayout<BN, STAGES>;
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
  const int nph = P.n_phases;
  uint32_t* err = P.err;
  const int grid = (int)gridDim.x;

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
    for (int p = 0; p < nph; ++p)
      for (int m = 0; m < 4; ++m) tma_prefetch_desc(&maps.m[4 * p + m]);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Weights never depend on earlier kernels: the producer starts streaming the
  // first stages' weight tiles before waiting for the previous kernel
  // (programmatic dependent launch), and adds the activation tiles afterwards.
  const bool producer = (warp == 0) && elect_one();
  uint64_t pol_w = 0, pol_x = 0;
  auto load_a = [&](int p, uint8_t* sa, uint64_t* bar, int kx, int to) {
    const GemmTcArgs& a = P.ph[p];
    const CUtensorMap* m = &maps.m[4 * p];
    if (P.epi[p] == GEMM_EPI_SWIGLU) {
      tma_load_2d(sa, m + 0, bar, kx, to * 64, pol_w);
      tma_load_2d(sa + kABytes / 2, m + 1, bar, kx, to * 64, pol_w);
    } else {
      const int row = to * kTileO;
      if (row < a.seg_rows[0]) {
        tma_load_2d(sa, m + 0, bar, kx, row, pol_w);
      } else if (row < a.seg_rows[0] + a.seg_rows[1]) {
        tma_load_2d(sa, m + 1, bar, kx, row - a.seg_rows[0], pol_w);
      } else {
        tma_load_2d(sa, m + 2, bar, kx, row - a.seg_rows[0] - a.seg_rows[1], pol_w);
      }
    }
  };
  int pre = 0;  // stages whose weight tile was issued before the wait
  if (producer) {
    pol_w = policy_evict_first();
    pol_x = policy_evict_last();
    WorkIter wi = work_of(P.ph[0]);
    int ut, kb0, kb1;
    if (wi.next(ut, kb0, kb1)) {
      const GemmTcArgs& a = P.ph[0];
      const int to = ut / a.tiles_t;
      pre = min(STAGES, kb1 - kb0);
      for (int s = 0; s < pre; ++s) {
        mbar_arrive_expect_tx(&full[s], kABytes + L::kBBytes);
        load_a(0, smem + L::a_off + s * kABytes, &full[s], (kb0 + s) * kTileK, to);
      }
    }
  }
  // activations written by the previous kernel are read only after this point
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (producer) {
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      // Activation tiles are held back until their producers have finished:
      // phase 0's come from the previous kernel (waited for above), a later
      // phase's from the whole previous phase (its grid-barrier count).
      int pend_stage[STAGES], pend_kx[STAGES], pend_row[STAGES];
      int npend = 0;
      bool first_b = true;
      bool phase_ready = false;
      auto b_ready = [&](int p, int, int) -> bool {
        if (p == 0) return true;
        if (!phase_ready) {
          phase_ready = phase_done(P.phase_bar + p - 1, grid);
          if (phase_ready) fence_proxy_async_global();  // acquired data is read next by TMA
        }
        return phase_ready;
      };
      auto issue_b = [&](int p, int st, int kx, int row) {
        if (first_b) {
          first_b = false;
          stamp(P.trace, p, 1);
        }
        tma_load_2d(smem + L::b_off + st * L::kBBytes, &maps.m[4 * p + 3], &full[st], kx, row, pol_x);
      };
      // issue pending activation loads in k order; `block` waits (bounded) for the first
      auto drain = [&](int p, int tt, bool block) -> bool {
        int done = 0;
        while (done < npend) {
          if (!b_ready(p, pend_kx[done], tt)) {
            if (!block) break;
            const uint64_t t0 = global_ns();
            while (!b_ready(p, pend_kx[done], tt)) {
              if (*abort_flag) return false;
              if (global_ns() - t0 > SPEC_WAIT_NS) {
                set_error(err, SPEC_DEVERR_TIMEOUT);
                *abort_flag = 1;
                return false;
              }
              __nanosleep(32);
            }
          }
          issue_b(p, pend_stage[done], pend_kx[done], pend_row[done]);
          ++done;
        }
        for (int i = done; i < npend; ++i) {
          pend_stage[i - done] = pend_stage[i];
          pend_kx[i - done] = pend_kx[i];
          pend_row[i - done] = pend_row[i];
        }
        npend -= done;
        return true;
      };
      for (int p = 0; p < nph && !*abort_flag; ++p) {
        const GemmTcArgs& a = P.ph[p];
        WorkIter wi = work_of(a);
        int ut, kb0, kb1;
        stamp(P.trace, p, 0);
        first_b = true;
        phase_ready = false;
        while (!*abort_flag && wi.next(ut, kb0, kb1)) {
          const int tt = ut % a.tiles_t;
          const int to = ut / a.tiles_t;
          for (int kb = kb0; kb < kb1 && !*abort_flag; ++kb, ++issued) {
            const int kx = kb * kTileK;
            if (issued >= pre) {
              if (!mbar_wait(&empty[stage], phase ^ 1, err, abort_flag)) break;
              mbar_arrive_expect_tx(&full[stage], kABytes + L::kBBytes);
              load_a(p, smem + L::a_off + stage * kABytes, &full[stage], kx, to);
            }
            pend_stage[npend] = stage;
            pend_kx[npend] = kx;
            pend_row[npend] = tt * 2 * BN;
            ++npend;
            // the ring is full of weight tiles: wait for the oldest activation tile
            if (!drain(p, tt, npend == STAGES)) break;
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          // a unit's activation tiles are all issued before the next unit's
          if (!*abort_flag && npend > 0 && !drain(p, tt, true)) break;
        }
        stamp(P.trace, p, 2);
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
      bool ok = true;
      for (int p = 0; p < nph && ok && !*abort_flag; ++p) {
        WorkIter wi = work_of(P.ph[p]);
        int ut, kb0, kb1;
        for (; ok && !*abort_flag && wi.next(ut, kb0, kb1); ++j) {
          const int acc = j & 1;
          const uint32_t acc_phase = (j >> 1) & 1;
          if (!mbar_wait(&tempty[acc], acc_phase ^ 1, err, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * L::acc_cols;
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(&full[stage], phase, err, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t adesc = sw128_kmajor_desc(smem_u32(smem + L::a_off + stage * kABytes));
            const uint64_t bdesc = sw128_kmajor_desc(smem_u32(smem + L::b_off + stage * L::kBBytes));
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
      }
      if (*abort_flag && last_acc >= 0) mbar_wait(&tfull[last_acc], last_phase, nullptr, nullptr);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int row_in_tile = quarter * 32 + lane;
    const int ep_tid = threadIdx.x - 64;  // 0..127
    const int ep_warp = ep_tid >> 5;
    float* r_s = reinterpret_cast<float*>(smem + L::epi_off);  // [BN]
    uint8_t* epx = smem + L::epi_off + BN * 4;
    int j = 0;
    bool alive = true;
    for (int p = 0; p < nph && alive; ++p) {
      const GemmTcArgs& args = P.ph[p];
      const int EPI = P.epi[p];
      const UnitIter it = units_of(args);
      WorkIter wi = work_of(args);
      const int S = args.splits;
      const int sp = it.split();
      const int KB = args.K / kTileK;
      if (p > 0) {
        // the previous phase wrote this phase's norm statistics and operands
        if (ep_tid == 0) *ep_ok = spin_until_geq(P.phase_bar + p - 1, grid, err) ? 1 : 0;
        named_sync(2, 128);
        if (!*ep_ok) {
          alive = false;
          break;
        }
      }
      if (ep_tid == 0) stamp(P.trace, p, 3);
      bool first_unit = true;
      int ut, kb0, kb1;
      for (; wi.next(ut, kb0, kb1); ++j) {
        const int tt = ut % args.tiles_t;
        const int to = ut / args.tiles_t;
        const int acc = j & 1;
        const uint32_t acc_phase = (j >> 1) & 1;
        const int t_base = tt * BN;
        const int t_end = min(t_base + BN, args.M);
        // per-token scale of the folded RMSNorm (1 when the operand is not normalised)
        for (int c = ep_tid; c < BN; c += 128) {
          const int t = t_base + c;
          float r = 1.f;
          if (args.ss_in && t < args.M) {
            float ssum = 0.f;
            for (int i = 0; i < args.n_ss; ++i) ssum += args.ss_in[(size_t)i * args.ss_ld + t];
            r = rsqrtf(ssum / (float)args.norm_d + args.eps);
          }
          r_s[c] = r;
        }
        // one thread waits, the four epilogue warps then agree on the outcome, so
        // that no warp can be left alone at a named barrier
        if (ep_tid == 0) *ep_ok = mbar_wait(&tfull[acc], acc_phase, err, abort_flag) ? 1 : 0;
        named_sync(2, 128);
        if (!*ep_ok) {
          alive = false;
          break;
        }
        tc_fence_after();
        if (first_unit && ep_tid == 0) stamp(P.trace, p, 4);
        const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * L::acc_cols;

        if (args.streamk && kb0 > 0) {
          // stream-K, a share that starts inside tile ut: its fp32 sums (hi + lo
          // columns) go to this CTA's slot [BN tokens][128 rows] for the CTA that
          // holds the tile's first k-block, which finishes the tile
          float* slot = args.part + (size_t)blockIdx.x * kTileO * BN + row_in_tile;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            float v[32];
            const bool two = c0 + 16 < BN;
            acc_sums32(taddr, c0, two, v);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < 16 || two) __stcg(slot + (size_t)(c0 + i) * kTileO, v[i]);
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
          named_sync(2, 128);  // every thread's stores precede the arrival
          if (ep_tid == 0) red_release_add_gpu(args.counters + ut, 1);
          first_unit = false;
          continue;
        }
        if (args.streamk && kb1 < KB) {
          // stream-K, the tile's first k-blocks, not all of them: the CTAs after this
          // one up to `last` hold the rest (each its share's first unit, which waits
          // on nothing); add their sums to this accumulator's hi columns
          const long long W = (long long)args.sk_tiles * KB;
          const int last = sk_cta_of(W, (long long)ut * KB + KB - 1, grid);
          if (ep_tid == 0) *ep_ok = spin_until_geq(args.counters + ut, last - (int)blockIdx.x, err) ? 1 : 0;
          named_sync(2, 128);
          if (!*ep_ok) {
            alive = false;
            break;
          }
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += kSplitGroup) {
            float vf[kSplitGroup];
            const uint32_t col = (c0 / kSplitGroup) * (2 * kSplitGroup);  // the group's hi columns
            tmem_ld16(taddr + col, vf);
            for (int c = (int)blockIdx.x + 1; c <= last; ++c) {
              const float* slot = args.part + (size_t)c * kTileO * BN + row_in_tile;
#pragma unroll
              for (int i = 0; i < kSplitGroup; ++i) vf[i] += __ldcg(slot + (size_t)(c0 + i) * kTileO);
            }
            uint32_t v[kSplitGroup];
#pragma unroll
            for (int i = 0; i < kSplitGroup; ++i) v[i] = __float_as_uint(vf[i]);
            tmem_st16_async(taddr + col, v);
          }
          tmem_wait_st();
        }

        if (EPI == GEMM_EPI_QKV || EPI == GEMM_EPI_RESID) {
          // 1) this split's partial sums
          const int o = to * kTileO + row_in_tile;
          float* out = args.part + (size_t)sp * args.split_stride + o;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 32) {
            // 32 tokens' hi and lo columns in two loads and one wait
            float v[32];
            const bool two = c0 + 16 < BN;
            acc_sums32(taddr, c0, two, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int t = t_base + c0 + i;
              if ((i < 16 || two) && t < args.M) out[(size_t)t * args.n_out] = v[i];
            }
          }
          if (first_unit && ep_tid == 0) stamp(P.trace, p, 8);
          tc_fence_before();
          mbar_arrive(&tempty[acc]);  // the accumulator is free for the next unit
          // 2) the S split CTAs of the tile meet at its arrival counter, then all of
          //    them share the finishing work, each taking 1/S of the tile's tokens
          int* ctr = args.counters + 2 * ut;
          named_sync(2, 128);
          if (S > 1) {
            if (ep_tid == 0) {
              red_release_add_gpu(ctr, 1);  // the barrier orders every thread's partial stores before it
              *ep_ok = spin_until_geq(ctr, S, err) ? 1 : 0;
            }
            named_sync(2, 128);
            if (!*ep_ok) {
              alive = false;
              break;
            }
          }
          if (first_unit && ep_tid == 0) stamp(P.trace, p, 5);
          const int per = (t_end - t_base + S - 1) / S;
          const int t0s = t_base + sp * per;
          const int t1s = min(t_end, t0s + per);
          const float* part = args.part;
          const size_t sst = args.split_stride;
          if (EPI == GEMM_EPI_QKV) {
            // tile `to` is one head of q|k|v (head_dim 128), rotate-half pairs (c, c+64).
            // lane: 4-column group c4 (columns 4c4.. and 64+4c4..) and one of two
            // tokens; warp: 2 more token lanes -> 8 tokens per pass
            const int hh = to;
            const int c4 = lane & 15;
            const int tl8 = ep_warp * 2 + (lane >> 4);
            const bool is_q = hh < args.Hq;
            const bool rot = hh < args.Hq + args.Hkv;
            const int G = args.Hq / args.Hkv;
            for (int t = t0s + tl8; t < t1s; t += 8) {
              // independent loads: this token's metadata, rotation and all split partials
              const int slot = is_q ? 0 : args.row_slot[t];
              const int sid = is_q ? 0 : args.row_sid[t];
              float4 cs0 = make_float4(1.f, 0.f, 1.f, 0.f), cs1 = cs0;
              if (rot) {
                const float4* csp = reinterpret_cast<const float4*>(args.rope_cs + (size_t)t * 64 + 4 * c4);
                cs0 = csp[0];
                cs1 = csp[1];
              }
              float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bq = a;
              constexpr int kQ = 8;
              for (int q0 = 0; q0 < S; q0 += kQ) {
                float4 pa[kQ], pb[kQ];
#pragma unroll
                for (int qq = 0; qq < kQ; ++qq) {
                  const bool ok = q0 + qq < S;
                  const float4* pr = reinterpret_cast<const float4*>(part + (size_t)(q0 + qq) * sst +
                                                                     (size_t)t * args.n_out + hh * 128 + 4 * c4);
                  pa[qq] = ok ? __ldcg(pr) : make_float4(0.f, 0.f, 0.f, 0.f);
                  pb[qq] = ok ? __ldcg(pr + 16) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int qq = 0; qq < kQ; ++qq) {  // fixed order: deterministic
                  a.x += pa[qq].x; a.y += pa[qq].y; a.z += pa[qq].z; a.w += pa[qq].w;
                  bq.x += pb[qq].x; bq.y += pb[qq].y; bq.z += pb[qq].z; bq.w += pb[qq].w;
                }
              }
              if (first_unit && ep_tid == 0 && t == t0s) stamp(P.trace, p, 9);
              const float r = r_s[t - t_base];
              float x1[4] = {a.x * r, a.y * r, a.z * r, a.w * r};
              float x2[4] = {bq.x * r, bq.y * r, bq.z * r, bq.w * r};
              const float cs[8] = {cs0.x, cs0.y, cs0.z, cs0.w, cs1.x, cs1.y, cs1.z, cs1.w};
              if (rot) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {  // (cos, sin) pairs
                  const float co = cs[2 * i], si = cs[2 * i + 1];
                  const float o1 = x1[i] * co - x2[i] * si;
                  const float o2 = x2[i] * co + x1[i] * si;
                  x1[i] = o1;
                  x2[i] = o2;
                }
              }
              // q and K are stored as two fp16 parts (hi, then lo = the rounding
              // error of hi): the attention scores use both; V keeps one part
              __half* dst = nullptr;
              __half* dst_lo = nullptr;
              if (is_q) {
                dst = args.q_out + ((size_t)(hh / G) * args.q_rows + (size_t)t * G + hh % G) * 128;
                dst_lo = dst + (size_t)args.Hkv * args.q_rows * 128;
              } else if (slot >= 0) {
                const int kvh = rot ? hh - args.Hq : hh - args.Hq - args.Hkv;
                const size_t off = (size_t)sid * args.kv_seq_stride + (size_t)kvh * args.kv_head_stride +
                                   (size_t)slot * 128;
                dst = (rot ? args.k_cache : args.v_cache) + off;
                if (rot) dst_lo = args.klo_cache + off;
              } else if (c4 == 0) {
                set_error(err, SPEC_DEVERR_BOUNDS);
              }
              if (dst) {
                // q and the K/V cache are fp16: a value beyond its range (or NaN) is
                // stored saturated and fails the step instead of turning into inf / NaN
                bool in_range = true;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  in_range = in_range && fabsf(x1[i]) <= 65504.f && fabsf(x2[i]) <= 65504.f;
                  x1[i] = fminf(fmaxf(x1[i], -65504.f), 65504.f);
                  x2[i] = fminf(fmaxf(x2[i], -65504.f), 65504.f);
                }
                if (!in_range) set_error(err, SPEC_DEVERR_RANGE);
                const __half2 h0 = __floats2half2_rn(x1[0], x1[1]), h1 = __floats2half2_rn(x1[2], x1[3]);
                const __half2 h2 = __floats2half2_rn(x2[0], x2[1]), h3 = __floats2half2_rn(x2[2], x2[3]);
                uint2 lo, hi;
                lo.x = *reinterpret_cast<const uint32_t*>(&h0);
                lo.y = *reinterpret_cast<const uint32_t*>(&h1);
                hi.x = *reinterpret_cast<const uint32_t*>(&h2);
                hi.y = *reinterpret_cast<const uint32_t*>(&h3);
                *reinterpret_cast<uint2*>(dst + 4 * c4) = lo;
                *reinterpret_cast<uint2*>(dst + 64 + 4 * c4) = hi;
                if (dst_lo) {
                  const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
                  const float2 f2 = __half22float2(h2), f3 = __half22float2(h3);
                  const __half2 e0 = __floats2half2_rn(x1[0] - f0.x, x1[1] - f0.y);
                  const __half2 e1 = __floats2half2_rn(x1[2] - f1.x, x1[3] - f1.y);
                  const __half2 e2 = __floats2half2_rn(x2[0] - f2.x, x2[1] - f2.y);
                  const __half2 e3 = __floats2half2_rn(x2[2] - f3.x, x2[3] - f3.y);
                  uint2 el, eh;
                  el.x = *reinterpret_cast<const uint32_t*>(&e0);
                  el.y = *reinterpret_cast<const uint32_t*>(&e1);
                  eh.x = *reinterpret_cast<const uint32_t*>(&e2);
                  eh.y = *reinterpret_cast<const uint32_t*>(&e3);
                  *reinterpret_cast<uint2*>(dst_lo + 4 * c4) = el;
                  *reinterpret_cast<uint2*>(dst_lo + 64 + 4 * c4) = eh;
                }
              }
            }
          } else {
            // residual update of this tile's 128 columns for this CTA's tokens, the
            // next operand x*w (split bf16) and per-token sums of squares of x over
            // the tile.  Warp = token (4 per pass), lane = 4 columns.
            const int col = to * kTileO + 4 * lane;
            const float2 w01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(args.norm_w_next + col));
            const float2 w23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(args.norm_w_next + col + 2));
            constexpr int kT = 2;  // tokens per warp and pass
            constexpr int kQ = 8;  // split partials per batch of loads
            for (int tb = t0s + ep_warp; tb < t1s; tb += 4 * kT) {
              float4 xv[kT];
#pragma unroll
              for (int k = 0; k < kT; ++k) {
                const int t = tb + 4 * k;
                xv[k] = t < t1s ? *reinterpret_cast<const float4*>(args.x + (size_t)t * args.n_out + col)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
              }
              for (int q0 = 0; q0 < S; q0 += kQ) {
                float4 pv[kQ][kT];
#pragma unroll
                for (int qq = 0; qq < kQ; ++qq)
#pragma unroll
                  for (int k = 0; k < kT; ++k) {
                    const int t = tb + 4 * k;
                    pv[qq][k] = (t < t1s && q0 + qq < S)
                                    ? __ldcg(reinterpret_cast<const float4*>(part + (size_t)(q0 + qq) * sst +
                                                                             (size_t)t * args.n_out + col))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                  }
#pragma unroll
                for (int qq = 0; qq < kQ; ++qq)  // fixed order: deterministic
#pragma unroll
                  for (int k = 0; k < kT; ++k) {
                    xv[k].x += pv[qq][k].x;
                    xv[k].y += pv[qq][k].y;
                    xv[k].z += pv[qq][k].z;
                    xv[k].w += pv[qq][k].w;
                  }
              }
              if (first_unit && ep_tid == 0 && tb == t0s) stamp(P.trace, p, 9);
#pragma unroll
              for (int k = 0; k < kT; ++k) {
                const int t = tb + 4 * k;
                const float4 v = xv[k];
                const float sq = warp_sum(v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w);
                if (t < t1s) {
                  *reinterpret_cast<float4*>(args.x + (size_t)t * args.n_out + col) = v;
                  split_store4(args.xn_out, t, args.n_out, col, make_float4(v.x * w01.x, v.y * w01.y, v.z * w23.x, v.w * w23.y));
                  if (lane == 0) args.ss_out[(size_t)to * args.ss_ld + t] = sq;
                }
              }
            }
            if (first_unit && ep_tid == 0) stamp(P.trace, p, 10);
          }
        } else if (EPI == GEMM_EPI_SWIGLU) {
          // gate rows 0-63 and up rows 64-127 of the tile meet in shared memory;
          // every thread then finishes 8 of the 16 tokens of one ffn column
          float* stage = reinterpret_cast<float*>(epx);  // [128][17]
          const int fl = ep_tid & 63;
          const int half = ep_tid >> 6;
          const int f = to * 64 + fl;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / kSplitGroup) * (2 * kSplitGroup) + (c0 % kSplitGroup);
            tmem_ld16x2(taddr + col, taddr + col + kSplitGroup, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) stage[row_in_tile * 17 + i] = (v[i] + vl[i]) * r_s[c0 + i];
            named_sync(1, 128);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int ii = half * 8 + i;
              const int t = t_base + c0 + ii;
              const float g = stage[fl * 17 + ii];
              const float up = stage[(64 + fl) * 17 + ii];
              // silu(g) = g / (1 + 2^(-g log2 e)): special-function exp2 and divide
              const float h = __fdividef(g, 1.0f + fast_exp2(-1.4426950408889634f * g)) * up;
              if (t < args.M) split_store(args.out_bf16, t, args.ld_out, f, h);
            }
            named_sync(1, 128);
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        } else if (EPI == GEMM_EPI_STORE) {
          // the accumulator as split bf16 (no split-K): thread = output row, warp
          // stores of one token are 32 consecutive columns
          const int o = to * kTileO + row_in_tile;
          const bool row_ok = o < args.n_out;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / kSplitGroup) * (2 * kSplitGroup) + (c0 % kSplitGroup);
            tmem_ld16x2(taddr + col, taddr + col + kSplitGroup, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int t = t_base + c0 + i;
              if (row_ok && t < args.M) split_store(args.out_bf16, t, args.ld_out, o, (v[i] + vl[i]) * r_s[c0 + i]);
            }
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        } else if (EPI == GEMM_EPI_TOPK) {
          // Per 16 tokens: the tile's 128 x 16 logits go to shared memory token-major;
          // warp w then takes tokens 4w .. 4w + 3 of the 16 side by side, each lane 4
          // of a token's 128 rows (lane + 32u), sorted.  T = the k-th largest of the
          // 32 lane maxima (a bitonic sort across the warp) is a lower bound for the
          // tile's k-th largest value, so the values >= T (a prefix of each lane's
          // four) hold the tile's k best: they become the tile's candidates (at most
          // kCandSlots; ties at T that would overflow them fall back to k rounds of an
          // exact warp-wide selection).  Also the tile's (max, sum of exp(l - max)).
          float* sT = reinterpret_cast<float*>(epx);  // [16][129]
          const int o = to * kTileO + row_in_tile;
          const bool row_ok = o < args.n_out;
          const int K = args.topk;
          const uint32_t lt_mask = (1u << lane) - 1u;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / kSplitGroup) * (2 * kSplitGroup) + (c0 % kSplitGroup);
            tmem_ld16x2(taddr + col, taddr + col + kSplitGroup, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float x = (v[i] + vl[i]) * r_s[c0 + i];
              const int t = t_base + c0 + i;
              if (args.dbg_logits && row_ok && t < args.M) args.dbg_logits[(size_t)t * args.n_out + o] = x;
              sT[i * 129 + row_in_tile] = row_ok ? x : -INFINITY;
            }
            named_sync(1, 128);
            float a[4][4];
            int ai[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int i = ep_warp * 4 + q;
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                a[q][u] = sT[i * 129 + lane + 32 * u];
                const int oo = to * kTileO + lane + 32 * u;
                ai[q][u] = oo < args.n_out ? oo : 0x7fffffff;
              }
            }
            named_sync(1, 128);  // the staging area is free for the next 16 tokens
            auto cx = [&](int q, int x, int y) {
              if (topk_better(a[q][y], ai[q][y], a[q][x], ai[q][x])) {
                const float tv = a[q][x];
                const int ti = ai[q][x];
                a[q][x] = a[q][y];
                ai[q][x] = ai[q][y];
                a[q][y] = tv;
                ai[q][y] = ti;
              }
            };
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              cx(q, 0, 1);
              cx(q, 2, 3);
              cx(q, 0, 2);
              cx(q, 1, 3);
              cx(q, 1, 2);
            }
            // bitonic sort (descending) of the lane maxima: lane r ends with the r-th largest
            float srt[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) srt[q] = a[q][0];
#pragma unroll
            for (int kk = 2; kk <= 32; kk <<= 1)
#pragma unroll
              for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                const bool keep_max = ((lane & jj) == 0) == ((lane & kk) == 0);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const float y = __shfl_xor_sync(0xffffffffu, srt[q], jj);
                  srt[q] = keep_max ? fmaxf(srt[q], y) : fminf(srt[q], y);
                }
              }
            float thr[4], mx[4], se[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              thr[q] = __shfl_sync(0xffffffffu, srt[q], K - 1);
              mx[q] = __shfl_sync(0xffffffffu, srt[q], 0);
              se[q] = 0.f;
              if (mx[q] > -INFINITY) {
#pragma unroll
                for (int u = 0; u < 4; ++u) se[q] += fast_exp2((a[q][u] - mx[q]) * 1.4426950408889634f);
              }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
              for (int q = 0; q < 4; ++q) se[q] += __shfl_xor_sync(0xffffffffu, se[q], off);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int t = t_base + c0 + ep_warp * 4 + q;
              if (t >= args.M) continue;  // (the same for the whole warp)
              const size_t cb = (size_t)t * args.cand_ld + to;
              float* cv = args.cand_v + cb * kCandSlots;
              int32_t* ci = args.cand_i + cb * kCandSlots;
              // candidates: this lane's values >= T, a prefix of its sorted four
              const int c = (a[q][0] >= thr[q]) + (a[q][1] >= thr[q]) + (a[q][2] >= thr[q]) + (a[q][3] >= thr[q]);
              const uint32_t b0 = __ballot_sync(0xffffffffu, c & 1);
              const uint32_t b1 = __ballot_sync(0xffffffffu, c & 2);
              const uint32_t b2 = __ballot_sync(0xffffffffu, c & 4);
              const int tot = __popc(b0) + 2 * __popc(b1) + 4 * __popc(b2);
              if (tot <= kCandSlots) {
                const int pre = __popc(b0 & lt_mask) + 2 * __popc(b1 & lt_mask) + 4 * __popc(b2 & lt_mask);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                  if (u < c) {
                    cv[pre + u] = a[q][u];
                    ci[pre + u] = ai[q][u];
                  }
                if (lane >= tot && lane < kCandSlots) {
                  cv[lane] = -INFINITY;
                  ci[lane] = 0x7fffffff;
                }
              } else {
                // many values tie at T: the k best by k rounds of a warp-wide maximum
                int head = 0;
                float rv = -INFINITY;
                int ri = 0x7fffffff;
                for (int rr = 0; rr < K; ++rr) {
                  const float hv = head == 0 ? a[q][0] : head == 1 ? a[q][1] : head == 2 ? a[q][2]
                                 : head == 3 ? a[q][3] : -INFINITY;
                  const int hi = head == 0 ? ai[q][0] : head == 1 ? ai[q][1] : head == 2 ? ai[q][2]
                               : head == 3 ? ai[q][3] : 0x7fffffff;
                  const uint32_t key = order_key(hv);
                  const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
                  const uint32_t imin = __reduce_min_sync(0xffffffffu, key == kmax ? (uint32_t)hi : 0xffffffffu);
                  const int wl = __ffs(__ballot_sync(0xffffffffu, key == kmax && (uint32_t)hi == imin)) - 1;
                  const float wv = __shfl_sync(0xffffffffu, hv, wl);
                  const int wi = __shfl_sync(0xffffffffu, hi, wl);
                  if (lane == wl) ++head;
                  if (lane == rr) {
                    rv = wv;
                    ri = wi;
                  }
                }
                if (lane < kCandSlots) {
                  cv[lane] = lane < K ? rv : -INFINITY;
                  ci[lane] = lane < K ? ri : 0x7fffffff;
                }
              }
              if (lane == 0) args.cand_lse[cb] = make_float2(mx[q], se[q]);
            }
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        } else {  // GEMM_EPI_ARGMAX
          // Per 16 tokens: the tile's 128 x 16 scores (logits, or logit / T + Gumbel
          // noise) go to shared memory token-major; then eight threads per token take
          // rows p, p + 8, ... (p = 0..7) each, keep their (best, index, runner-up),
          // and meet in three shuffle rounds.  (Rows 136 floats apart: the reads of a
          // warp's 4 tokens x 8 threads hit 32 different banks.)
          float* sT = reinterpret_cast<float*>(epx);  // [16][136]
          const int o = to * kTileO + row_in_tile;
          const bool row_ok = o < args.n_out;
          const int tok = ep_tid >> 3;  // this thread's token of the 16
          const int part = ep_tid & 7;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / kSplitGroup) * (2 * kSplitGroup) + (c0 % kSplitGroup);
            tmem_ld16x2(taddr + col, taddr + col + kSplitGroup, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (v[i] + vl[i]) * r_s[c0 + i];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int t = t_base + c0 + i;
              if (args.dbg_logits && row_ok && t < args.M) args.dbg_logits[(size_t)t * args.n_out + o] = v[i];
              if (args.inv_temp > 0.f && row_ok && t < args.M)  // temperature sampling: Gumbel-max
                v[i] = fmaf(v[i], args.inv_temp,
                            gumbel_noise(args.seed_lo, args.seed_hi, args.row_sid[t], args.row_pos[t], o));
              sT[i * 136 + row_in_tile] = row_ok ? v[i] : -INFINITY;
            }
            named_sync(1, 128);
            Top2 x;
            x.v1 = -INFINITY;
            x.i1 = 0x7fffffff;
            x.v2 = -INFINITY;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              const int r = part + 8 * u;
              const float val = sT[tok * 136 + r];
              const int idx = to * kTileO + r < args.n_out ? to * kTileO + r : 0x7fffffff;
              if (val > x.v1 || (val == x.v1 && idx < x.i1)) {
                x.v2 = x.v1;
                x.v1 = val;
                x.i1 = idx;
              } else {
                x.v2 = fmaxf(x.v2, val);
              }
            }
#pragma unroll
            for (int off = 4; off > 0; off >>= 1) {
              Top2 y;
              y.v1 = __shfl_xor_sync(0xffffffffu, x.v1, off);
              y.i1 = __shfl_xor_sync(0xffffffffu, x.i1, off);
              y.v2 = __shfl_xor_sync(0xffffffffu, x.v2, off);
              x = top2_merge(x, y);
            }
            const int t = t_base + c0 + tok;
            if (part == 0 && t < args.M) args.top_part[(size_t)to * args.top_ld + t] = x;
            named_sync(1, 128);  // the staging area is free for the next 16 tokens
          }
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        }
        // unit done (a phase's arrival counters serve it alone and are zeroed with
        // the step, so nothing is reset here)
        named_sync(2, 128);  // r_s and the staging areas are reused by the next unit
        if (first_unit && ep_tid == 0) stamp(P.trace, p, 11);
        first_unit = false;
      }
      if (!alive) break;
      if (ep_tid == 0) stamp(P.trace, p, 6);
      // this CTA is done with phase p: make its writes visible, then count it
      if (p + 1 < nph) {
        fence_proxy_async_global();  // later phases read this phase's outputs with TMA
        named_sync(2, 128);
        if (ep_tid == 0) red_release_add_gpu(P.phase_bar + p, 1);
      }
      if (ep_tid == 0) stamp(P.trace, p, 7);
    }
  }

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

// BN = 64 tokens: 3 stages of 32 KB (two CTAs per SM); BN = 80: 6 stages of 36 KB, BN = 96: 5
// stages of 40 KB and BN = 128: 4 stages of 48 KB (one CTA per SM).  96 KB of weight tiles are in
// flight per SM at 64 and 80 tokens, 80 KB at 96 and 64 KB at 128.
template <int BN, int STAGES>
static cudaError_t launch_impl(const GemmMultiLaunch& L_, cudaStream_t stream, bool pdl) {
  using L = SmemLayout<BN, STAGES>;
  static_assert(L::dyn_bytes <= 227 * 1024, "shared memory per CTA");
  static_assert(BN % kSplitGroup == 0 && 2 * BN <= 256, "token tile: whole split groups, one TMA box");
  GemmMaps maps;
  GemmPhases ph;
  memset(&maps, 0, sizeof(maps));
  memset(&ph, 0, sizeof(ph));
  ph.n_phases = L_.n_phases;
  ph.phase_bar = L_.phase_bar;
  ph.err = L_.err;
  ph.trace = L_.trace;
  for (int p = 0; p < L_.n_phases; ++p) {
    const GemmPhase& q = L_.ph[p];
    maps.m[4 * p + 0] = *q.mA0;
    maps.m[4 * p + 1] = *(q.mA1 ? q.mA1 : q.mA0);
    maps.m[4 * p + 2] = *(q.mA2 ? q.mA2 : q.mA0);
    maps.m[4 * p + 3] = *q.mB;
    ph.epi[p] = q.epi;
    ph.ph[p] = q.args;
  }
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
  return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, STAGES>, maps, ph);
}

uint32_t gemm_tc_smem_bytes(int bn) {
  return bn == 64   ? SmemLayout<64, 3>::dyn_bytes
         : bn == 80 ? SmemLayout<80, 6>::dyn_bytes
         : bn == 96 ? SmemLayout<96, 5>::dyn_bytes
                    : SmemLayout<128, 4>::dyn_bytes;
}

const void* gemm_tc_function(int bn) {
  return bn == 64   ? (const void*)gemm_tc_kernel<64, 3>
         : bn == 80 ? (const void*)gemm_tc_kernel<80, 6>
         : bn == 96 ? (const void*)gemm_tc_kernel<96, 5>
                    : (const void*)gemm_tc_kernel<128, 4>;
}

cudaError_t gemm_multi_launch(const GemmMultiLaunch& L, cudaStream_t stream, bool pdl) {
  if (L.n_phases < 1 || L.n_phases > kMaxGemmPhases) return cudaErrorInvalidValue;
  if (L.n_phases > 1 && !L.phase_bar) return cudaErrorInvalidValue;
  if (L.bn == 64) return launch_impl<64, 3>(L, stream, pdl);
  if (L.bn == 80) return launch_impl<80, 6>(L, stream, pdl);
  if (L.bn == 96) return launch_impl<96, 5>(L, stream, pdl);
  if (L.bn == 128) return launch_impl<128, 4>(L, stream, pdl);
  return cudaErrorInvalidValue;
}

cudaError_t gemm_tc_launch(const GemmTcLaunch& L, cudaStream_t stream, bool pdl) {
  GemmMultiLaunch m{};
  m.bn = L.bn;
  m.grid = L.grid;
  m.n_phases = 1;
  m.err = L.args.err;
  m.ph[0].epi = L.epi;
  m.ph[0].mA0 = L.mA0;
  m.ph[0].mA1 = L.mA1;
  m.ph[0].mA2 = L.mA2;
  m.ph[0].mB = L.mB;
  m.ph[0].args = L.args;
  return gemm_multi_launch(m, stream, pdl);
}

}  // namespace spec
