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
  // per-token norm scale r[BN], then the largest of: SWIGLU up values [64][17]
  // (padded row: conflict-free), ARGMAX per-warp results [4][BN], RESID per-warp
  // sums of squares [4][BN]
  static constexpr uint32_t epi_extra = cmax(64 * 17 * 4, cmax(4 * BN * (uint32_t)sizeof(Top2), 4 * BN * 4));
  static constexpr uint32_t epi_bytes = BN * 4 + epi_extra;
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

// Units of a phase done by CTA b: with split-K one unit (b / S, b % S) if
// b < tiles * S; otherwise tiles b, b + grid, ...
struct UnitIter {
  int tiles, S, grid, b;
  __device__ int first() const { return S > 1 ? (b < tiles * S ? b / S : tiles) : b; }
  __device__ int next(int ut) const { return S > 1 ? tiles : ut + grid; }
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

// Optional timeline: stamp k of phase p of this CTA.  Stamps: 0 producer
// starts the phase, 1 producer may load the phase's activations, 2 producer
// has issued the phase's last load, 3 epilogue starts the phase, 4 first
// accumulator of the phase complete, 5 split-K rendezvous passed, 6 epilogue
// done with the phase's units, 7 phase counted at the grid barrier.
__device__ __forceinline__ void stamp(uint64_t* trace, int p, int k) {
  if (trace) trace[((size_t)blockIdx.x * kMaxGemmPhases + p) * 8 + k] = global_ns();
}

__device__ __forceinline__ bool phase_done(const int* bar, int need) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
  return v >= need;
}

}  // namespace

template <int BN, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
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
  auto prefetch_a = [&](int p, int kx, int to) {
    const GemmTcArgs& a = P.ph[p];
    const CUtensorMap* m = &maps.m[4 * p];
    if (P.epi[p] == GEMM_EPI_SWIGLU) {
      tma_prefetch_l2_2d(m + 0, kx, to * 64);
      tma_prefetch_l2_2d(m + 1, kx, to * 64);
    } else {
      const int row = to * kTileO;
      if (row < a.seg_rows[0]) tma_prefetch_l2_2d(m + 0, kx, row);
      else if (row < a.seg_rows[0] + a.seg_rows[1]) tma_prefetch_l2_2d(m + 1, kx, row - a.seg_rows[0]);
      else tma_prefetch_l2_2d(m + 2, kx, row - a.seg_rows[0] - a.seg_rows[1]);
    }
  };
  // L2 prefetch of this CTA's first k-blocks of phase p (issued when the
  // producer is done with phase p - 1, so that HBM keeps streaming while the
  // epilogue finishes phase p - 1 and the grid meets at its barrier)
  auto prefetch_phase_l2 = [&](int p) {
    const GemmTcArgs& a = P.ph[p];
    const UnitIter it = units_of(a);
    const int ut = it.first();
    if (ut >= it.tiles) return;
    const int KB = a.K / kTileK;
    const int kb0 = it.split() * a.kb_per_split;
    const int kb1 = min(min(kb0 + a.kb_per_split, KB), kb0 + P.pf_next);
    const int to = ut / a.tiles_t;
    for (int kb = kb0; kb < kb1; ++kb) prefetch_a(p, kb * kTileK, to);
  };
  int pre = 0;  // stages whose weight tile was issued before the wait
  if (producer) {
    pol_w = policy_evict_first();
    pol_x = policy_evict_last();
    const UnitIter it = units_of(P.ph[0]);
    const int ut = it.first();
    if (ut < it.tiles) {
      const GemmTcArgs& a = P.ph[0];
      const int KB = a.K / kTileK;
      const int kb0 = it.split() * a.kb_per_split;
      const int kb1 = min(kb0 + a.kb_per_split, KB);
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
      // activation tiles held back until the previous phase has completed
      int pend_stage[STAGES], pend_kx[STAGES], pend_row[STAGES];
      int npend = 0, pend_p = 0;
      auto flush = [&]() {
        for (int i = 0; i < npend; ++i)
          tma_load_2d(smem + L::b_off + pend_stage[i] * L::kBBytes, &maps.m[4 * pend_p + 3], &full[pend_stage[i]],
                      pend_kx[i], pend_row[i], pol_x);
        npend = 0;
      };
      for (int p = 0; p < nph && !*abort_flag; ++p) {
        const GemmTcArgs& a = P.ph[p];
        const UnitIter it = units_of(a);
        const int KB = a.K / kTileK;
        const int kb0 = it.split() * a.kb_per_split;
        const int kb1 = min(kb0 + a.kb_per_split, KB);
        bool ready = p == 0;  // phase 0's operand is ready: the kernel waited for its predecessor
        stamp(P.trace, p, 0);
        if (ready) stamp(P.trace, p, 1);
        for (int ut = it.first(); ut < it.tiles && !*abort_flag; ut = it.next(ut)) {
          const int tt = ut % a.tiles_t;
          const int to = ut / a.tiles_t;
          for (int kb = kb0; kb < kb1 && !*abort_flag; ++kb, ++issued) {
            const int kx = kb * kTileK;
            if (issued >= pre) {
              if (!mbar_wait(&empty[stage], phase ^ 1, err, abort_flag)) break;
              mbar_arrive_expect_tx(&full[stage], kABytes + L::kBBytes);
              load_a(p, smem + L::a_off + stage * kABytes, &full[stage], kx, to);
            }
            if (P.pf_ahead > 0 && kb + P.pf_ahead < kb1) prefetch_a(p, (kb + P.pf_ahead) * kTileK, to);
            if (!ready) {
              ready = phase_done(P.phase_bar + p - 1, grid);
              if (ready) stamp(P.trace, p, 1);
            }
            if (ready) {
              flush();
              tma_load_2d(smem + L::b_off + stage * L::kBBytes, &maps.m[4 * p + 3], &full[stage], kx, tt * 2 * BN,
                          pol_x);
            } else {
              pend_stage[npend] = stage;
              pend_kx[npend] = kx;
              pend_row[npend] = tt * 2 * BN;
              pend_p = p;
              ++npend;
              if (npend == STAGES) {  // the ring is full of weight tiles: wait for the phase
                if (!spin_until_geq(P.phase_bar + p - 1, grid, err)) {
                  *abort_flag = 1;
                  break;
                }
                ready = true;
                stamp(P.trace, p, 1);
                flush();
              }
            }
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        if (npend > 0 && !*abort_flag) {
          if (spin_until_geq(P.phase_bar + p - 1, grid, err)) {
            stamp(P.trace, p, 1);
            flush();
          } else {
            *abort_flag = 1;
          }
        }
        stamp(P.trace, p, 2);
        if (p + 1 < nph && !*abort_flag) prefetch_phase_l2(p + 1);
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
        const GemmTcArgs& a = P.ph[p];
        const UnitIter it = units_of(a);
        const int KB = a.K / kTileK;
        const int kb0 = it.split() * a.kb_per_split;
        const int kb1 = min(kb0 + a.kb_per_split, KB);
        for (int ut = it.first(); ut < it.tiles && ok && !*abort_flag; ut = it.next(ut), ++j) {
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
      const int S = args.splits;
      const int sp = it.split();
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
      for (int ut = it.first(); ut < it.tiles; ut = it.next(ut), ++j) {
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

        if (EPI == GEMM_EPI_QKV || EPI == GEMM_EPI_RESID) {
          // 1) this split's partial sums
          const int o = to * kTileO + row_in_tile;
          float* out = args.part + (size_t)sp * args.split_stride + o;
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
          tc_fence_before();
          mbar_arrive(&tempty[acc]);  // the accumulator is free for the next unit
          // 2) the S split CTAs of the tile meet at its arrival counter, then all of
          //    them share the finishing work, each taking 1/S of the tile's tokens
          int* ctr = args.counters + 2 * ut;
          __threadfence();
          named_sync(2, 128);
          if (S > 1) {
            if (ep_tid == 0) {
              atomicAdd(ctr, 1);
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
            // tile `to` is one head of q|k|v (head_dim 128): rotate-half pairs (c, c+64)
            const int hh = to;
            const int c = ep_tid & 63;
            const int par = ep_tid >> 6;
            for (int tb = t0s; tb < t1s; tb += 8) {
              float v1[4], v2[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) v1[i] = v2[i] = 0.f;
              for (int q = 0; q < S; ++q) {  // L2 loads: the peers wrote these
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  const int t = tb + 2 * i + par;
                  if (t < t1s) {
                    const float* pr = part + q * sst + (size_t)t * args.n_out + hh * 128 + c;
                    v1[i] += __ldcg(pr);
                    v2[i] += __ldcg(pr + 64);
                  }
                }
              }
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int t = tb + 2 * i + par;
                if (t >= t1s) continue;
                const float r = r_s[t - t_base];
                float a1 = v1[i] * r, a2 = v2[i] * r;
                if (hh < args.Hq + args.Hkv) {
                  const float2 cs = args.rope_cs[(size_t)t * 64 + c];
                  const float o1 = a1 * cs.x - a2 * cs.y;
                  const float o2 = a2 * cs.x + a1 * cs.y;
                  a1 = o1;
                  a2 = o2;
                }
                if (hh < args.Hq) {
                  const int G = args.Hq / args.Hkv;
                  __half* qo = args.q_out + ((size_t)(hh / G) * args.q_rows + (size_t)t * G + hh % G) * 128;
                  qo[c] = __float2half_rn(a1);
                  qo[c + 64] = __float2half_rn(a2);
                } else {
                  const int b = args.row_seq[t];
                  const int slot = args.P_step[b] + args.row_local[t];
                  if (slot < args.max_seq) {
                    const bool is_k = hh < args.Hq + args.Hkv;
                    const int kvh = is_k ? hh - args.Hq : hh - args.Hq - args.Hkv;
                    __half* dst = (is_k ? args.k_cache : args.v_cache) + args.seq_ids[b] * args.kv_seq_stride +
                                  kvh * args.kv_head_stride + (size_t)slot * 128;
                    dst[c] = __float2half_rn(a1);
                    dst[c + 64] = __float2half_rn(a2);
                  } else if (c == 0) {
                    set_error(err, SPEC_DEVERR_BOUNDS);
                  }
                }
              }
            }
          } else {
            // residual update of this tile's 128 columns for this CTA's tokens, the
            // next operand x*w (split bf16) and per-token sums of squares of x
            float* ssw = reinterpret_cast<float*>(epx);  // [4][BN]
            const int col = to * kTileO + ep_tid;
            const float w = __bfloat162float(args.norm_w_next[col]);
            for (int tb = t0s; tb < t1s; tb += 8) {
              float xv[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                xv[i] = (tb + i < t1s) ? args.x[(size_t)(tb + i) * args.n_out + col] : 0.f;
              for (int q = 0; q < S; ++q) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  if (tb + i < t1s) xv[i] += __ldcg(part + q * sst + (size_t)(tb + i) * args.n_out + col);
              }
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const int t = tb + i;
                if (t >= t1s) continue;
                args.x[(size_t)t * args.n_out + col] = xv[i];
                split_store(args.xn_out, t, args.n_out, col, xv[i] * w);
                const float sq = warp_sum(xv[i] * xv[i]);
                if (lane == 0) ssw[ep_warp * BN + (t - t_base)] = sq;
              }
            }
            named_sync(2, 128);
            for (int t = t0s + ep_tid; t < t1s; t += 128) {
              const int c = t - t_base;
              args.ss_out[(size_t)to * args.ss_ld + t] = ssw[c] + ssw[BN + c] + ssw[2 * BN + c] + ssw[3 * BN + c];
            }
          }
          // the last CTA of the tile to leave resets its counters for the next launch
          if (S > 1) {
            named_sync(2, 128);
            if (ep_tid == 0 && atomicAdd(ctr + 1, 1) == S - 1) {
              ctr[0] = 0;
              ctr[1] = 0;
            }
          }
        } else if (EPI == GEMM_EPI_SWIGLU) {
          float* stage_up = reinterpret_cast<float*>(epx);  // [64][17]
          const int f = to * 64 + (row_in_tile & 63);
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / 64) * 128 + (c0 % 64);
            tmem_ld16x2(taddr + col, taddr + col + 64, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (v[i] + vl[i]) * r_s[c0 + i];
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
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
        } else {  // GEMM_EPI_ARGMAX
          Top2* wres = reinterpret_cast<Top2*>(epx);  // [4][BN]
          const int o = to * kTileO + row_in_tile;
          const bool row_ok = o < args.n_out;
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            float v[16], vl[16];
            const uint32_t col = (c0 / 64) * 128 + (c0 % 64);
            tmem_ld16x2(taddr + col, taddr + col + 64, v, vl);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (v[i] + vl[i]) * r_s[c0 + i];
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
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
          named_sync(1, 128);
          for (int c = ep_tid; c < BN; c += 128) {
            Top2 r = wres[c];
#pragma unroll
            for (int q = 1; q < 4; ++q) r = top2_merge(r, wres[q * BN + c]);
            const int t = t_base + c;
            if (t < args.M) args.top_part[(size_t)to * args.top_ld + t] = r;
          }
        }
        named_sync(2, 128);  // r_s and the staging areas are reused by the next unit
        first_unit = false;
      }
      if (!alive) break;
      if (ep_tid == 0) stamp(P.trace, p, 6);
      // this CTA is done with phase p: make its writes visible, then count it
      if (p + 1 < nph) {
        __threadfence();
        named_sync(2, 128);
        if (ep_tid == 0) atomicAdd(P.phase_bar + p, 1);
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

// BN = 64 tokens: 3 stages of 32 KB (two CTAs per SM); BN = 128: 4 stages of 48 KB (one per SM)
template <int BN, int STAGES>
static cudaError_t launch_impl(const GemmMultiLaunch& L_, cudaStream_t stream, bool pdl) {
  using L = SmemLayout<BN, STAGES>;
  GemmMaps maps;
  GemmPhases ph;
  memset(&maps, 0, sizeof(maps));
  memset(&ph, 0, sizeof(ph));
  ph.n_phases = L_.n_phases;
  ph.phase_bar = L_.phase_bar;
  ph.err = L_.err;
  ph.trace = L_.trace;
  ph.pf_next = L_.pf_next;
  ph.pf_ahead = L_.pf_ahead;
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
  return bn == 64 ? SmemLayout<64, 3>::dyn_bytes : SmemLayout<128, 4>::dyn_bytes;
}

const void* gemm_tc_function(int bn) {
  return bn == 64 ? (const void*)gemm_tc_kernel<64, 3> : (const void*)gemm_tc_kernel<128, 4>;
}

cudaError_t gemm_multi_launch(const GemmMultiLaunch& L, cudaStream_t stream, bool pdl) {
  if (L.n_phases < 1 || L.n_phases > kMaxGemmPhases) return cudaErrorInvalidValue;
  if (L.n_phases > 1 && !L.phase_bar) return cudaErrorInvalidValue;
  if (L.bn == 64) return launch_impl<64, 3>(L, stream, pdl);
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
