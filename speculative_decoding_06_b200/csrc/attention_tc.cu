// Tree attention of bf16 models on the 5th-generation tensor cores.
//
// Node i of a tree (local index) sits at cache slot P_b + i and at position
// P_b + depth(i).  A query row sees every prefix key (slots 0 .. P_b-1) and the
// tree keys of its own ancestors, itself included ("EAGLE-3投机解码：
// 树验证器方法", section 树draft vs 链draft).  Grouped-query attention: query
// head h reads key/value head h / (Hq/Hkv).
//
// One CTA handles one (sequence, kv head, tile of 128 query rows, key chunk).
// The query rows of a kv head are its G = Hq/Hkv heads for every tree node
// (row = node * G + g), so one K/V block serves all of them.
//
// Precision: the scores carry ~22 bits.  q and K come in two fp16 parts each
// (hi, and lo = the rounding error of hi; the cache holds K, V and K_lo
// planes), and S = Q_hi K_hi^T + Q_hi K_lo^T + Q_lo K_hi^T accumulates in fp32
// in tensor memory; the probabilities come in two fp16 parts too,
// O += P_hi V + P_lo V, with V single fp16 and O accumulating in fp32.  (With
// one fp16 part for q and K the scores' rounding dominated the logit error of a
// 32-layer model of the 8B shape; P's rounding made a node's logits depend on
// where key chunks start.)
//
//   warp 17 (one thread): TMA loads of Q (hi, lo) and of 64-key blocks of K,
//                        K_lo and V (two K stages and two V stages, each
//                        refilled once its MMAs are done; the later blocks of
//                        the chunk are brought into L2 up front);
//   warp 16 (one thread): the S MMAs of a block into one of two TMEM buffers and
//                        O += P_j V_j into a 128-column TMEM buffer (P_j read
//                        from tensor memory, V from shared memory MN-major);
//   warps 0-15:          four threads per query row (warps w, w + 4, w + 8 and
//                        w + 12 share the row's TMEM lane; each takes 16 of the
//                        block's keys and 32 output dims): read S_j, apply the
//                        ancestor mask and the online softmax (the running max
//                        moves only when a block's max exceeds it by more than
//                        the slack, 8 in log2 units by default: every p stays
//                        <= 2^8 and O is rescaled rarely), write P_j (hi and lo)
//                        into one of two P buffers in tensor memory, and at the
//                        end normalise O.
//
// A sequence's keys are cut into chunks so that short-prefix, small-batch steps
// still occupy the GPU; the chunk CTAs of one (sequence, kv head, row tile)
// are co-resident (the plan keeps the grid within one CTA per SM), publish
// fp32 partials (normalised O and log2-sum-exp) and merge them through global
// memory (a bounded counter, then each CTA merges a slice of the rows) or,
// when every group's cluster fits on the GPU at once, through distributed
// shared memory.  With one chunk the CTA writes its rows directly.  The output
// is split bf16 (hi, lo) for the O-projection GEMM.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace spec {

namespace {

constexpr int kRows = 128;                   // query rows per CTA (the MMA M)
constexpr int kKeys = kAttnTcKeys;           // keys per block (S's N, P.V's K): 64
constexpr int kRowWarps = 16;                // softmax warps: four threads per query row
constexpr int kPerRow = kRowWarps / 4;       // threads of a row (warps w, w + 4, w + 8, w + 12 share its TMEM lane)
constexpr int kKeysPT = 64 / kPerRow;        // keys of a block per thread: 16
constexpr int kDimsPT = 128 / kPerRow;       // output dims per thread: 32
constexpr int kThreads = 32 * (kRowWarps + 2);  // + warp 16: MMA issue, warp 17: TMA loads
constexpr int kCtrlWarp = kRowWarps;
constexpr int kLoadWarp = kRowWarps + 1;
constexpr uint32_t kQHalf = kRows * 128;     // [128 rows][64 fp16] swizzled: 16 KB
constexpr uint32_t kQTile = 2 * kQHalf;      // 128 x 128 fp16: 32 KB
constexpr uint32_t kKHalf = kKeys * 128;     // [64 keys][64 fp16] swizzled: 8 KB
constexpr uint32_t kKTile = 2 * kKHalf;      // 64 x 128 fp16: 16 KB
// a K stage holds, per 64-dim half, K's 64 rows then K_lo's 64 rows: one 128-row
// operand [K; K_lo] per half, so Q_hi [K; K_lo]^T is one N = 128 product
constexpr uint32_t kKStage = 2 * kKTile;     // 32 KB
static_assert(kKeys == 64, "a P row is one 128-byte swizzled row; two 32-key pieces per block");

// K and V stages are filled and released separately: a K stage is free once the
// scores that read it are done, a V stage once P.V is
enum { B_QFULL = 0, B_KFULL = 1, B_VFULL = 3, B_KEMPTY = 5, B_VEMPTY = 7, B_SFULL = 9, B_SFREE = 11, B_PFULL = 13,
       B_PEMPTY = 15, B_OFULL = 17, B_DRAIN = 18, kNumBars = 19 };

struct Smem {
  static constexpr uint32_t q = 0;                   // Q hi
  static constexpr uint32_t qlo = q + kQTile;        // Q lo
  static constexpr uint32_t k = qlo + kQTile;        // 2 stages of [K; K_lo]; 64 KB of output staging at the end
  static constexpr uint32_t v = k + 2 * kKStage;     // 2 stages
  static constexpr uint32_t xchg = v + 2 * kKTile;   // row maxima [2][kPerRow][128] and sums [kPerRow][128]
  static constexpr uint32_t lse = xchg + 3 * kPerRow * 128 * 4; // this chunk's log2-sum-exp per row (cluster merge)
  static constexpr uint32_t bars = lse + 128 * 4;
  static constexpr uint32_t misc = bars + kNumBars * 8;  // tmem slot, abort flag, merge flag
  static constexpr uint32_t end = misc + 16;
  static constexpr uint32_t dyn = end + 1024;            // 1024-byte alignment slack
};
static_assert(Smem::dyn <= 227 * 1024, "shared memory");

// tensor-memory columns: two S buffers of 128 (keys 0-63: Q_hi K^T + Q_lo K^T, 64-127:
// Q_hi K_lo^T, added by the softmax) at 0 and 128, O at 256, and two P buffers of 64
// at 384 and 448: the P.V MMAs' A operand (P_hi in 32 columns, then P_lo; two fp16 keys
// per 32-bit column, the even key in the low half)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCols = 2 * kKeys;
constexpr uint32_t kColO = 2 * kSCols;
constexpr uint32_t kColP = kColO + 128;
constexpr uint32_t kPCols = kKeys;  // one buffer: 32 columns of P_hi, 32 of P_lo
static_assert(kColP + 2 * kPCols <= kTmemCols, "tensor memory");
static_assert(Smem::v - Smem::k >= 128 * 512, "output staging (128 rows x 512 B) fits in the K ring");

// fp16 A and B, f32 D, M = 128; S: N = 128 ([K; K_lo]) and N = 64 (K); P.V: N = 128 dims, B MN-major (bit 16)
constexpr uint32_t kIdescS = (1u << 4) | ((uint32_t)(kKeys >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
constexpr uint32_t kIdescS2 = (1u << 4) | ((uint32_t)(2 * kKeys >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
constexpr uint32_t kIdescPV = (1u << 4) | (1u << 16) | ((uint32_t)(128 >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);

// MN-major operand with the 128-byte swizzle: 64 fp16 along N per 128-byte row,
// 8-row (K) groups 1024 B apart (stride byte offset), N atoms `lbo` bytes apart
// (leading byte offset).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// optional timeline: trace[cta][k] = %globaltimer at mark k (thread 0 of the
// softmax warps, or the issuing thread for marks 1, 2, 11, 12)
constexpr int kTraceMarks = 16;
__device__ __forceinline__ void stamp_at(uint64_t* trace, int k) {
  if (!trace) return;
  const unsigned cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
  if (cta < (unsigned)kAttnPartCtas) trace[cta * kTraceMarks + k] = global_ns();
}

__device__ __forceinline__ void named_sync_rows() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kRowWarps) : "memory"); }
// the kPerRow warps whose threads share TMEM lanes 32 q .. 32 q + 31 (warps q, q + 4, ...)
__device__ __forceinline__ void named_sync_quad(int q) {
  asm volatile("bar.sync %0, %1;" ::"r"(2 + q), "n"(32 * kPerRow) : "memory");
}




// Bits j = 0..31 of the 128-bit ancestor set (a1:a0) starting at bit s, with
// zeros for bit positions outside [0, 128); s in [-31, 127].
__device__ __forceinline__ uint32_t anc_window(uint64_t a0, uint64_t a1, int s) {
  if (s < 0) return (uint32_t)(a0 << (-s));
  const uint64_t lo = s < 64 ? a0 : a1;
  const uint64_t hi = s < 64 ? a1 : 0ull;
  const int sh = s & 63;
  return (uint32_t)(sh ? (lo >> sh) | (hi << (64 - sh)) : lo);
}

// Visible keys among key0 .. key0+31 for one query row: keys below c1, and
// either prefix keys (below P) or tree keys whose node is an ancestor of the
// row's node (bit key - P of the ancestor set).
__device__ __forceinline__ uint32_t visible_word(int key0, int P, int c1, uint64_t a0, uint64_t a1) {
  const int nv = c1 - key0;
  const uint32_t lim = nv >= 32 ? 0xffffffffu : (nv <= 0 ? 0u : (1u << nv) - 1u);
  const int np = P - key0;
  const uint32_t pre = np >= 32 ? 0xffffffffu : (np <= 0 ? 0u : (1u << np) - 1u);
  const int s = key0 - P;
  const uint32_t tree = (s <= -32 || s >= 128) ? 0u : anc_window(a0, a1, s);
  return lim & (pre | tree);
}

// Partial / output staging in shared memory: 128 rows x 32 float4 chunks,
// chunk k of row r at position k ^ (r & 7) within its group of eight, so that
// per-row writes by 32 threads and per-row reads by one warp are both free of
// bank conflicts.
__device__ __forceinline__ float4* stage_at(uint8_t* base, int r, int k) {
  return reinterpret_cast<float4*>(base) + r * 32 + (k ^ (r & 7));
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ AttnTcMaps maps, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Smem::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Smem::misc + 4);
  volatile int* merge_ok = reinterpret_cast<volatile int*>(smem + Smem::misc + 8);

  // The step's row metadata was written kernels ago (every kernel in between
  // waited for its predecessor), so it may be read before this launch waits for
  // the previous kernel; q, the tree's K/V and every output come after the wait.
  const StepView& sv = a.sv;
  const int Hkv = a.kv.Hkv;
  const int G = a.Hq / Hkv;
  const int bk = blockIdx.z;
  const int bi = bk / Hkv;  // position in the work order (longest sequences first)
  const int kvh = bk - bi * Hkv;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (bi >= sv.B) {
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int b = sv.order ? sv.order[bi] : bi;
  const int base = sv.node_off[b];
  const int n_b = sv.node_off[b + 1] - base;
  const int rows = n_b * G;
  const int row0 = blockIdx.y * kRows;
  const int P = sv.P_step[b];
  const int Lk = P + n_b;
  const int c0 = blockIdx.x * a.chunk;
  // (cluster merge: a chunk CTA beyond this sequence's keys stays in its
  // cluster with an empty partial; the whole cluster shares b and row0)
  const bool idle = c0 >= Lk;
  if (row0 >= rows || (idle && !a.cluster_merge)) {  // nothing here: no partial, no arrival
    pdl_wait();
    pdl_launch_dependents();
    return;
  }
  const int c1 = idle ? c0 : min(c0 + a.chunk, Lk);
  const int nc_b = (Lk + a.chunk - 1) / a.chunk;  // chunk CTAs of this sequence
  const int nb = (c1 - c0 + kKeys - 1) / kKeys;   // 0 when idle
  const int seq = sv.seq_ids[b];
  uint32_t* err = sv.err;
  auto stamp = [&](uint64_t* trace, int k) {
    if (tid == 0) stamp_at(trace, k);
  };
  stamp(a.trace, 0);

  if (warp == kCtrlWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar[B_QFULL], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_KFULL + s], 1);
      mbar_init(&bar[B_VFULL + s], 1);
      mbar_init(&bar[B_KEMPTY + s], 1);
      mbar_init(&bar[B_VEMPTY + s], 1);
      mbar_init(&bar[B_SFULL + s], 1);
      mbar_init(&bar[B_SFREE + s], kRowWarps);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar[B_PFULL + s], kRowWarps);
      mbar_init(&bar[B_PEMPTY + s], 1);
    }
    mbar_init(&bar[B_OFULL], 1);
    mbar_init(&bar[B_DRAIN], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ TMA loads
    if (nb == 0) {
      pdl_wait();
      pdl_launch_dependents();
    } else if (elect_one()) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.kv);
      // cache rows: [layer][K | V | K_lo][max_batch][Hkv][max_seq]
      const int planes = a.kv.planes;
      const int krow = (((a.layer * planes + 0) * a.kv.max_batch + seq) * Hkv + kvh) * a.kv.max_seq;
      const int vrow = (((a.layer * planes + 1) * a.kv.max_batch + seq) * Hkv + kvh) * a.kv.max_seq;
      const int klrow = (((a.layer * planes + 2) * a.kv.max_batch + seq) * Hkv + kvh) * a.kv.max_seq;
      const int qrow = kvh * a.q_rows + base * G + row0;
      const int qlrow = qrow + Hkv * a.q_rows;  // the lo part follows all kv heads' hi parts
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol = policy_evict_normal();  // the other row tiles read the same K/V blocks
      int kloaded = 0, vloaded = 0;  // blocks whose K (K_lo) / V copies were issued
      auto load_k = [&](int j) {
        const int st = j & 1;
        const int key = c0 + j * kKeys;
        uint8_t* sk = smem + Smem::k + st * kKStage;
        mbar_arrive_expect_tx(&bar[B_KFULL + st], 2 * kKTile);
        tma_load_2d(sk, &maps.kv, &bar[B_KFULL + st], 0, krow + key, pol);
        tma_load_2d(sk + kKHalf, &maps.kv, &bar[B_KFULL + st], 0, klrow + key, pol);
        tma_load_2d(sk + kKTile, &maps.kv, &bar[B_KFULL + st], 64, krow + key, pol);
        tma_load_2d(sk + kKTile + kKHalf, &maps.kv, &bar[B_KFULL + st], 64, klrow + key, pol);
        kloaded = j + 1;
      };
      auto load_v = [&](int j) {
        const int st = j & 1;
        const int key = c0 + j * kKeys;
        uint8_t* svb = smem + Smem::v + st * kKTile;
        mbar_arrive_expect_tx(&bar[B_VFULL + st], kKTile);
        tma_load_2d(svb, &maps.kv, &bar[B_VFULL + st], 0, vrow + key, pol);
        tma_load_2d(svb + kKHalf, &maps.kv, &bar[B_VFULL + st], 64, vrow + key, pol);
        vloaded = j + 1;
      };
      // the blocks beyond the two stages go into L2 now, so that their copies into
      // shared memory later wait on L2 rather than on HBM
      auto prefetch_kv = [&](int j) {
        const int key = c0 + j * kKeys;
        tma_prefetch_l2_2d(&maps.kv, 0, krow + key);
        tma_prefetch_l2_2d(&maps.kv, 64, krow + key);
        tma_prefetch_l2_2d(&maps.kv, 0, klrow + key);
        tma_prefetch_l2_2d(&maps.kv, 64, klrow + key);
        tma_prefetch_l2_2d(&maps.kv, 0, vrow + key);
        tma_prefetch_l2_2d(&maps.kv, 64, vrow + key);
      };
      // blocks made only of prefix keys were written by earlier steps: load
      // them before waiting for the previous kernel
      const int first = min(nb, 2);
      int pre = 0;
      while (pre < first && c0 + (pre + 1) * kKeys <= P) {
        load_k(pre);
        load_v(pre);
        ++pre;
      }
      int pf = first;
      while (pf < nb && c0 + (pf + 1) * kKeys <= P) prefetch_kv(pf++);
      pdl_wait();
      pdl_launch_dependents();
      mbar_arrive_expect_tx(&bar[B_QFULL], 2 * kQTile);
      tma_load_2d(smem + Smem::q, &maps.q, &bar[B_QFULL], 0, qrow, pol_q);
      tma_load_2d(smem + Smem::q + kQHalf, &maps.q, &bar[B_QFULL], 64, qrow, pol_q);
      tma_load_2d(smem + Smem::qlo, &maps.q, &bar[B_QFULL], 0, qlrow, pol_q);
      tma_load_2d(smem + Smem::qlo + kQHalf, &maps.q, &bar[B_QFULL], 64, qlrow, pol_q);
      for (int j = pre; j < first; ++j) {
        load_k(j);
        load_v(j);
      }
      while (pf < nb) prefetch_kv(pf++);
      // block j >= 2 into the stages of block j - 2: K once its scores are done,
      // V once its P.V is done (the MMA issuer commits both)
      bool ok = true;
      for (int j = 2; j < nb && ok; ++j) {
        ok = mbar_wait(&bar[B_KEMPTY + (j & 1)], ((j - 2) >> 1) & 1, err, abort_flag);
        if (ok) load_k(j);
        if (ok) ok = mbar_wait(&bar[B_VEMPTY + (j & 1)], ((j - 2) >> 1) & 1, err, abort_flag);
        if (ok) load_v(j);
      }
      if (!ok) {
        *abort_flag = 1;
        // let this thread's copies land before the CTA's shared memory is released:
        // only the last copy into each stage can be outstanding (an earlier one was
        // consumed before the stage was refilled)
        for (int j = max(0, kloaded - 2); j < kloaded; ++j)
          mbar_wait(&bar[B_KFULL + (j & 1)], (j >> 1) & 1, nullptr, nullptr);
        for (int j = max(0, vloaded - 2); j < vloaded; ++j)
          mbar_wait(&bar[B_VFULL + (j & 1)], (j >> 1) & 1, nullptr, nullptr);
      }
    } else {
      pdl_wait();
      pdl_launch_dependents();
    }
    __syncwarp();
  } else if (warp == kCtrlWarp) {
    // ------------------------------------------------------------ MMA issue
    if (nb == 0) {
      pdl_wait();
      pdl_launch_dependents();
    } else if (elect_one()) {
      pdl_wait();
      pdl_launch_dependents();
      const uint32_t sq = smem_u32(smem + Smem::q);
      const uint32_t sql = smem_u32(smem + Smem::qlo);
      auto issue_pv = [&](int j) {
        const uint32_t svv = smem_u32(smem + Smem::v + (j & 1) * kKTile);
#pragma unroll
        for (int kk = 0; kk < kKeys / 16; ++kk) {
          // P: one 128-byte row of 64 keys per query row; V: 16 keys (rows) per step,
          // its two 64-dim halves kKHalf apart (the N atoms of the MN-major operand)
          const uint64_t bd = sw128_mnmajor_desc(svv + kk * 16 * 128, kKHalf);
          const uint32_t pa = tmem + kColP + (j & 1) * kPCols + kk * 8;  // 16 keys: 8 columns
          tc_mma_ts(tmem + kColO, pa, bd, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
          tc_mma_ts(tmem + kColO, pa + kPCols / 2, bd, kIdescPV, 1u);
        }
      };
      // P.V of block j (its P written, its V landed)
      auto pv_step = [&](int j) -> bool {
        if (!mbar_wait(&bar[B_PFULL + (j & 1)], (j >> 1) & 1, err, abort_flag)) return false;
        if (!mbar_wait(&bar[B_VFULL + (j & 1)], (j >> 1) & 1, err, abort_flag)) return false;
        tc_fence_after();
        issue_pv(j);
        tc_commit(&bar[B_PEMPTY + (j & 1)]);
        tc_commit(&bar[B_VEMPTY + (j & 1)]);
        return true;
      };
      bool ok = mbar_wait(&bar[B_QFULL], 0, err, abort_flag);
      stamp_at(a.trace, 1);
      for (int j = 0; j < nb && ok; ++j) {
        const int st = j & 1;
        ok = mbar_wait(&bar[B_KFULL + st], (j >> 1) & 1, err, abort_flag);
        if (!ok) break;
        if (j == 0) stamp_at(a.trace, 2);
        if (j >= 2) ok = mbar_wait(&bar[B_SFREE + st], ((j - 2) >> 1) & 1, err, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t sk = smem_u32(smem + Smem::k + st * kKStage);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // 16 head dims per step
          const uint32_t oq = (ks >> 2) * kQHalf + (ks & 3) * 32;
          const uint32_t okey = (ks >> 2) * kKTile + (ks & 3) * 32;  // [K; K_lo] rows of this dim half
          const uint64_t dk2 = sw128_kmajor_desc(sk + okey);         // N = 128: K then K_lo
          tc_mma_bf16(tmem + st * kSCols, sw128_kmajor_desc(sq + oq), dk2, kIdescS2, ks > 0 ? 1u : 0u);
          tc_mma_bf16(tmem + st * kSCols, sw128_kmajor_desc(sql + oq), dk2, kIdescS, 1u);  // N = 64: K only
        }
        tc_commit(&bar[B_SFULL + st]);
        tc_commit(&bar[B_KEMPTY + st]);
        if (j == 0) stamp_at(a.trace, 11);
        if (j >= 1) ok = pv_step(j - 1);
      }
      stamp_at(a.trace, 12);
      if (ok && nb > 0) ok = pv_step(nb - 1);
      if (ok) {
        tc_commit(&bar[B_OFULL]);
      } else {
        *abort_flag = 1;
        // let issued MMAs finish before the CTA's memory is released
        tc_commit(&bar[B_DRAIN]);
        mbar_wait(&bar[B_DRAIN], 0, nullptr, nullptr);
      }
    } else {
      pdl_wait();
      pdl_launch_dependents();
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax rows
    // Four threads per query row: warps w, w + 4, w + 8 and w + 12 read the same
    // TMEM lanes; quarter q = warp / 4 takes keys 16q .. 16q + 15 of every block
    // and output dims 32q .. 32q + 31, and the four exchange row maxima and sums
    // through shared memory.  Every thread passes every named barrier, also after
    // a failed wait (its work is then skipped), so no barrier is left short.
    pdl_wait();
    pdl_launch_dependents();
    const int qtr = warp >> 2;
    const int r = (warp & 3) * 32 + lane;
    const int qr = row0 + r;
    const bool row_ok = qr < rows;
    const int node = row_ok ? qr / G : 0;
    const uint64_t anc0 = sv.row_anc[2 * (base + node)];
    const uint64_t anc1 = sv.row_anc[2 * (base + node) + 1];
    const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's TMEM lanes
    const float sl2 = 1.4426950408889634f * 0.08838834764831845f;      // log2(e) / sqrt(128)
    float* xmax = reinterpret_cast<float*>(smem + Smem::xchg);           // [parity][quarter][row]
    float* xsum = xmax + 2 * kPerRow * 128;                              // [quarter][row]
    const uint32_t kmask = (1u << kKeysPT) - 1u;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nb; ++j) {
      const int st = j & 1;
      const int key0 = c0 + j * kKeys;
      const uint32_t ts = tl + st * kSCols + qtr * kKeysPT;  // this thread's keys of S (+ kKeys: the K_lo part)
      if (ok) ok = mbar_wait(&bar[B_SFULL + st], (j >> 1) & 1, err, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (j == 0) stamp(a.trace, 3);
      // a block of prefix keys of this chunk is visible to every row of the warp
      const bool wfull = __all_sync(0xffffffffu, row_ok && key0 + kKeys <= min(P, c1));
      // pass 1: this thread's scores (hidden keys set to -inf, so that pass 2 needs
      // no mask) and their max (raw scores; the scale is positive), then the row's
      float x[kKeysPT];
      if (ok) {
        tc_fence_after();
        float xl[kKeysPT];
        tmem_ld16x2(ts, ts + kKeys, x, xl);
#pragma unroll
        for (int c = 0; c < kKeysPT; c += 2)
          f2_unpack(f2_add(f2_pack(x[c], x[c + 1]), f2_pack(xl[c], xl[c + 1])), x[c], x[c + 1]);
        if (!wfull) {
          const uint32_t w = row_ok ? visible_word(key0 + kKeysPT * qtr, P, c1, anc0, anc1) & kmask : 0u;
#pragma unroll
          for (int c = 0; c < kKeysPT; ++c) x[c] = ((w >> c) & 1u) ? x[c] : -INFINITY;
        }
      } else {
#pragma unroll
        for (int c = 0; c < kKeysPT; ++c) x[c] = -INFINITY;
      }
      static_assert(kKeysPT == 16, "max tree over 16 scores");
      xmax[(st * kPerRow + qtr) * 128 + r] =
          fmaxf(fmax3(fmax3(x[0], x[1], x[2]), fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[8])),
                fmax3(fmax3(x[9], x[10], x[11]), fmax3(x[12], x[13], x[14]), x[15]));
      named_sync_quad(warp & 3);  // the four warps that share these rows
      float mraw = xmax[(st * kPerRow) * 128 + r];
#pragma unroll
      for (int q = 1; q < kPerRow; ++q) mraw = fmaxf(mraw, xmax[(st * kPerRow + q) * 128 + r]);
      const float mblk = mraw * sl2;
      if (j == 0) stamp(a.trace, 8);
      float corr = 1.f;
      if (mblk > m + a.rescale_slack) {
        corr = fast_exp2(m - mblk);  // 0 while nothing was visible
        m = mblk;
      }
      const float nm = (m == -INFINITY) ? 0.f : -m;
      // pass 2: P = 2^(s - m) as two fp16 parts, in registers until the P buffer is
      // free (2^-inf = 0 for hidden keys; the scale and the sums go two keys at a time)
      const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(nm, nm);
      const uint64_t dn2 = f2_pack(0x1p-112f, 0x1p-112f), up2 = f2_pack(0x1p112f, 0x1p112f);
      uint64_t lsa = f2_pack(0.f, 0.f), lsb = lsa;
      uint32_t pk[kKeysPT / 2], pl[kKeysPT / 2];
#pragma unroll
      for (int c = 0; c < kKeysPT / 2; ++c) {
        float y0, y1;
        f2_unpack(f2_fma(f2_pack(x[2 * c], x[2 * c + 1]), sc2, nm2), y0, y1);
        const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
        const uint64_t p2 = f2_pack(p0, p1);
        if (c & 1) lsb = f2_add(lsb, p2);
        else lsa = f2_add(lsa, p2);
        // hi: p truncated to fp16's 11 significant bits, formed without a conversion:
        // p * 2^-112 carries fp16's exponent bias (127 - 112 = 15), so its bits 13-27
        // are the fp16 bits (p < 2^-14, below fp16's normal range, flushes to zero and
        // goes wholly into lo); lo: the exact remainder p - hi, rounded to fp16
        uint32_t u0, u1;
        u2_unpack(f2_mul_ftz(p2, dn2), u0, u1);
        u0 &= 0xFFFFE000u;
        u1 &= 0xFFFFE000u;
        pk[c] = (u0 >> 13) | (u1 << 3);
        float d0, d1;
        f2_unpack(f2_sub(p2, f2_mul(u2_pack(u0, u1), up2)), d0, d1);
        const __half2 l2 = __floats2half2_rn(d0, d1);
        pl[c] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      float la0, la1;
      f2_unpack(f2_add(lsa, lsb), la0, la1);
      // a larger running max rescales O: P.V of block j - 1 must have finished
      if (j >= 1 && ok && __any_sync(0xffffffffu, corr != 1.f)) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bar[B_PEMPTY + ((j - 1) & 1)], ((j - 1) >> 1) & 1, err, abort_flag));
        if (ok) {
          tc_fence_after();
          {
            uint32_t o[32];
            const uint32_t to_ = tl + kColO + qtr * kDimsPT;
            tmem_ld32_async(to_, o);
            tmem_wait_ld();
            tmem_reg_fence32(o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * corr);
            tmem_st32_async(to_, o);
            tmem_wait_st();
          }
        }
      }
      // P buffer j & 1 is free once P.V of block j - 2 has finished
      if (j >= 2 && ok) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar[B_PEMPTY + (j & 1)], ((j - 2) >> 1) & 1, err, abort_flag));
        if (ok) tc_fence_after();
      }
      // this thread's 16 keys: 8 columns of P_hi and 8 of P_lo in its TMEM lane
      if (ok) {
        const uint32_t tp = tl + kColP + (j & 1) * kPCols + qtr * (kKeysPT / 2);
        tmem_st8_async(tp, pk);
        tmem_st8_async(tp + kPCols / 2, pl);
        tmem_wait_st();
        if (j == 0) stamp(a.trace, 9);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar[B_SFREE + st]);
          mbar_arrive(&bar[B_PFULL + (j & 1)]);
        }
      }
      l = l * corr + (la0 + la1);
    }
    if (!ok) *abort_flag = 1;
    // ---- normalised output of this chunk, staged in shared memory (the K/V
    // ring is idle once the last P.V has completed)
    if (ok && nb > 0) ok = mbar_wait(&bar[B_OFULL], 0, err, abort_flag);  // (an idle CTA issued no MMA)
    ok = __all_sync(0xffffffffu, ok);
    stamp(a.trace, 4);
    xsum[qtr * 128 + r] = l;
    named_sync_rows();
    float lt = 0.f;
#pragma unroll
    for (int q = 0; q < kPerRow; ++q) lt += xsum[q * 128 + r];
    const bool any = lt > 0.f;
    const float inv = any ? 1.f / lt : 0.f;
    uint8_t* stg = smem + Smem::k;  // 128 rows x 512 B
    if (ok && nb > 0) {
      tc_fence_after();
      uint32_t o[32];
      tmem_ld32_async(tl + kColO + qtr * kDimsPT, o);
      tmem_wait_ld();
      tmem_reg_fence32(o);
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4)
        *stage_at(stg, r, qtr * 8 + q4) =
            make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                        __uint_as_float(o[4 * q4 + 2]) * inv, __uint_as_float(o[4 * q4 + 3]) * inv);
    }
    const int grp = (b * Hkv + kvh) * gridDim.y + blockIdx.y;
    const size_t slot = (size_t)grp * a.n_chunks + blockIdx.x;
    const float my_lse = (ok && any && nb > 0) ? m + __log2f(lt) : -INFINITY;
    if (a.cluster_merge) {
      if (qtr == 0) reinterpret_cast<float*>(smem + Smem::lse)[r] = my_lse;
    } else if (nc_b > 1 && ok && qtr == 0) {
      a.part_lse[slot * kRows + r] = my_lse;
    }
    named_sync_rows();
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    const int ld = a.Hq * 128;
    const int valid = min(kRows, rows - row0);
    if (nc_b == 1) {
      // one chunk: each warp writes whole rows, lane = 4 columns, as split bf16
      if (ok && nb > 0) {
        for (int rr = warp; rr < valid; rr += kRowWarps) {
          const float4 v = *stage_at(stg, rr, lane);
          const int q2 = row0 + rr;
          const int nd = q2 / G;
          const int col = (kvh * G + (q2 - nd * G)) * 128 + lane * 4;
          split_store4(out, base + nd, ld, col, v);
        }
      }
    } else if (!a.cluster_merge) {
      // partial rows, coalesced: lane = 4 columns of one row
      float4* po = reinterpret_cast<float4*>(a.part_o + slot * kRows * 128);
      if (ok)
        for (int rr = warp; rr < valid; rr += kRowWarps) __stcg(po + rr * 32 + lane, *stage_at(stg, rr, lane));
      named_sync_rows();
      stamp(a.trace, 5);
      int* ctr = a.counters + 2 * grp;
      if (tid == 0) {
        bool met = false;
        if (!*abort_flag) {
          red_release_add_gpu(ctr, 1);  // the barrier orders every thread's partial stores before it
          met = spin_until_geq(ctr, nc_b, err);
        }
        *merge_ok = met ? 1 : 0;
      }
      named_sync_rows();
      stamp(a.trace, 6);
      if (*merge_ok) {
        const int per = (valid + nc_b - 1) / nc_b;
        const int rb = blockIdx.x * per;
        const int R = max(0, min(valid, rb + per) - rb);
        const float* lse0 = a.part_lse + (size_t)grp * a.n_chunks * kRows + rb;
        const float4* po0 = reinterpret_cast<const float4*>(a.part_o + (size_t)grp * a.n_chunks * kRows * 128) +
                            (size_t)rb * 32 + lane;
        // One slice row per warp and round;
        // every chunk's log-sum-exp and partial in flight at once
        // (chunks <= kAttnMaxChunks).
        for (int rr = warp; rr < R; rr += kRowWarps) {
          float lv[kAttnMaxChunks];
          float4 pv[kAttnMaxChunks];
#pragma unroll
          for (int c = 0; c < kAttnMaxChunks; ++c) {
            const bool on = c < nc_b;
            lv[c] = on ? __ldcg(lse0 + (size_t)c * kRows + rr) : -INFINITY;
            pv[c] = on ? __ldcg(po0 + ((size_t)c * kRows + rr) * 32) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < kAttnMaxChunks; ++c) mx = fmaxf(mx, lv[c]);
          float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
          float wsum = 0.f;
#pragma unroll
          for (int c = 0; c < kAttnMaxChunks; ++c) {
            const float w = fast_exp2(lv[c] - mx);  // 2^-inf = 0 for empty chunks and padding
            wsum += w;
            acc.x = fmaf(w, pv[c].x, acc.x);
            acc.y = fmaf(w, pv[c].y, acc.y);
            acc.z = fmaf(w, pv[c].z, acc.z);
            acc.w = fmaf(w, pv[c].w, acc.w);
          }
          const float wi = wsum > 0.f ? 1.f / wsum : 0.f;
          acc.x *= wi;
          acc.y *= wi;
          acc.z *= wi;
          acc.w *= wi;
          const int q2 = row0 + rb + rr;
          const int nd = q2 / G;
          const int col = (kvh * G + (q2 - nd * G)) * 128 + lane * 4;
          split_store4(out, base + nd, ld, col, acc);
        }
        named_sync_rows();
        stamp(a.trace, 7);
        // (each layer has its own counters, zeroed with the step: nothing to reset)
      }
    }
  }
  if (a.cluster_merge) {
    // every chunk CTA of the cluster has staged its normalised output and
    // log2-sum-exps in its own shared memory; each merges a slice of the rows
    // by reading its peers' (distributed shared memory), then the cluster
    // meets again so that no CTA leaves while a peer still reads it
    cluster_sync_all();
    if (warp < kRowWarps && nc_b > 1) {
      const int valid = min(kRows, rows - row0);
      const int per = (valid + nc_b - 1) / nc_b;
      const int rb = blockIdx.x * per;
      const int R = max(0, min(valid, rb + per) - rb);
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
      const int ld = a.Hq * 128;
      const uint32_t lse_base = smem_u32(smem + Smem::lse);
      const uint32_t stg_base = smem_u32(smem + Smem::k);
      for (int rr = warp; rr < R; rr += kRowWarps) {
        const int row = rb + rr;
        const uint32_t soff = (uint32_t)(reinterpret_cast<uint8_t*>(stage_at(smem + Smem::k, row, lane)) -
                                         (smem + Smem::k));
        float lv[kAttnMaxChunks];
        float4 pv[kAttnMaxChunks];
#pragma unroll
        for (int c = 0; c < kAttnMaxChunks; ++c) {
          if (c < nc_b) {
            lv[c] = dsmem_ld_f32(map_peer(lse_base + 4 * row, c));
            pv[c] = dsmem_ld_f4(map_peer(stg_base + soff, c));
          } else {
            lv[c] = -INFINITY;
            pv[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kAttnMaxChunks; ++c) mx = fmaxf(mx, lv[c]);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        float wsum = 0.f;
#pragma unroll
        for (int c = 0; c < kAttnMaxChunks; ++c) {
          if (lv[c] == -INFINITY) continue;  // empty chunk: its staged values are not written
          const float w = fast_exp2(lv[c] - mx);
          wsum += w;
          acc.x = fmaf(w, pv[c].x, acc.x);
          acc.y = fmaf(w, pv[c].y, acc.y);
          acc.z = fmaf(w, pv[c].z, acc.z);
          acc.w = fmaf(w, pv[c].w, acc.w);
        }
        const float wi = wsum > 0.f ? 1.f / wsum : 0.f;
        acc.x *= wi;
        acc.y *= wi;
        acc.z *= wi;
        acc.w *= wi;
        const int q2 = row0 + row;
        const int nd = q2 / G;
        const int col = (kvh * G + (q2 - nd * G)) * 128 + lane * 4;
        split_store4(out, base + nd, ld, col, acc);
      }
    }
    stamp(a.trace, 7);
    cluster_sync_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kCtrlWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

size_t attention_tc_smem_bytes() { return Smem::dyn; }

cudaError_t attention_tc_configure(int* max_clusters) {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)attention_tc_smem_bytes());
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  // how many clusters of cs chunk CTAs the GPU holds at once (0: none)
  const bool nonportable =
      cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
  for (int cs = 0; cs <= kAttnMaxChunks; ++cs) {
    max_clusters[cs] = 0;
    if (cs < 2 || (cs > 8 && !nonportable)) continue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = attention_tc_smem_bytes();
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = cs;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void*)attn_tc_kernel, &cfg) == cudaSuccess) max_clusters[cs] = n;
  }
  (void)cudaGetLastError();  // a rejected size is not an error of the library
  return cudaSuccess;
}

cudaError_t launch_attention_tc(const AttnArgs& a, const AttnTcMaps& maps, cudaStream_t s, bool pdl) {
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (a.cluster_merge) {  // the chunk CTAs of a row tile form one cluster
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = a.n_chunks;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_chunks, (a.max_rows + kRows - 1) / kRows, a.sv.B * a.kv.Hkv);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = attention_tc_smem_bytes();
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel, maps, a);
}

}  // namespace spec
