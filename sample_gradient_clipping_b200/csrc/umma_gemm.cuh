// Persistent, warp-specialised tcgen05 contraction engine for sm_100a.
//
// One CTA per SM (192 threads) walks a static list of work units:
//   warp 0      TMA producer: loads 128-byte-swizzled A/B tiles into a STAGES-deep smem ring;
//   warp 1      MMA issuer: allocates all 512 TMEM columns, one lane issues tcgen05.mma
//               (M = 128, N = BN, K = 16 per instruction) into a TMEM accumulator;
//               accumulators are double-buffered (all but kEpiGhostShared, whose four
//               accumulators fill TMEM) so the epilogue of unit u overlaps the mainloop of
//               unit u + 1;
//   warps 2..5  epilogue: each thread owns one accumulator row (TMEM lane) and reads it
//               back 32 columns at a time with tcgen05.ld.
//
// The same engine serves these contractions of the step:
//   kEpiClipSum      S[a, b] = sum_t Xs[t, a] dYs[t, b] over all B*T tokens (both operands
//                    MN-major; the clip factor is already folded into one operand), with the
//                    Philox/Box-Muller noise added in the epilogue before the fp32 store;
//   kEpiExplicitNorm per (sample, output tile): the tile of G_i = X_i^T dY_i over the
//                    sample's T tokens, squared and summed on chip; each epilogue warp writes
//                    its partial to its own slot, and the slots of a sample are summed later
//                    in a fixed order (norms reproducible bit for bit);
//   kEpiGhostNorm    per (sample, upper-triangular pair of 128-token blocks): the X Gram
//                    tile and the dY Gram tile in two TMEM accumulators; the epilogue sums
//                    w * Gx * Gy with w = 2 above the diagonal, 1 on it, 0 below;
//   kEpiStoreBf16    Z = dY P (K-major dY, MN-major P), rounded to bf16;
//   kEpiExplicitStore as kEpiExplicitNorm, and the tile of G_i is also written to HBM in bf16
//                    so that the clipped sum reuses it instead of forming G_i again
//                    (each per-sample gradient is formed once);
//   kEpiAxpy         W[a, b] += alpha * sum_k U[a, k] P[b, k] (both K-major): the projected
//                    optimizer's update mapped back to the weights through P^T;
//   kEpiGhostShared  the ghost norm of up to three linears that read the same input X (q/k/v,
//                    gate/up): one X Gram tile and each linear's dY Gram tile in four TMEM
//                    accumulators, so the X Gram is formed once for the group.
//
// All waits are bounded (ptx.cuh); a wait that runs out sets the CTA's abort flag, records
// its site in the status word and the CTA drains and exits.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rng.cuh"

namespace dpclip {

enum EpiKind : int {
  kEpiClipSum = 0,
  kEpiExplicitNorm = 1,
  kEpiGhostNorm = 2,
  kEpiStoreBf16 = 3,
  kEpiExplicitStore = 4,
  kEpiAxpy = 5,
  kEpiGhostShared = 6
};

constexpr int kGhostSharedMaxOps = 3;  // dY operands per shared X Gram (TMEM: 4 x 128 columns)

// K-blocks ahead of the smem ring that the clipped-sum producer asks TMA to pull into L2.
constexpr int kL2PrefetchDistance = 8;

// kOutSplitPartials (a sum split over K): each unit stores its partial sum into its split's
// slot of a scratch array [k_splits][out_rows][out_cols]; a combining launch then adds the
// slots in split order, so the result does not depend on the order in which units finish.
enum OutMode : int { kOutStore = 0, kOutAtomicAdd = 1, kOutAdd = 2, kOutSplitPartials = 3 };

struct alignas(64) UmmaParams {
  CUtensorMap tmA0, tmB0, tmA1, tmB1;  // phase-1 maps are used by the ghost norm only
  int num_units;
  int m_tiles, n_tiles;       // output tile grid (128 x BN tiles)
  int k_blocks;               // 64-deep K blocks of phase 0
  int k_blocks1;              // 64-deep K blocks of phase 1 (ghost: the dY Gram)
  int k_splits, k_blocks_per_split;
  int t_tiles;                // ghost: 128-token blocks per sample
  int pairs_per_sample;       // ghost: t_tiles (t_tiles + 1) / 2
  int out_rows, out_cols;     // row-major output, leading dimension out_cols
  int out_mode;               // OutMode (clip-sum)
  float* out_f32;
  __nv_bfloat16* out_bf16;
  double noise_std;           // 0 disables the noise
  uint32_t key0, key1, layer_id, step_lo;
  const unsigned long long* step_dev;  // non-null: the step is read here when the kernel runs
  float alpha;                // axpy: W += alpha * acc
  float* partials;            // [B][partial_stride] per-warp squared-norm partials
  int partial_stride;         // slots per sample: 4 per unit of that sample
  int ghost_ops;              // shared ghost: dY operands (1..3); phase 1 + k reads operand k
  long long partial_op_stride;  // shared ghost: floats between the operands' partial arrays
  uint32_t* status;
  long long out_elems;        // elements of the output buffer (device-side checks; 0 = unknown)
  long long partials_elems;   // floats of the partials buffer (device-side checks; 0 = unknown)
  // Ghost kinds: (sample, pair) units [0, split_full_units) whole, each later one in
  // split_parts parts of the K of the X Gram (split_over_x) or of the dY Grams.  The norm is
  // linear in each Gram, so the parts' partial sums add up.  split_parts 0 or 1: none.
  int split_full_units, split_parts, split_over_x;
  float* split_scratch;  // kOutSplitPartials: [k_splits][out_rows][out_cols] fp32
};

// Several independent problems of one contraction kind in one launch: the projections
// Z_l = dY_l P_l of a block's projected linears (kEpiStoreBf16), or the clipped sums of a
// block's ghost/explicit linears (kEpiClipSum, split over K: each split stores its partial sum,
// and a combining launch forms the outputs).  Problem q has its own operand maps, output,
// rows and K depth, and the units [unit_begin[q], unit_begin[q + 1]) of the launch.  Passed as
// a second __grid_constant__ parameter, so launches of one problem keep their parameter size.
constexpr int kMaxGroup = 8;
struct alignas(64) UmmaGroup {
  CUtensorMap tmA[kMaxGroup], tmB[kMaxGroup];
  __nv_bfloat16* out_bf16[kMaxGroup];   // kEpiStoreBf16
  float* out_f32[kMaxGroup];            // kEpiClipSum
  int out_rows[kMaxGroup];              // kEpiClipSum: rows of problem q (m_tiles[q] 128-row tiles)
  int m_tiles[kMaxGroup];               // kEpiClipSum
  int k_blocks[kMaxGroup];
  int k_blocks1[kMaxGroup];             // kEpiGhostNorm: K blocks of the dY (or Z) Gram
  int split_full_units[kMaxGroup];      // kEpiGhostNorm: as in UmmaParams, per problem
  int split_parts[kMaxGroup];
  int split_over_x[kMaxGroup];
  float* partials[kMaxGroup];           // kEpiGhostNorm: the problem's norm-partial set
  int unit_begin[kMaxGroup + 1];
  int count;
  int k_blocks_per_split;               // kEpiClipSum: the group's K split
  float* split_scratch[kMaxGroup];      // kEpiClipSum, kOutSplitPartials: the problem's partials
};

template <int BN_, int EPI_, bool GROUPED_ = false>
struct UmmaConfig {
  static constexpr bool GROUPED = GROUPED_;  // problems from a UmmaGroup (kEpiStoreBf16 only)
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int BK = 64;  // 64 bf16 = 128 bytes: one swizzle atom row
  static constexpr int EPI = EPI_;
  static constexpr bool PER_SAMPLE = (EPI == kEpiExplicitNorm || EPI == kEpiExplicitStore);
  static constexpr bool A_MN = (EPI == kEpiClipSum || PER_SAMPLE);
  static constexpr bool GHOST = (EPI == kEpiGhostNorm || EPI == kEpiGhostShared);
  static constexpr bool B_MN = (!GHOST && EPI != kEpiAxpy);
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static_assert(!GHOST || BM == BN, "ghost tiles are square: a diagonal tile is its own B operand");
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // As many stages as the 227 KB of shared memory hold next to the barriers, up to 8.
  static constexpr int STAGES = ((232448 - 1280) / STAGE_BYTES) < 8 ? ((232448 - 1280) / STAGE_BYTES) : 8;
  static constexpr int ACCS = (EPI == kEpiGhostNorm)     ? 2
                              : (EPI == kEpiGhostShared) ? 1 + kGhostSharedMaxOps
                                                         : 1;  // accumulators per unit
  static constexpr int ACC_COLS = BN * ACCS;
  static constexpr int NUM_BUFS = 512 / ACC_COLS;
  static constexpr int THREADS = 192;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
  static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per block");
  static constexpr uint32_t IDESC = umma_idesc_bf16(BM, BN, A_MN, B_MN);
  static_assert(NUM_BUFS >= 1, "TMEM budget");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(!GROUPED_ || EPI_ == kEpiStoreBf16 || EPI_ == kEpiClipSum || EPI_ == kEpiGhostNorm,
                "grouped launches serve the projection, the clipped sum and the ghost norm");
};

struct Unit {
  int m_blk, n_blk, kb_begin, kb_end, sample, split;
  int local;  // index of the unit among the units of its sample (norm partial slots)
  int prob;   // grouped launch: the problem of the unit
  int kb1;    // ghost kinds: K blocks of the phases after the first (the dY Grams), end
  int kb1_begin;   // ... and first (a unit split over the dY Grams' K)
  int zero_slots;  // ghost kinds: partial slot groups after this unit's own to write as zero
};

// Pair r of one sample's upper-triangular pairs of 128-token blocks -> (row block, column
// block); local = r.
__device__ __forceinline__ void ghost_pair(int r, int t_tiles, Unit& w) {
  w.local = r;
  int c = r, row = 0;
  while (c >= t_tiles - row) {
    c -= t_tiles - row;
    ++row;
  }
  w.m_blk = row;
  w.n_blk = row + c;
}

// Ghost unit r of one problem (pairs per sample, X Gram K blocks kx, dY Gram K blocks k1).
// With parts > 1, the (sample, pair) units from `full` on are each cut in `parts` parts of the
// K of the X Gram (over_x) or of the dY Grams.  Every pair then owns `parts` groups of four
// partial slots (one per epilogue warp), and a whole unit writes zeros into the groups it does
// not use, so that no slot of a sample holds a stale value.
__device__ __forceinline__ void ghost_unit(int r, int pairs, int t_tiles, int full, int parts, bool over_x,
                                           int kx, int k1, Unit& w) {
  const bool split = parts > 1 && r >= full;
  const int base = split ? full + (r - full) / parts : r;
  const int part = split ? (r - full) % parts : 0;
  w.sample = base / pairs;
  ghost_pair(base % pairs, t_tiles, w);
  w.local = w.local * (parts > 1 ? parts : 1) + part;  // its warps write slots 4 local .. 4 local + 3
  w.zero_slots = (parts > 1 && !split) ? parts - 1 : 0;
  w.kb_begin = 0;
  w.kb_end = kx;
  w.kb1_begin = 0;
  w.kb1 = k1;
  if (split && over_x) {
    const int per = (kx + parts - 1) / parts;
    w.kb_begin = part * per;
    w.kb_end = min(kx, w.kb_begin + per);
  } else if (split) {
    const int per = (k1 + parts - 1) / parts;
    w.kb1_begin = part * per;
    w.kb1 = min(k1, w.kb1_begin + per);
  }
}

template <class Cfg>
__device__ __forceinline__ Unit decode_unit(const UmmaParams& p, int u, const UmmaGroup* grp = nullptr) {
  Unit w{};
  if constexpr (Cfg::GROUPED) {
    // Problem q owns units unit_begin[q] .. unit_begin[q+1]-1, row-tile-major, n_tiles each row.
    int q = 0;
    while (q + 1 < grp->count && u >= grp->unit_begin[q + 1]) ++q;
    const int r = u - grp->unit_begin[q];
    w.prob = q;
    if (Cfg::EPI == kEpiClipSum) {  // split-major, then row tiles, then column tiles
      const int tiles = grp->m_tiles[q] * p.n_tiles;
      w.split = r / tiles;
      w.m_blk = (r % tiles) / p.n_tiles;
      w.n_blk = (r % tiles) % p.n_tiles;
      w.kb_begin = w.split * grp->k_blocks_per_split;
      w.kb_end = min(grp->k_blocks[q], w.kb_begin + grp->k_blocks_per_split);
      return w;
    }
    if (Cfg::EPI == kEpiGhostNorm) {
      ghost_unit(r, p.pairs_per_sample, p.t_tiles, grp->split_full_units[q], grp->split_parts[q],
                 grp->split_over_x[q] != 0, grp->k_blocks[q], grp->k_blocks1[q], w);
      return w;
    }
    w.m_blk = r / p.n_tiles;
    w.n_blk = r % p.n_tiles;
    w.kb_begin = 0;
    w.kb_end = grp->k_blocks[q];
    return w;
  }
  if (Cfg::GHOST) {
    ghost_unit(u, p.pairs_per_sample, p.t_tiles, p.split_full_units, p.split_parts, p.split_over_x != 0,
               p.k_blocks, p.k_blocks1, w);
    return w;
  }
  const int tiles = p.m_tiles * p.n_tiles;
  int r = u % tiles;
  const int outer = u / tiles;
  w.local = r;
  // Rasterise in groups of 8 row-tiles so that concurrently running CTAs share operand tiles
  // in L2.
  constexpr int G = 8;
  const int per_group = G * p.n_tiles;
  const int first_m = (r / per_group) * G;
  const int gsz = min(G, p.m_tiles - first_m);
  const int within = r % per_group;
  w.m_blk = first_m + within % gsz;
  w.n_blk = within / gsz;
  if (Cfg::PER_SAMPLE) {
    w.sample = outer;
    w.split = 0;
    w.kb_begin = 0;
    w.kb_end = p.k_blocks;
  } else {
    w.sample = 0;
    w.split = outer;
    w.kb_begin = outer * p.k_blocks_per_split;
    w.kb_end = min(p.k_blocks, w.kb_begin + p.k_blocks_per_split);
  }
  return w;
}

// A ghost unit on the diagonal (both token blocks the same) forms X_a X_a^T and dY_a dY_a^T:
// its two operands are one tile, loaded once into the A slot and read by both descriptors.
template <class Cfg>
__device__ __forceinline__ bool ghost_diagonal(const Unit& w) {
  if constexpr (Cfg::GHOST) return w.m_blk == w.n_blk;
  return false;
}

template <class Cfg>
__device__ __forceinline__ void issue_stage_loads(const UmmaParams& p, const Unit& w, int phase,
                                                  int kb, uint32_t sA, uint32_t sB,
                                                  uint32_t bar, const UmmaGroup* grp = nullptr) {
  const int k0 = kb * Cfg::BK;
  if constexpr (Cfg::GROUPED && Cfg::EPI == kEpiClipSum) {  // both operands MN-major, per problem
#pragma unroll
    for (int h = 0; h < Cfg::BM / 64; ++h)
      tma_load_2d(sA + h * (Cfg::BK * 128), &grp->tmA[w.prob], bar, w.m_blk * Cfg::BM + 64 * h, k0);
#pragma unroll
    for (int h = 0; h < Cfg::BN / 64; ++h)
      tma_load_2d(sB + h * (Cfg::BK * 128), &grp->tmB[w.prob], bar, w.n_blk * Cfg::BN + 64 * h, k0);
    return;
  } else if constexpr (Cfg::GROUPED && Cfg::EPI == kEpiStoreBf16) {  // per problem: A = dY rows (K-major), B = P (MN-major)
    tma_load_2d(sA, &grp->tmA[w.prob], bar, k0, w.m_blk * Cfg::BM);
#pragma unroll
    for (int h = 0; h < Cfg::BN / 64; ++h)
      tma_load_2d(sB + h * (Cfg::BK * 128), &grp->tmB[w.prob], bar, w.n_blk * Cfg::BN + 64 * h, k0);
    return;
  }
  if (Cfg::EPI == kEpiClipSum) {
#pragma unroll
    for (int h = 0; h < Cfg::BM / 64; ++h)
      tma_load_2d(sA + h * (Cfg::BK * 128), &p.tmA0, bar, w.m_blk * Cfg::BM + 64 * h, k0);
#pragma unroll
    for (int h = 0; h < Cfg::BN / 64; ++h)
      tma_load_2d(sB + h * (Cfg::BK * 128), &p.tmB0, bar, w.n_blk * Cfg::BN + 64 * h, k0);
  } else if (Cfg::PER_SAMPLE) {
#pragma unroll
    for (int h = 0; h < Cfg::BM / 64; ++h)
      tma_load_3d(sA + h * (Cfg::BK * 128), &p.tmA0, bar, w.m_blk * Cfg::BM + 64 * h, k0,
                  w.sample);
#pragma unroll
    for (int h = 0; h < Cfg::BN / 64; ++h)
      tma_load_3d(sB + h * (Cfg::BK * 128), &p.tmB0, bar, w.n_blk * Cfg::BN + 64 * h, k0,
                  w.sample);
  } else if (Cfg::EPI == kEpiGhostNorm) {
    // Both operands of a Gram tile from one map (X, or dY / Z), at the pair's two token blocks.
    const CUtensorMap* ma = Cfg::GROUPED ? (phase ? &grp->tmB[w.prob] : &grp->tmA[w.prob])
                                         : (phase ? &p.tmA1 : &p.tmA0);
    const CUtensorMap* mb = Cfg::GROUPED ? ma : (phase ? &p.tmB1 : &p.tmB0);
    tma_load_3d(sA, ma, bar, k0, w.m_blk * Cfg::BM, w.sample);
    if (!ghost_diagonal<Cfg>(w)) tma_load_3d(sB, mb, bar, k0, w.n_blk * Cfg::BN, w.sample);
  } else if (Cfg::EPI == kEpiGhostShared) {
    // Phase 0 reads X (tmA0), phase 1 + k reads dY operand k (tmB0, tmA1, tmB1); both
    // operands of a Gram tile come from the same map, at the two token blocks of the pair.
    const CUtensorMap* m = phase == 0 ? &p.tmA0 : phase == 1 ? &p.tmB0 : phase == 2 ? &p.tmA1 : &p.tmB1;
    tma_load_3d(sA, m, bar, k0, w.m_blk * Cfg::BM, w.sample);
    if (!ghost_diagonal<Cfg>(w)) tma_load_3d(sB, m, bar, k0, w.n_blk * Cfg::BN, w.sample);
  } else if (Cfg::EPI == kEpiAxpy) {  // A = U rows, B = P rows, both K-major
    tma_load_2d(sA, &p.tmA0, bar, k0, w.m_blk * Cfg::BM);
    tma_load_2d(sB, &p.tmB0, bar, k0, w.n_blk * Cfg::BN);
  } else {  // kEpiStoreBf16: A = dY rows (K-major), B = P (MN-major)
    tma_load_2d(sA, &p.tmA0, bar, k0, w.m_blk * Cfg::BM);
#pragma unroll
    for (int h = 0; h < Cfg::BN / 64; ++h)
      tma_load_2d(sB + h * (Cfg::BK * 128), &p.tmB0, bar, w.n_blk * Cfg::BN + 64 * h, k0);
  }
}

// Clipped sum only: pull the A/B boxes of K-block `kb` into L2 ahead of their smem loads.
// Every k-slice of the long token dimension is first touched by one CTA and then re-read by
// the others, so its DRAM latency would otherwise stall the MMA.
template <class Cfg>
__device__ __forceinline__ void prefetch_stage_l2(const UmmaParams& p, const Unit& w, int kb) {
  const int k0 = kb * Cfg::BK;
#pragma unroll
  for (int h = 0; h < Cfg::BM / 64; ++h) tma_prefetch_l2_2d(&p.tmA0, w.m_blk * Cfg::BM + 64 * h, k0);
#pragma unroll
  for (int h = 0; h < Cfg::BN / 64; ++h) tma_prefetch_l2_2d(&p.tmB0, w.n_blk * Cfg::BN + 64 * h, k0);
}

template <class Cfg>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int ks, bool mn_major) {
  // MN-major: 16 K-rows of 128 bytes per MMA step; MN chunks of 64 elements BK*128 bytes apart.
  // K-major : 32 bytes (16 bf16) per MMA step inside the 128-byte swizzle row.
  return mn_major ? umma_desc_sw128(base + ks * 2048, Cfg::BK * 128, 1024)
                  : umma_desc_sw128(base + ks * 32, 16, 1024);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

template <class Cfg>
__device__ __forceinline__ void epilogue_unit(const UmmaParams& p, const Unit& w, uint32_t tacc,
                                              int wq, uint32_t lane, const UmmaGroup* grp = nullptr) {
  const int row = wq * 32 + static_cast<int>(lane);
  if (Cfg::EPI == kEpiClipSum) {
    const long long grow = static_cast<long long>(w.m_blk) * Cfg::BM + row;
    const int out_rows = Cfg::GROUPED ? grp->out_rows[w.prob] : p.out_rows;
    float* const out_base = Cfg::GROUPED ? grp->out_f32[w.prob] : p.out_f32;
    [[maybe_unused]] const long long out_elems =
        Cfg::GROUPED ? static_cast<long long>(out_rows) * p.out_cols : p.out_elems;
    const bool row_ok = grow < out_rows;
    const bool noisy = (p.noise_std != 0.0) && (w.split == 0);
    const PhiloxKey key{p.key0, p.key1};
    const uint32_t step_lo = StepRef{p.step_lo, p.step_dev}.get();
    const bool partial = (p.out_mode == kOutSplitPartials);
    float* const scratch = Cfg::GROUPED ? grp->split_scratch[w.prob] : p.split_scratch;
    const long long split_stride = static_cast<long long>(out_rows) * p.out_cols;
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float v[32];
      __syncwarp();
      tmem_ld32(tacc + c0, v);
      tmem_ld_wait();
      const long long gcol0 = static_cast<long long>(w.n_blk) * Cfg::BN + c0;
      if (!row_ok || gcol0 >= p.out_cols) continue;  // the next tmem_ld32 reconverges first
      float* dst = out_base + grow * p.out_cols + gcol0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (gcol0 + 4 * q >= p.out_cols) break;  // out_cols is a multiple of 4
        float4 val = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        if (noisy) {
          const unsigned long long k = static_cast<unsigned long long>(grow) * p.out_cols + gcol0 + 4 * q;
          double z[4];
          normals4(static_cast<uint32_t>(k >> 2), p.layer_id, step_lo, kStreamNoise, key, z);
          val.x = static_cast<float>(static_cast<double>(val.x) + p.noise_std * z[0]);
          val.y = static_cast<float>(static_cast<double>(val.y) + p.noise_std * z[1]);
          val.z = static_cast<float>(static_cast<double>(val.z) + p.noise_std * z[2]);
          val.w = static_cast<float>(static_cast<double>(val.w) + p.noise_std * z[3]);
        }
        if (!DP_DCHECK(in_buffer(grow * p.out_cols + gcol0 + 4 * q, 4, out_elems), 1u, p.status)) break;
        float4* d4 = reinterpret_cast<float4*>(dst + 4 * q);
        if (partial) {
          if (!DP_DCHECK(w.split >= 0 && w.split < p.k_splits, 30u, p.status)) break;
          *reinterpret_cast<float4*>(scratch + w.split * split_stride + grow * p.out_cols + gcol0 + 4 * q) = val;
        } else if (p.out_mode == kOutStore) {
          *d4 = val;
        } else if (p.out_mode == kOutAtomicAdd) {
          atomicAdd(d4, val);
        } else {
          float4 o = *d4;
          o.x += val.x; o.y += val.y; o.z += val.z; o.w += val.w;
          *d4 = o;
        }
      }
    }
  } else if (Cfg::PER_SAMPLE) {
    // Rows and columns past d_in / ne were zero-filled by TMA and add nothing.
    float ss = 0.f;
    const long long grow = static_cast<long long>(w.m_blk) * Cfg::BM + row;
    const bool row_ok = grow < p.out_rows;
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float v[32];
      __syncwarp();
      tmem_ld32(tacc + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) ss = fmaf(v[e], v[e], ss);
      if (Cfg::EPI == kEpiExplicitStore && row_ok) {
        const long long gcol0 = static_cast<long long>(w.n_blk) * Cfg::BN + c0;
        __nv_bfloat16* dst = p.out_bf16 + (static_cast<long long>(w.sample) * p.out_rows + grow) * p.out_cols + gcol0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (gcol0 + 8 * q >= p.out_cols) break;  // out_cols is a multiple of 8
          uint4 pk;
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
          for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
          if (!DP_DCHECK(in_buffer((static_cast<long long>(w.sample) * p.out_rows + grow) * p.out_cols + gcol0 + 8 * q,
                                   8, p.out_elems), 2u, p.status))
            break;
          *reinterpret_cast<uint4*>(dst + 8 * q) = pk;
        }
      }
    }
    ss = warp_sum(ss);
    const long long slot = static_cast<long long>(w.sample) * p.partial_stride + 4 * w.local + wq;
    if (lane == 0 && DP_DCHECK(4 * w.local + wq < p.partial_stride && in_buffer(slot, 1, p.partials_elems), 3u,
                               p.status))
      p.partials[slot] = ss;
  } else if (Cfg::EPI == kEpiGhostNorm) {
    // Rows and columns past T were zero-filled by TMA, so their Gram entries are 0.
    const int t = w.m_blk * Cfg::BM + row;
    float ss = 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float gx[32], gy[32];
      tmem_ld32(tacc + c0, gx);
      tmem_ld32(tacc + Cfg::BN + c0, gy);
      tmem_ld_wait();
      const int s0 = w.n_blk * Cfg::BN + c0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int s = s0 + e;
        const float wgt = (t < s) ? 2.f : ((t == s) ? 1.f : 0.f);
        ss = fmaf(wgt * gx[e], gy[e], ss);
      }
    }
    ss = warp_sum(ss);
    const long long slot = static_cast<long long>(w.sample) * p.partial_stride + 4 * w.local + wq;
    float* const partials = Cfg::GROUPED ? grp->partials[w.prob] : p.partials;
    if (lane == 0 && DP_DCHECK(4 * (w.local + w.zero_slots) + wq < p.partial_stride &&
                                   in_buffer(slot, 1 + 4 * w.zero_slots, p.partials_elems), 4u, p.status)) {
      partials[slot] = ss;
      for (int z = 1; z <= w.zero_slots; ++z) partials[slot + 4 * z] = 0.f;
    }
  } else if (Cfg::EPI == kEpiGhostShared) {
    const int t = w.m_blk * Cfg::BM + row;
    float ss[kGhostSharedMaxOps] = {0.f, 0.f, 0.f};
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float gx[32];
      tmem_ld32(tacc + c0, gx);
      tmem_ld_wait();
      const int s0 = w.n_blk * Cfg::BN + c0;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int s = s0 + e;
        gx[e] *= (t < s) ? 2.f : ((t == s) ? 1.f : 0.f);
      }
#pragma unroll
      for (int op = 0; op < kGhostSharedMaxOps; ++op) {
        if (op < p.ghost_ops) {  // uniform across the CTA
          float gy[32];
          tmem_ld32(tacc + (1 + op) * Cfg::BN + c0, gy);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) ss[op] = fmaf(gx[e], gy[e], ss[op]);
        }
      }
    }
#pragma unroll
    for (int op = 0; op < kGhostSharedMaxOps; ++op) {
      if (op < p.ghost_ops) {
        const float v = warp_sum(ss[op]);
        const long long slot = op * p.partial_op_stride + static_cast<long long>(w.sample) * p.partial_stride +
                               4 * w.local + wq;
        if (lane == 0 && DP_DCHECK(4 * (w.local + w.zero_slots) + wq < p.partial_stride &&
                                       in_buffer(slot, 1 + 4 * w.zero_slots, p.partials_elems), 5u, p.status)) {
          p.partials[slot] = v;
          for (int z = 1; z <= w.zero_slots; ++z) p.partials[slot + 4 * z] = 0.f;
        }
      }
    }
  } else if (Cfg::EPI == kEpiAxpy) {
    const long long grow = static_cast<long long>(w.m_blk) * Cfg::BM + row;
    const bool row_ok = grow < p.out_rows;
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float v[32];
      __syncwarp();
      tmem_ld32(tacc + c0, v);
      tmem_ld_wait();
      const long long gcol0 = static_cast<long long>(w.n_blk) * Cfg::BN + c0;
      if (!row_ok || gcol0 >= p.out_cols) continue;  // the next tmem_ld32 reconverges first
      float* dst = p.out_f32 + grow * p.out_cols + gcol0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (gcol0 + 4 * q >= p.out_cols) break;  // out_cols is a multiple of 4
        if (!DP_DCHECK(in_buffer(grow * p.out_cols + gcol0 + 4 * q, 4, p.out_elems), 6u, p.status)) break;
        float4* d4 = reinterpret_cast<float4*>(dst + 4 * q);
        float4 o = *d4;
        o.x = fmaf(p.alpha, v[4 * q], o.x);
        o.y = fmaf(p.alpha, v[4 * q + 1], o.y);
        o.z = fmaf(p.alpha, v[4 * q + 2], o.z);
        o.w = fmaf(p.alpha, v[4 * q + 3], o.w);
        *d4 = o;
      }
    }
  } else {  // kEpiStoreBf16
    const long long grow = static_cast<long long>(w.m_blk) * Cfg::BM + row;
#pragma unroll 1
    for (int c0 = 0; c0 < Cfg::BN; c0 += 32) {
      float v[32];
      __syncwarp();
      tmem_ld32(tacc + c0, v);
      tmem_ld_wait();
      const long long gcol0 = static_cast<long long>(w.n_blk) * Cfg::BN + c0;
      if (grow >= p.out_rows) continue;  // the next tmem_ld32 reconverges first
      __nv_bfloat16* dst = (Cfg::GROUPED ? grp->out_bf16[w.prob] : p.out_bf16) + grow * p.out_cols + gcol0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (gcol0 + 8 * q >= p.out_cols) break;  // out_cols is a multiple of 8
        uint4 pk;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&pk);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
        if (!DP_DCHECK(in_buffer(grow * p.out_cols + gcol0 + 8 * q, 8, p.out_elems), 7u, p.status)) break;
        *reinterpret_cast<uint4*>(dst + 8 * q) = pk;
      }
    }
  }
}

template <class Cfg>
__device__ __forceinline__ void umma_body(const UmmaParams& p, const UmmaGroup* grp) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::STAGES * Cfg::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + Cfg::STAGES;
  uint64_t* acc_full = bars + 2 * Cfg::STAGES;
  uint64_t* acc_empty = acc_full + Cfg::NUM_BUFS;
  uint64_t* drain = acc_empty + Cfg::NUM_BUFS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), 1);
    }
    for (int b = 0; b < Cfg::NUM_BUFS; ++b) {
      mbar_init(smem_addr(acc_full + b), 1);
      mbar_init(smem_addr(acc_empty + b), 4);  // one arrival per epilogue warp
    }
    mbar_init(smem_addr(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    if constexpr (Cfg::GROUPED) {
      for (int q = 0; q < grp->count; ++q) {
        tma_prefetch_desc(&grp->tmA[q]);
        tma_prefetch_desc(&grp->tmB[q]);
      }
    } else {
      tma_prefetch_desc(&p.tmA0);
      tma_prefetch_desc(&p.tmB0);
    }
    if (Cfg::GHOST) {
      tma_prefetch_desc(&p.tmA1);
      tma_prefetch_desc(&p.tmB1);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), 512);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // barriers and TMEM are ready; global memory only from here
  const int nphases = (Cfg::EPI == kEpiGhostNorm) ? 2 : (Cfg::EPI == kEpiGhostShared) ? 1 + p.ghost_ops : 1;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
        const Unit w = decode_unit<Cfg>(p, u, grp);
        for (int ph = 0; ok && ph < nphases; ++ph) {
          const int kb_end = ph ? w.kb1 : w.kb_end;
          const int kb_begin = ph ? w.kb1_begin : w.kb_begin;
          for (int kb = kb_begin; kb < kb_end; ++kb) {
            if (!mbar_wait_bounded(smem_addr(empty + stage), phase ^ 1u, abort_flag, p.status, 1u)) {
              ok = false;
              break;
            }
            const uint32_t sA = smem_addr(smem + stage * Cfg::STAGE_BYTES);
            const uint32_t bar = smem_addr(full + stage);
            mbar_arrive_expect_tx(bar, ghost_diagonal<Cfg>(w) ? Cfg::A_BYTES : Cfg::STAGE_BYTES);
            issue_stage_loads<Cfg>(p, w, ph, kb, sA, sA + Cfg::A_BYTES, bar, grp);
            if (Cfg::EPI == kEpiClipSum && !Cfg::GROUPED) {
              if (kb == kb_begin) {
                for (int d = 1; d <= kL2PrefetchDistance && kb + d < kb_end; ++d)
                  prefetch_stage_l2<Cfg>(p, w, kb + d);
              } else if (kb + kL2PrefetchDistance < kb_end) {
                prefetch_stage_l2<Cfg>(p, w, kb + kL2PrefetchDistance);
              }
            }
            if (++stage == Cfg::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
        const Unit w = decode_unit<Cfg>(p, u, grp);
        if (!mbar_wait_bounded(smem_addr(acc_empty + buf), buf_phase ^ 1u, abort_flag, p.status, 2u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ph = 0; ok && ph < nphases; ++ph) {
          const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_COLS + ph * Cfg::BN;
          const int kb_end = ph ? w.kb1 : w.kb_end;
          const int kb_begin = ph ? w.kb1_begin : w.kb_begin;
          for (int kb = kb_begin; kb < kb_end; ++kb) {
            if (!mbar_wait_bounded(smem_addr(full + stage), phase, abort_flag, p.status, 3u)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sA = smem_addr(smem + stage * Cfg::STAGE_BYTES);
            const uint32_t sB = ghost_diagonal<Cfg>(w) ? sA : sA + Cfg::A_BYTES;
#pragma unroll
            for (int ks = 0; ks < Cfg::BK / 16; ++ks) {
              umma_bf16(d_tmem, operand_desc<Cfg>(sA, ks, Cfg::A_MN),
                        operand_desc<Cfg>(sB, ks, Cfg::B_MN), Cfg::IDESC,
                        (kb > kb_begin || ks > 0) ? 1u : 0u);
            }
            umma_commit(smem_addr(empty + stage));  // frees the smem stage once read
            if (++stage == Cfg::STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(smem_addr(acc_full + buf));  // accumulator ready for the epilogue
        if (++buf == Cfg::NUM_BUFS) {
          buf = 0;
          buf_phase ^= 1u;
        }
      }
      // Make sure no MMA is still writing TMEM before it is released.
      umma_commit(smem_addr(drain));
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(smem_addr(drain), 0u)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          if (p.status) atomicCAS(p.status, 0u, 5u);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
      const Unit w = decode_unit<Cfg>(p, u, grp);
      if (!mbar_wait_bounded(smem_addr(acc_full + buf), buf_phase, abort_flag, p.status, 4u)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * Cfg::ACC_COLS + (static_cast<uint32_t>(wq * 32) << 16);
      epilogue_unit<Cfg>(p, w, tacc, wq, lane, grp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(acc_empty + buf));
      if (++buf == Cfg::NUM_BUFS) {
        buf = 0;
        buf_phase ^= 1u;
      }
    }
  }
  __syncthreads();
  griddep_launch_dependents();  // every role is done: the next kernel may take the SM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1) umma_kernel(const __grid_constant__ UmmaParams p) {
  umma_body<Cfg>(p, nullptr);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    umma_group_kernel(const __grid_constant__ UmmaParams p, const __grid_constant__ UmmaGroup g) {
  umma_body<Cfg>(p, &g);
}

}  // namespace dpclip
