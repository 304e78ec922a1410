// Two-SM (cta_group::2) variant of the per-sample explicit contraction and of the clipped
// sum, for sm_100a.
//
// A cluster of two CTAs on two SMs computes one 256 x 256 tile of G_i = X_i^T dY_i (per
// sample), or of S = Xs^T dYs over all B*T tokens (clipped sum, one operand pre-scaled).
//   * Each CTA loads half of A (its 128 rows of d_in) and half of B (its 128 columns of
//     d_out).  So each SM moves 32 KB per 64-token K-block instead of the 48 KB of a
//     128 x 256 one-SM tile, for twice the MMA work per pair.  With 32 KB stages the
//     smem ring is 6 deep (7 for the per-sample store kernel).
//   * The leader CTA (rank 0) issues one tcgen05.mma.cta_group::2 (M = 256, N = 256,
//     K = 16) per step.  It reads both CTAs' smem at the same offsets and writes each CTA's
//     TMEM: rows 0..127 land in the leader's 128 lanes, rows 128..255 in the peer's.
//   * Both CTAs' TMA loads complete on the leader's full barrier.  The leader's commits
//     arrive on both CTAs' empty and accumulator-full barriers through a CTA mask.  Each
//     CTA's epilogue reads its own 128 TMEM lanes and then arrives on the leader's
//     accumulator-empty barrier, remotely in the peer's case.
// The epilogues are those of the one-SM engine (explicit norm, explicit store, clipped sum
// with its noise), applied to the CTA's 128 rows.  (An L2 prefetch of later k-blocks along
// the clipped sum's long token dimension was measured and dropped: 8, 16 or 32 blocks ahead
// it made that kernel 5% slower than no prefetch.  256 x 128 pair tiles, which fill the last
// wave of a 4096 x 4096 output better, were 10% slower there and 40% slower on GPT-2's
// 768 x 3072.)  Every wait is bounded, as in the one-SM engine.
#pragma once
#include "umma_gemm.cuh"

namespace dpclip {

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared-memory address of the same variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar_cluster,
                                                 int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar_cluster,
                                                 int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8, %9, %10, %11, %12}, p;\n\t}\n" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive on `bar` (same smem offset) in every CTA of `cta_mask` once the pair's MMAs issued so
// far have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}
// Arrive on the leader's own `bar` once the pair's MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_local(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

template <int EPI_>
struct Umma2Config {
  static constexpr bool GROUPED = false;
  static constexpr int BM = 128;     // rows per CTA (256 per pair)
  static constexpr int BN = 256;     // columns of the pair's tile (each CTA loads half)
  static constexpr int BK = 64;
  static constexpr int EPI = EPI_;
  static constexpr bool PER_SAMPLE = (EPI_ != kEpiClipSum);
  static constexpr bool A_MN = true;
  static constexpr bool B_MN = true;
  static constexpr int A_BYTES = BM * BK * 2;         // 16 KB
  static constexpr int B_BYTES = (BN / 2) * BK * 2;   // 16 KB: this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // The per-sample store kernel runs 7 stages (230,656 of 232,448 bytes): measured 0.6% (7B) and
  // 3% (13B) faster than 6; the others keep 6.
  static constexpr int STAGES = (EPI_ == kEpiExplicitStore) ? 7 : 6;
  static constexpr int ACC_COLS = BN;
  static constexpr int NUM_BUFS = 2;
  static constexpr int THREADS = 192;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
  static constexpr uint32_t IDESC = umma_idesc_bf16(2 * BM, BN, true, true);
  static_assert(EPI_ == kEpiExplicitNorm || EPI_ == kEpiExplicitStore || EPI_ == kEpiClipSum,
                "per-sample explicit kernels and the clipped sum");
};

// Units: (sample or K split, 256-row tile, 256-column tile), sample- or split-major; p.m_tiles
// counts 256-row tiles.
template <class Cfg>
__device__ __forceinline__ Unit decode_unit_pair(const UmmaParams& p, int u) {
  Unit w{};
  const int tiles = p.m_tiles * p.n_tiles;
  const int r = u % tiles;
  w.local = r;
  if (Cfg::PER_SAMPLE) {
    w.sample = u / tiles;
    w.kb_begin = 0;
    w.kb_end = p.k_blocks;
  } else {
    w.split = u / tiles;
    w.kb_begin = w.split * p.k_blocks_per_split;
    w.kb_end = min(p.k_blocks, w.kb_begin + p.k_blocks_per_split);
  }
  constexpr int G = 8;
  const int per_group = G * p.n_tiles;
  const int first_m = (r / per_group) * G;
  const int gsz = min(G, p.m_tiles - first_m);
  const int within = r % per_group;
  w.m_blk = first_m + within % gsz;
  w.n_blk = within / gsz;
  return w;
}

template <class Cfg>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg::THREADS, 1)
    umma_pair_kernel(const __grid_constant__ UmmaParams p) {
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
  const uint32_t rank = cluster_rank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x / 2;
  const int num_pairs = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(smem_addr(full + s), 1);   // leader's arrive_expect_tx; bytes of both CTAs
      mbar_init(smem_addr(empty + s), 1);  // one pair commit per use
    }
    for (int b = 0; b < Cfg::NUM_BUFS; ++b) {
      mbar_init(smem_addr(acc_full + b), 1);
      mbar_init(smem_addr(acc_empty + b), 8);  // 4 epilogue warps in each CTA
    }
    mbar_init(smem_addr(drain), 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tmA0);
    tma_prefetch_desc(&p.tmB0);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), 512);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // barriers and TMEM are ready; global memory only from here

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = pair; ok && u < p.num_units; u += num_pairs) {
        const Unit w = decode_unit_pair<Cfg>(p, u);
        const int a0 = w.m_blk * (2 * Cfg::BM) + static_cast<int>(rank) * Cfg::BM;
        const int b0 = w.n_blk * Cfg::BN + static_cast<int>(rank) * (Cfg::BN / 2);
        for (int kb = w.kb_begin; kb < w.kb_end; ++kb) {
          if (!mbar_wait_bounded(smem_addr(empty + stage), phase ^ 1u, abort_flag, p.status, 11u)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_addr(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sB = sA + Cfg::A_BYTES;
          const uint32_t bar_leader = map_to_rank(smem_addr(full + stage), 0);
          if (leader) mbar_arrive_expect_tx(smem_addr(full + stage), 2 * Cfg::STAGE_BYTES);
          const int k0 = kb * Cfg::BK;
          if constexpr (Cfg::PER_SAMPLE) {
#pragma unroll
            for (int h = 0; h < Cfg::BM / 64; ++h)
              tma_load_3d_pair(sA + h * (Cfg::BK * 128), &p.tmA0, bar_leader, a0 + 64 * h, k0, w.sample);
#pragma unroll
            for (int h = 0; h < Cfg::BN / 128; ++h)
              tma_load_3d_pair(sB + h * (Cfg::BK * 128), &p.tmB0, bar_leader, b0 + 64 * h, k0, w.sample);
          } else {
#pragma unroll
            for (int h = 0; h < Cfg::BM / 64; ++h)
              tma_load_2d_pair(sA + h * (Cfg::BK * 128), &p.tmA0, bar_leader, a0 + 64 * h, k0);
#pragma unroll
            for (int h = 0; h < Cfg::BN / 128; ++h)
              tma_load_2d_pair(sB + h * (Cfg::BK * 128), &p.tmB0, bar_leader, b0 + 64 * h, k0);
          }
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int buf = 0;
      uint32_t buf_phase = 0;
      bool ok = true;
      for (int u = pair; ok && u < p.num_units; u += num_pairs) {
        const Unit w = decode_unit_pair<Cfg>(p, u);
        if (!mbar_wait_bounded(smem_addr(acc_empty + buf), buf_phase ^ 1u, abort_flag, p.status, 12u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * Cfg::ACC_COLS;
        for (int kb = w.kb_begin; kb < w.kb_end; ++kb) {
          if (!mbar_wait_bounded(smem_addr(full + stage), phase, abort_flag, p.status, 13u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_addr(smem + stage * Cfg::STAGE_BYTES);
          const uint32_t sB = sA + Cfg::A_BYTES;
#pragma unroll
          for (int ks = 0; ks < Cfg::BK / 16; ++ks) {
            umma_bf16_pair(d_tmem, umma_desc_sw128(sA + ks * 2048, Cfg::BK * 128, 1024),
                           umma_desc_sw128(sB + ks * 2048, Cfg::BK * 128, 1024), Cfg::IDESC,
                           (kb > w.kb_begin || ks > 0) ? 1u : 0u);
          }
          umma_commit_pair(smem_addr(empty + stage), 0x3);  // frees the stage in both CTAs
          if (++stage == Cfg::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(smem_addr(acc_full + buf), 0x3);  // both halves of the tile are ready
        if (++buf == Cfg::NUM_BUFS) {
          buf = 0;
          buf_phase ^= 1u;
        }
      }
      umma_commit_pair_local(smem_addr(drain));
      const unsigned long long t0 = global_timer_ns();
      while (!mbar_try_wait(smem_addr(drain), 0u)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          if (p.status) atomicCAS(p.status, 0u, 15u);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5 (both CTAs)
    const int wq = warp & 3;
    int buf = 0;
    uint32_t buf_phase = 0;
    for (int u = pair; u < p.num_units; u += num_pairs) {
      Unit w = decode_unit_pair<Cfg>(p, u);
      if (!mbar_wait_bounded(smem_addr(acc_full + buf), buf_phase, abort_flag, p.status, 14u)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + buf * Cfg::ACC_COLS + (static_cast<uint32_t>(wq * 32) << 16);
      // Present this CTA's 128 rows to the one-SM epilogue: a 128-row tile with index
      // 2 m_blk + rank; its norm partial slot is 2 local + rank (4 warps each).
      Unit half = w;
      half.m_blk = 2 * w.m_blk + static_cast<int>(rank);
      half.local = 2 * w.local + static_cast<int>(rank);
      epilogue_unit<Cfg>(p, half, tacc, wq, lane);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(smem_addr(acc_empty + buf), 0));
      if (++buf == Cfg::NUM_BUFS) {
        buf = 0;
        buf_phase ^= 1u;
      }
    }
  }
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still signal it or use its smem
  griddep_launch_dependents();  // every role is done: the next kernel may take the SM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace dpclip
