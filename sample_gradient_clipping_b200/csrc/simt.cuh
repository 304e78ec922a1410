// CUDA-core kernels of the step: Gaussian noise, the projection matrix, the clip-factor
// row scaling, and the fp32 path.
//
// The scaling kernel is an HBM-bound stream; the noise and projection kernels are bound by
// their Box-Muller arithmetic.  All use 16-byte vector loads and stores and grids sized in
// multiples of the SM count.  The fp32 path keeps fp64
// accumulators.  A product of two fp32 values is exact in fp64, so the fp32 parity bounds
// (1e-5 on the sum, 1e-6 on the norms) hold at any T.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>
#include <type_traits>

#include "ptx.cuh"
#include "rng.cuh"

namespace dpclip {

// G[k] = fp32(G[k] + std * z_k), z from stream 0.  One thread per Philox block of 4 elements.
// STAGED: the Box-Muller tables are copied to shared memory once per block (large G); else
// they are read through the read-only cache, which saves the copy's latency on small G.
template <bool STAGED>
__global__ void noise_add_kernel(float* __restrict__ G, unsigned long long total, double std_dev,
                                 PhiloxKey key, uint32_t layer_id, StepRef step) {
  griddep_enter();
  __shared__ double2 tab_s[STAGED ? kNoiseSharedEntries : 1];
  const uint32_t step_lo = step.get();
  if constexpr (STAGED) {
    stage_noise_tables(tab_s);
    __syncthreads();
  }
  using Tab = typename std::conditional<STAGED, NoiseTablesShared, NoiseTablesGlobal>::type;
  Tab tab;
  if constexpr (STAGED) tab = NoiseTablesShared{tab_s};
  const unsigned long long nblk = (total + 3) / 4;
  for (unsigned long long j = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x;
       j < nblk; j += static_cast<unsigned long long>(gridDim.x) * blockDim.x) {
    double z[4];
    normals4(static_cast<uint32_t>(j), layer_id, step_lo, kStreamNoise, key, z, tab, std_dev);
    const unsigned long long k0 = 4 * j;
    if (k0 + 3 < total) {
      if (!DP_DCHECK(in_buffer(static_cast<long long>(k0), 4, static_cast<long long>(total)), 20u, nullptr)) continue;
      float4* p = reinterpret_cast<float4*>(G + k0);
      float4 g = *p;
      g.x = static_cast<float>(static_cast<double>(g.x) + z[0]);
      g.y = static_cast<float>(static_cast<double>(g.y) + z[1]);
      g.z = static_cast<float>(static_cast<double>(g.z) + z[2]);
      g.w = static_cast<float>(static_cast<double>(g.w) + z[3]);
      *p = g;
    } else {
      for (int q = 0; q < 4 && k0 + q < total; ++q)
        G[k0 + q] = static_cast<float>(static_cast<double>(G[k0 + q]) + z[q]);
    }
  }
}

// The noise of several fp32 outputs in one launch: G_s[k] = fp32(G_s[k] + std_s * z_k) with
// z from stream 0 under each segment's own layer_id.  A block step defers to this the noise of
// every linear whose clipped sum was split over K (small outputs), so a block pays one small
// launch instead of one per linear.  The values are those of noise_add_kernel.
constexpr int kMaxNoiseSegments = 16;
struct NoiseSegment {
  float* G;
  unsigned long long total;   // elements
  double std_dev;
  uint32_t layer_id;
};
struct NoiseBatch {
  NoiseSegment seg[kMaxNoiseSegments];
  int count;
};

__global__ void noise_add_batch_kernel(NoiseBatch b, PhiloxKey key, StepRef step) {
  griddep_enter();
  const uint32_t step_lo = step.get();
  unsigned long long nblk_total = 0;
  for (int q = 0; q < b.count; ++q) nblk_total += (b.seg[q].total + 3) / 4;
  for (unsigned long long j = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x;
       j < nblk_total; j += static_cast<unsigned long long>(gridDim.x) * blockDim.x) {
    unsigned long long jj = j;
    int q = 0;
    while ((b.seg[q].total + 3) / 4 <= jj) {  // the segment holding global block j
      jj -= (b.seg[q].total + 3) / 4;
      ++q;
    }
    const NoiseSegment& sg = b.seg[q];
    double z[4];
    normals4(static_cast<uint32_t>(jj), sg.layer_id, step_lo, kStreamNoise, key, z, NoiseTablesGlobal{},
             sg.std_dev);
    const unsigned long long k0 = 4 * jj;
    for (int e = 0; e < 4 && k0 + e < sg.total; ++e)
      sg.G[k0 + e] = static_cast<float>(static_cast<double>(sg.G[k0 + e]) + z[e]);
  }
}

// (z[2q], z[2q+1]) = the noise's Box-Muller transform of words (2q, 2q+1), unscaled
// (verification of the transform on chosen words).
__global__ void box_muller_words_kernel(const uint2* __restrict__ words, double2* __restrict__ z,
                                        unsigned long long npairs) {
  griddep_enter();
  for (unsigned long long q = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x;
       q < npairs; q += static_cast<unsigned long long>(gridDim.x) * blockDim.x) {
    const uint2 w = words[q];
    double a, b;
    box_muller_f64(w.x, w.y, NoiseTablesGlobal{}, 1.0, a, b);
    z[q] = make_double2(a, b);
  }
}

// out[4 j + q] = word q of Philox block j (verification of the raw uint32 stream).
__global__ void philox_blocks_kernel(uint4* __restrict__ out, unsigned long long nblocks,
                                     PhiloxKey key, uint32_t layer_id, uint32_t step_lo,
                                     uint32_t stream_id) {
  griddep_enter();
  for (unsigned long long j = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x;
       j < nblocks; j += static_cast<unsigned long long>(gridDim.x) * blockDim.x)
    out[j] = philox4x32_10(make_uint4(static_cast<uint32_t>(j), layer_id, step_lo, stream_id), key);
}

// P[k] = round(z_k / sqrt(r)), z from stream 1 at step 0: fp64 -> fp32 (RN) [-> bf16 (RN)].
template <bool BF16>
__global__ void projection_kernel(void* __restrict__ P, unsigned long long total, int r,
                                  PhiloxKey key, uint32_t layer_id) {
  griddep_enter();
  const double scale = sqrt(static_cast<double>(r));
  const unsigned long long nblk = (total + 3) / 4;
  for (unsigned long long j = blockIdx.x * static_cast<unsigned long long>(blockDim.x) + threadIdx.x;
       j < nblk; j += static_cast<unsigned long long>(gridDim.x) * blockDim.x) {
    double z[4];
    normals4_precise(static_cast<uint32_t>(j), layer_id, 0u, kStreamProjection, key, z);
    float f[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) f[q] = static_cast<float>(z[q] / scale);
    const unsigned long long k0 = 4 * j;
    if (BF16) {
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(P);
      if (k0 + 3 < total) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(f[2], f[3]);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out + k0) = pk;
      } else {
        for (int q = 0; q < 4 && k0 + q < total; ++q) out[k0 + q] = __float2bfloat16_rn(f[q]);
      }
    } else {
      float* out = static_cast<float*>(P);
      if (k0 + 3 < total) {
        *reinterpret_cast<float4*>(out + k0) = make_float4(f[0], f[1], f[2], f[3]);
      } else {
        for (int q = 0; q < 4 && k0 + q < total; ++q) out[k0 + q] = f[q];
      }
    }
  }
}

// Clip factors that clip_reduce_kernel keeps in shared memory (the rest are recomputed).
constexpr int kReduceCachedSamples = 4096;

// Clip factor of sample i from either squared-norm accumulators or final norms.
__device__ __forceinline__ float clip_factor(float norm, float C) {
  return (norm <= C) ? 1.0f : C / norm;
}

struct NormSource {
  const float* norm2_f32;   // bf16 path: fp32 accumulators of n_i^2
  const double* norm2_f64;  // fp32 path: fp64 accumulators of n_i^2
  const float* norms;       // caller-given norms
  __device__ __forceinline__ float norm(int i) const {
    if (norms) return norms[i];
    if (norm2_f64) return static_cast<float>(sqrt(norm2_f64[i]));
    return sqrtf(norm2_f32[i]);
  }
};

// Sample i's squared norm from its `count` per-warp partials, summed by one warp in a fixed
// order in fp64 (lane-strided, then a butterfly), so the norms and the clip factors that follow
// from them are reproducible bit for bit.  Every lane returns the same value.
__device__ __forceinline__ float warp_norm2_from_partials(const float* __restrict__ partials, int stride,
                                                          int count, int i, int lane) {
  if (!DP_DCHECK(count <= stride && i >= 0, 26u, nullptr)) return 0.0f;
  double acc = 0.0;
  for (int k = lane; k < count; k += 32) acc += static_cast<double>(partials[static_cast<long long>(i) * stride + k]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  return static_cast<float>(acc);
}

// Partials that the bulk-copy reduce sums itself in its prologue (partials == null: the clip
// factors come from its NormSource instead).  Block 0 also writes norm2, norms_out and c_out
// when they are given.
struct PartialsRef {
  const float* partials;
  int stride, count;
  float* norm2;
  float* norms_out;
  float* c_out;
};

// norm2[i] = warp_norm2_from_partials(sample i), one warp per sample.  Also writes
// norms_out[i] = n_i and c_out[i] = c_i when given.
__global__ void reduce_norm_partials_kernel(const float* __restrict__ partials, int stride, int count,
                                            int B, float C, float* __restrict__ norm2,
                                            float* __restrict__ norms_out, float* __restrict__ c_out) {
  griddep_enter();
  const int i = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (i >= B) return;
  const float n2 = warp_norm2_from_partials(partials, stride, count, i, lane);
  if (lane == 0) {
    norm2[i] = n2;
    const float n = sqrtf(n2);
    if (norms_out) norms_out[i] = n;
    if (c_out) c_out[i] = clip_factor(n, C);
  }
}

// flat[i] = sum_l norm2[l][i] over the L layers of a block, in layer order (fp64), and
// flat_norms_out[i] = sqrt(flat[i]) when given: the squared norm of each sample's gradient
// over all the block's weights.
template <typename T>
__global__ void flat_norm2_kernel(const T* __restrict__ norm2_layers, int L, int B, T* __restrict__ flat,
                                  float* __restrict__ flat_norms_out) {
  griddep_enter();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B; i += gridDim.x * blockDim.x) {
    double acc = 0.0;
    for (int l = 0; l < L; ++l) acc += static_cast<double>(norm2_layers[static_cast<long long>(l) * B + i]);
    flat[i] = static_cast<T>(acc);
    if (flat_norms_out) flat_norms_out[i] = static_cast<float>(sqrt(acc));
  }
}

// norms_out[i] = n_i and c_out[i] = c_i for i < B (either may be null).
__global__ void finalize_norms_kernel(NormSource src, int B, float C, float* __restrict__ norms_out,
                                      float* __restrict__ c_out) {
  griddep_enter();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B; i += gridDim.x * blockDim.x) {
    const float n = src.norm(i);
    if (norms_out) norms_out[i] = n;
    if (c_out) c_out[i] = clip_factor(n, C);
  }
}

// out[row, :] = bf16(c_{row / T} * in[row, :]) for a [rows, cols] bf16 matrix, 8 elements per
// thread (cols is a multiple of 8, rows are 16-byte aligned).
// With pr.partials, each block takes one contiguous range of the matrix, which covers the rows
// of one or a few samples, and first turns the per-warp norm partials of just those samples into
// clip factors in shared memory (one warp per sample, the fixed-order routine above, so every
// block gets the same bits).  The block that holds a sample's first row writes its norm2 /
// norms_out / c_out.  The separate partials kernel is then not needed.
constexpr long long kScaleFusedPartialSlots = 1 << 16;  // samples * count per block, at most
constexpr int kScaleFusedMaxSamples = 4096;              // samples one block may cover

// The work of block `blk` of `nblk` blocks (the kernel's own grid, or a segment's share of a
// batched grid).
__device__ __forceinline__ void scale_rows_body(const __nv_bfloat16* __restrict__ in, __nv_bfloat16* __restrict__ out,
                                                long long rows, int cols, int T, const NormSource& src,
                                                const PartialsRef& pr, float C, long long blk, long long nblk) {
  extern __shared__ float scale_c[];  // with pr.partials: c of samples s_lo .. s_hi
  const int vec_per_row = cols / 8;
  const long long total = rows * vec_per_row;
  const long long sample_vecs = static_cast<long long>(T) * vec_per_row;
  // Plain: the block strides over all vectors.  With pr.partials: one contiguous range [v0, v1)
  // per block, which touches few samples.
  long long v_begin = blk * static_cast<long long>(blockDim.x) + threadIdx.x;
  long long v_end = total;
  long long v_step = nblk * blockDim.x;
  long long v0 = 0, v1 = 0;
  if (pr.partials != nullptr) {
    const long long per = (total + nblk - 1) / nblk;
    v0 = blk * per < total ? blk * per : total;
    v1 = v0 + per < total ? v0 + per : total;
    v_begin = v0 + threadIdx.x;
    v_end = v1;
    v_step = blockDim.x;
  }
  // kU vectors per thread and iteration, all kU loads issued before the first is used (one at
  // a time left the stream latency-bound).  The first iteration's loads are issued before the
  // clip factors are formed, so they are in flight meanwhile.
  constexpr int kU = 4;  // 8 measured slower (RoBERTa 0.118 against 0.116 ms a step)
  uint4 pk[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u)
    if (v_begin + u * v_step < v_end) pk[u] = reinterpret_cast<const uint4*>(in)[v_begin + u * v_step];
  int s_lo = 0;
  if (pr.partials != nullptr) {
    if (v0 < v1) {
      const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, warps = blockDim.x / 32;
      s_lo = static_cast<int>(v0 / sample_vecs);
      const int s_hi = static_cast<int>((v1 - 1) / sample_vecs);
      for (int i = s_lo + warp; i <= s_hi; i += warps) {
        const float n2 = warp_norm2_from_partials(pr.partials, pr.stride, pr.count, i, lane);
        if (lane == 0) {
          const float n = sqrtf(n2);
          const float c = clip_factor(n, C);
          scale_c[i - s_lo] = c;
          if (static_cast<long long>(i) * sample_vecs >= v0) {  // the sample's first row is here
            if (pr.norm2) pr.norm2[i] = n2;
            if (pr.norms_out) pr.norms_out[i] = n;
            if (pr.c_out) pr.c_out[i] = c;
          }
        }
      }
    }
    __syncthreads();
  }
  // A thread's vectors only move forward, so its sample index is advanced at each sample
  // boundary instead of divided out per vector (a 64-bit division was most of the kernel's
  // instructions).
  int i_cur = v_begin < v_end ? static_cast<int>(v_begin / sample_vecs) : 0;
  long long next_sample = static_cast<long long>(i_cur + 1) * sample_vecs;  // first vector of sample i_cur + 1
  for (long long v = v_begin; v < v_end; v += kU * v_step) {
    if (v != v_begin) {
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (v + u * v_step < v_end) pk[u] = reinterpret_cast<const uint4*>(in)[v + u * v_step];
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const long long vu = v + u * v_step;
      if (vu >= v_end) break;
      if (vu >= next_sample) {
        if (vu - next_sample < sample_vecs) {
          ++i_cur;
          next_sample += sample_vecs;
        } else {
          i_cur = static_cast<int>(vu / sample_vecs);
          next_sample = static_cast<long long>(i_cur + 1) * sample_vecs;
        }
      }
      const int i = i_cur;
      if (pr.partials != nullptr &&
          !DP_DCHECK(i >= s_lo && (i - s_lo + 1) * sizeof(float) <= dynamic_smem_bytes(), 21u, nullptr))
        break;
      if (!DP_DCHECK(vu >= 0 && vu < total, 22u, nullptr)) break;
      const float c = pr.partials != nullptr ? scale_c[i - s_lo] : clip_factor(src.norm(i), C);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&pk[u]);
      uint4 res;
      __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        o[e] = __floats2bfloat162_rn(c * f.x, c * f.y);
      }
      reinterpret_cast<uint4*>(out)[vu] = res;
    }
  }
}

// The noise of a clipped sum that adds its result to its output (an unsplit sum whose units
// all run in one wave, or a sum split over K without workspace for its split partials, whose
// splits then add by atomics), written into that output before the sum: out[k] = fp32(std *
// z_k), z from stream 0 under the layer's counter; std = 0 writes zeros.  The row-scaling
// kernel that precedes the sum carries it: the scaling is an HBM stream with idle arithmetic
// pipes, and the sum needs both.
struct NoiseFill {
  float* G;                   // null: nothing to write
  unsigned long long total;   // elements
  double std_dev;
  uint32_t layer_id;
};

// This block's share (block `blk` of `nblk`) of the Philox blocks of `fills` (count of them):
// global block j of the fills' concatenation goes to thread j mod (nblk * blockDim.x), which
// walks each fill directly from its first such block.
__device__ __forceinline__ void noise_fill_share(const NoiseFill* fills, int count, PhiloxKey key, uint32_t step_lo,
                                                 long long blk, long long nblk) {
  const unsigned long long stride = static_cast<unsigned long long>(nblk) * blockDim.x;
  const unsigned long long j0 = static_cast<unsigned long long>(blk) * blockDim.x + threadIdx.x;
  unsigned long long seg_begin = 0;  // global index of the fill's first block
  for (int q = 0; q < count; ++q) {
    const NoiseFill f = fills[q];
    const unsigned long long nb = (f.total + 3) / 4;
    // This thread's first global block at or after seg_begin, as an index into the fill.
    const unsigned long long first =
        j0 >= seg_begin ? j0 - seg_begin : (stride - (seg_begin - j0) % stride) % stride;
    for (unsigned long long jj = first; jj < nb; jj += stride) {
      double z[4] = {0.0, 0.0, 0.0, 0.0};
      if (f.std_dev != 0.0)
        normals4(static_cast<uint32_t>(jj), f.layer_id, step_lo, kStreamNoise, key, z, NoiseTablesGlobal{}, f.std_dev);
      const unsigned long long k0 = 4 * jj;
      if (k0 + 3 < f.total) {
        if (!DP_DCHECK(in_buffer(static_cast<long long>(k0), 4, static_cast<long long>(f.total)), 28u, nullptr)) break;
        *reinterpret_cast<float4*>(f.G + k0) = make_float4(__double2float_rn(z[0]), __double2float_rn(z[1]),
                                                           __double2float_rn(z[2]), __double2float_rn(z[3]));
      } else {
        for (int e = 0; e < 4 && k0 + e < f.total; ++e) f.G[k0 + e] = __double2float_rn(z[e]);
      }
    }
    seg_begin += nb;
  }
}

__global__ void __launch_bounds__(256, 4) scale_rows_bf16_kernel(const __nv_bfloat16* __restrict__ in,
                                       __nv_bfloat16* __restrict__ out, long long rows, int cols,
                                       int T, NormSource src, PartialsRef pr, float C, NoiseFill fill,
                                       PhiloxKey key, StepRef step) {
  griddep_enter();
  scale_rows_body(in, out, rows, cols, T, src, pr, C, blockIdx.x, gridDim.x);
  if (fill.G != nullptr) noise_fill_share(&fill, 1, key, step.get(), blockIdx.x, gridDim.x);
}

// The row scalings of several layers in one launch (a per-layer block step scales every
// layer's narrower operand after all the norm passes): segment q takes blocks
// [first_block, first_block + blocks) of the grid and is scaled as scale_rows_bf16_kernel
// would with that many blocks, each block summing its samples' norm partials itself.
constexpr int kMaxScaleSegments = 16;
struct ScaleSegment {
  const __nv_bfloat16* in;
  __nv_bfloat16* out;
  long long rows;
  int cols;
  PartialsRef pr;   // pr.partials null: the clip factors come from src
  NormSource src;
  float C;
  int first_block, blocks;
};
struct ScaleBatch {
  ScaleSegment seg[kMaxScaleSegments];
  int count;
  int T;
  NoiseFill fill[kMaxScaleSegments];  // noise for the one-wave sums that follow, which add to it
  int fills;
  PhiloxKey key;
  StepRef step;
};

__global__ void __launch_bounds__(256, 4) scale_rows_bf16_batch_kernel(ScaleBatch b) {
  griddep_enter();
  int q = 0;
  while (q + 1 < b.count && static_cast<int>(blockIdx.x) >= b.seg[q + 1].first_block) ++q;
  const ScaleSegment& sg = b.seg[q];
  if (!DP_DCHECK(static_cast<int>(blockIdx.x) - sg.first_block < sg.blocks, 27u, nullptr)) return;
  scale_rows_body(sg.in, sg.out, sg.rows, sg.cols, b.T, sg.src, sg.pr, sg.C, blockIdx.x - sg.first_block, sg.blocks);
  if (b.fills > 0) noise_fill_share(b.fill, b.fills, b.key, b.step.get(), blockIdx.x, gridDim.x);
}

// The eight noise values of elements 8 v2 .. 8 v2 + 7 (two Philox blocks), each rounded to
// fp32 once, scaled by the std.
template <class Tab>
__device__ __forceinline__ void noise8_f32(uint32_t blk0, uint32_t layer_id, uint32_t step_lo, PhiloxKey key,
                                           const Tab& tab, double std_dev, float (&n)[8]) {
  double z[8];
  normals4(blk0, layer_id, step_lo, kStreamNoise, key, *reinterpret_cast<double(*)[4]>(z), tab, std_dev);
  normals4(blk0 + 1u, layer_id, step_lo, kStreamNoise, key, *reinterpret_cast<double(*)[4]>(z + 4), tab, std_dev);
#pragma unroll
  for (int q = 0; q < 8; ++q) n[q] = __double2float_rn(z[q]);
}

// The last step of clipped sums split over K: out[e] = fp32(o + std z_e + sum_k scratch[k][e]),
// added in fp64 (the split partials in split order) and rounded once, where o is what out
// holds (the caller's accumulator, or noise written by a row-scaling launch) when read_out,
// else 0, and z_e is the output's noise (stream 0 under the layer's counter; none at std 0).
// The result is the same whatever order the split units ran in, and the noise goes on the
// finished sum as in an unsplit epilogue.  Segments are walked as in noise_fill_share: global
// vector j of their concatenation goes to thread j mod (grid size); vector j of a segment is
// its Philox block j.
constexpr int kMaxCombineSegments = 8;
struct CombineSegment {
  float* out;
  const float* scratch;     // [splits][elems]
  unsigned long long elems;  // a multiple of 4
  int splits;
  int read_out;
  double std_dev;            // 0: no noise
  uint32_t layer_id;
};
struct CombineBatch {
  CombineSegment seg[kMaxCombineSegments];
  int count;
  PhiloxKey key;
  StepRef step;
};

__global__ void __launch_bounds__(256, 4) combine_splits_kernel(CombineBatch b) {
  griddep_enter();
  const unsigned long long stride = static_cast<unsigned long long>(gridDim.x) * blockDim.x;
  const unsigned long long j0 = static_cast<unsigned long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint32_t step_lo = b.step.get();
  unsigned long long seg_begin = 0;
  for (int q = 0; q < b.count; ++q) {
    const CombineSegment sg = b.seg[q];
    const unsigned long long nv = sg.elems / 4;
    const unsigned long long first =
        j0 >= seg_begin ? j0 - seg_begin : (stride - (seg_begin - j0) % stride) % stride;
    // One vector an iteration: the output and the partials are read before any add, and the
    // noise is formed while they land.  (Two vectors an iteration kept more loads in flight per
    // thread but took 80 registers, 3 blocks per SM, and left a tail of one iteration in
    // three: GPT-2 14.8 against 13.0 us at 64 registers and 4 blocks.)
    constexpr int kV = 1;
    for (unsigned long long v = first; v < nv; v += kV * stride) {
      float4 o[kV], p0[kV], p1[kV];
#pragma unroll
      for (int u = 0; u < kV; ++u) {
        const unsigned long long vu = v + u * stride;
        if (vu >= nv) break;
        o[u] = sg.read_out ? __ldcs(reinterpret_cast<const float4*>(sg.out) + vu) : make_float4(0.f, 0.f, 0.f, 0.f);
        p0[u] = __ldcs(reinterpret_cast<const float4*>(sg.scratch) + vu);
        p1[u] = sg.splits > 1 ? __ldcs(reinterpret_cast<const float4*>(sg.scratch + sg.elems) + vu)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < kV; ++u) {
        const unsigned long long vu = v + u * stride;
        if (vu >= nv) break;
        if (!DP_DCHECK(in_buffer(static_cast<long long>(4 * vu), 4, static_cast<long long>(sg.elems)), 32u, nullptr))
          break;
        double a[4] = {0.0, 0.0, 0.0, 0.0};
        if (sg.std_dev != 0.0)
          normals4(static_cast<uint32_t>(vu), sg.layer_id, step_lo, kStreamNoise, b.key, a, NoiseTablesGlobal{},
                   sg.std_dev);
        a[0] += o[u].x; a[1] += o[u].y; a[2] += o[u].z; a[3] += o[u].w;
        a[0] += p0[u].x; a[1] += p0[u].y; a[2] += p0[u].z; a[3] += p0[u].w;
        a[0] += p1[u].x; a[1] += p1[u].y; a[2] += p1[u].z; a[3] += p1[u].w;
        for (int k = 2; k < sg.splits; ++k) {
          const float4 pk = __ldcs(reinterpret_cast<const float4*>(sg.scratch + k * sg.elems) + vu);
          a[0] += pk.x; a[1] += pk.y; a[2] += pk.z; a[3] += pk.w;
        }
        reinterpret_cast<float4*>(sg.out)[vu] = make_float4(static_cast<float>(a[0]), static_cast<float>(a[1]),
                                                           static_cast<float>(a[2]), static_cast<float>(a[3]));
      }
    }
    seg_begin += nv;
  }
}

// out[e] = fp32(sum_i c_i Gs[i][e] + std * z_e) over the per-sample bf16 gradients that the
// explicit-store pass left in the workspace: the clipped sum without forming any G_i again.
// This is the kernel for B > 8 samples (smaller batches take clip_reduce_tma_kernel below).
//
// Each thread owns 8 consecutive elements: two Philox blocks and four independent fp64
// Box-Muller pairs.  The noise sigma C z is rounded to fp32 once and added to the fp32 sum
// (one conversion an element instead of two; the result is within 1 ulp of the fp64 sum
// rounded once).  A persistent grid of two blocks per SM; each block stages the Box-Muller
// tables in shared memory once.
//
// STAGED: the Box-Muller tables are staged in shared memory (32 KB); otherwise they are read
// through the read-only cache and the block needs only the clip factors' few bytes of shared
// memory, so it fits on an SM beside a running tensor-core CTA (the overlapped block step).
// BU > 0: exactly BU samples, unrolled: each thread issues all BU loads of its 8 elements,
// computes their noise while the loads are in flight, then forms the weighted sum.  BU = 0: a
// runtime loop over B samples.
// With pr.partials (BU > 0 only), warp i of every block first sums sample i's norm partials
// (the fixed-order routine, so every block gets the same bits) and block 0 writes norm2 /
// norms_out / c_out, as the bulk-copy reduce does: no separate partials kernel.
template <bool STAGED, int BU>
__global__ void __launch_bounds__(256, 2) clip_reduce_kernel(
    const __nv_bfloat16* __restrict__ Gs, int B, long long mn, NormSource src, PartialsRef pr, float C,
    float* __restrict__ out, double noise_std, PhiloxKey key, uint32_t layer_id, StepRef step) {
  griddep_enter();
  const uint32_t step_lo = step.get();
  extern __shared__ double2 reduce_smem[];  // noise tables (STAGED), then the cached clip factors
  float* c_smem = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(reduce_smem) + (STAGED ? kNoiseSharedBytes : 0));
  const int cached = B < kReduceCachedSamples ? B : kReduceCachedSamples;
  if (BU > 0 && pr.partials != nullptr) {
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int i = warp; i < BU; i += static_cast<int>(blockDim.x / 32)) {
      const float n2 = warp_norm2_from_partials(pr.partials, pr.stride, pr.count, i, lane);
      if (lane == 0) {
        const float n = sqrtf(n2);
        c_smem[i] = clip_factor(n, C);
        if (blockIdx.x == 0) {
          if (pr.norm2) pr.norm2[i] = n2;
          if (pr.norms_out) pr.norms_out[i] = n;
          if (pr.c_out) pr.c_out[i] = c_smem[i];
        }
      }
    }
  } else {
    for (int i = threadIdx.x; i < cached; i += blockDim.x) c_smem[i] = clip_factor(src.norm(i), C);
  }
  if (STAGED && noise_std != 0.0) stage_noise_tables(reduce_smem);
  __syncthreads();
  using Tab = typename std::conditional<STAGED, NoiseTablesShared, NoiseTablesGlobal>::type;
  Tab tab;
  if constexpr (STAGED) tab = NoiseTablesShared{reduce_smem};
  const long long nvec = mn / 8;  // 16-byte vectors per sample
  for (long long v = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; v < nvec;
       v += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4* g = reinterpret_cast<const uint4*>(Gs) + v;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    float z[8];
    if constexpr (BU > 0) {
      uint4 pk[BU];
#pragma unroll
      for (int i = 0; i < BU; ++i) pk[i] = __ldcs(g + static_cast<long long>(i) * nvec);
      if (noise_std != 0.0)
        noise8_f32(static_cast<uint32_t>(2 * v), layer_id, step_lo, key, tab, noise_std, z);
#pragma unroll
      for (int i = 0; i < BU; ++i) {
        const float c = c_smem[i];
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&pk[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(hv[e]);
          acc[2 * e] = fmaf(c, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(c, f.y, acc[2 * e + 1]);
        }
      }
    } else {
      for (int i = 0; i < B; ++i) {
        const float c = i < cached ? c_smem[i] : clip_factor(src.norm(i), C);
        const uint4 pk = __ldcs(g + static_cast<long long>(i) * nvec);
        const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&pk);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(hv[e]);
          acc[2 * e] = fmaf(c, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(c, f.y, acc[2 * e + 1]);
        }
      }
      if (noise_std != 0.0)
        noise8_f32(static_cast<uint32_t>(2 * v), layer_id, step_lo, key, tab, noise_std, z);
    }
    if (noise_std != 0.0) {
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = acc[q] + z[q];
    }
    if (!DP_DCHECK(in_buffer(8 * v, 8, mn), 23u, nullptr)) break;
    // Streaming stores (evict first), like the loads: beside a tensor-core pass they should not
    // push that pass's operand tiles out of L2.
    float4* o = reinterpret_cast<float4*>(out) + 2 * v;
    __stcs(o, make_float4(acc[0], acc[1], acc[2], acc[3]));
    __stcs(o + 1, make_float4(acc[4], acc[5], acc[6], acc[7]));
  }
}

// Warp-specialised variant of clip_reduce_kernel for B <= 8 samples.
//   warp 0      : one lane streams chunks of kReduceChunk elements of every sample's bf16
//                 tiles into a ring of shared-memory stages with 1-D bulk async copies;
//   warps 1..23 : each thread owns 8 consecutive elements of a chunk.  It first computes
//                 their fp64 noise, which needs no data, then waits for the stage, forms
//                 sum_i c_i G_i from shared memory, adds the noise and stores fp32.
// The copies are issued by one thread with a few instructions each, so HBM stays busy while
// the compute warps spend their issue slots on the noise.  Waits are bounded as in the
// tensor-core engine.
constexpr int kReduceComputeWarps = 23;  // 24 warps at 80 registers fill the register file
constexpr int kReduceChunk = 8 * 32 * kReduceComputeWarps;
static_assert(kReduceComputeWarps >= 8, "one compute warp per sample sums the norm partials");

template <int BU>
struct ReduceTmaConfig {
  static constexpr int STAGE_BYTES = BU * kReduceChunk * 2;
  static constexpr int STAGES = (196608 / STAGE_BYTES) < 8 ? (196608 / STAGE_BYTES) : 8;
  static constexpr int THREADS = 32 * (1 + kReduceComputeWarps);
  static constexpr int TABLE_OFFSET = STAGES * STAGE_BYTES + 256;  // after the barriers
  static constexpr int SMEM_BYTES = 1024 + TABLE_OFFSET + kNoiseSharedBytes;
  static_assert(SMEM_BYTES <= 232448, "dynamic shared memory per block");
  static_assert(kReduceChunk == 8 * 32 * kReduceComputeWarps, "8 elements per compute thread");
};

template <int BU>
__global__ void __launch_bounds__(ReduceTmaConfig<BU>::THREADS, 1) clip_reduce_tma_kernel(
    const __nv_bfloat16* __restrict__ Gs, long long mn, NormSource src, PartialsRef pr, float C,
    float* __restrict__ out, double noise_std, PhiloxKey key, uint32_t layer_id, StepRef step,
    uint32_t* status) {
  griddep_enter();
  const uint32_t step_lo = step.get();
  using Cfg = ReduceTmaConfig<BU>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::STAGES * Cfg::STAGE_BYTES);
  uint64_t* empty = full + Cfg::STAGES;
  float* c_s = reinterpret_cast<float*>(empty + Cfg::STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(c_s + 8);
  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::STAGES; ++s) {
      mbar_init(smem_addr(full + s), 1);
      mbar_init(smem_addr(empty + s), kReduceComputeWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (pr.partials == nullptr && threadIdx.x < BU) c_s[threadIdx.x] = clip_factor(src.norm(threadIdx.x), C);
  double2* tab_s = reinterpret_cast<double2*>(smem + Cfg::TABLE_OFFSET);
  if (noise_std != 0.0) stage_noise_tables(tab_s);
  __syncthreads();
  const NoiseTablesShared tab{tab_s};
  const long long chunks = (mn + kReduceChunk - 1) / kReduceChunk;
  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      for (long long ch = blockIdx.x; ch < chunks; ch += gridDim.x) {
        if (!mbar_wait_bounded(smem_addr(empty + stage), phase ^ 1u, abort_flag, status, 21u)) break;
        const long long e0 = ch * kReduceChunk;
        const long long n = (mn - e0) < kReduceChunk ? (mn - e0) : kReduceChunk;  // multiple of 8
        const uint32_t bytes = static_cast<uint32_t>(n * 2);
        const uint32_t bar = smem_addr(full + stage);
        if (DP_DCHECK(n > 0 && n % 8 == 0 && in_buffer((BU - 1) * mn + e0, n, BU * mn), 24u, status)) {
          mbar_arrive_expect_tx(bar, BU * bytes);
          const uint32_t dst = smem_addr(smem + stage * Cfg::STAGE_BYTES);
#pragma unroll
          for (int i = 0; i < BU; ++i)
            bulk_load(dst + i * kReduceChunk * 2, Gs + static_cast<long long>(i) * mn + e0, bytes, bar);
        } else {
          mbar_arrive(bar);  // no copy: the stage completes empty, nothing is left in flight
        }
        if (++stage == Cfg::STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else {
    const int t = threadIdx.x - 32;  // 0 .. 32 * kReduceComputeWarps - 1
    if (pr.partials != nullptr && warp - 1 < BU) {
      // Warp 1 + i sums sample i's norm partials while the producer starts streaming.
      const int i = warp - 1;
      const float n2 = warp_norm2_from_partials(pr.partials, pr.stride, pr.count, i, static_cast<int>(lane));
      const float n = sqrtf(n2);
      if (lane == 0) {
        c_s[i] = clip_factor(n, C);
        if (blockIdx.x == 0) {
          if (pr.norm2) pr.norm2[i] = n2;
          if (pr.norms_out) pr.norms_out[i] = n;
          if (pr.c_out) pr.c_out[i] = c_s[i];
        }
      }
    }
    bool need_c = (pr.partials != nullptr);  // c_s is read first after the first chunk's noise
    int stage = 0;
    uint32_t phase = 0;
    for (long long ch = blockIdx.x; ch < chunks; ch += gridDim.x) {
      const long long e = ch * kReduceChunk + 8 * t;  // first of this thread's 8 elements
      float z[8];
      if (noise_std != 0.0 && e < mn)
        noise8_f32(static_cast<uint32_t>(e >> 2), layer_id, step_lo, key, tab, noise_std, z);
      if (need_c) {
        // Every compute warp passes here in its first iteration (the trip count is the same
        // for all of them), before any wait that could end the loop early.
        asm volatile("bar.sync 1, %0;" ::"r"(32 * kReduceComputeWarps) : "memory");
        need_c = false;
      }
      if (!mbar_wait_bounded(smem_addr(full + stage), phase, abort_flag, status, 22u)) break;
      if (e < mn) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        const uint8_t* base = smem + stage * Cfg::STAGE_BYTES + 16 * t;
#pragma unroll
        for (int i = 0; i < BU; ++i) {
          const uint4 pk = *reinterpret_cast<const uint4*>(base + i * kReduceChunk * 2);
          const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&pk);
          const float c = c_s[i];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(hv[q]);
            acc[2 * q] = fmaf(c, f.x, acc[2 * q]);
            acc[2 * q + 1] = fmaf(c, f.y, acc[2 * q + 1]);
          }
        }
        if (noise_std != 0.0) {
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[q] = acc[q] + z[q];
        }
        if (DP_DCHECK(in_buffer(e, 8, mn), 25u, status)) {
          float4* o = reinterpret_cast<float4*>(out + e);
          o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
          o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(empty + stage));
      if (++stage == Cfg::STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
  }
  __syncthreads();
}

// Projected Adam in r-space: g = scale R; m <- b1 m + (1 - b1) g; v <- b2 v + (1 - b2) g^2;
// U = (m / bc1) / (sqrt(v / bc2) + eps), written in bf16 for the tensor-core back-projection
// (bc1 = 1 - b1^t, bc2 = 1 - b2^t).  Four elements per thread.
__global__ void adam_rspace_kernel(const float* __restrict__ R, float* __restrict__ m, float* __restrict__ v,
                                   __nv_bfloat16* __restrict__ U, long long n, float scale, float b1, float b2,
                                   float eps, float bc1, float bc2) {
  griddep_enter();
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; 4 * q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 r4 = reinterpret_cast<const float4*>(R)[q];
    float4 m4 = reinterpret_cast<float4*>(m)[q];
    float4 v4 = reinterpret_cast<float4*>(v)[q];
    const float gr[4] = {r4.x, r4.y, r4.z, r4.w};
    float* mm = &m4.x;
    float* vv = &v4.x;
    float u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float g = scale * gr[e];
      mm[e] = fmaf(b1, mm[e], (1.0f - b1) * g);
      vv[e] = fmaf(b2, vv[e], (1.0f - b2) * g * g);
      u[e] = (mm[e] / bc1) / (sqrtf(vv[e] / bc2) + eps);
    }
    reinterpret_cast<float4*>(m)[q] = m4;
    reinterpret_cast<float4*>(v)[q] = v4;
    __nv_bfloat162 lo = __floats2bfloat162_rn(u[0], u[1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(u[2], u[3]);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(U)[q] = pk;
  }
}

// Failure-detection self-test: one thread waits, with the bounded wait every pipeline uses,
// on an mbarrier that nothing ever arrives at.  After `limit_ns` the wait gives up, records
// its site (code 99) in the status word and the kernel returns; the GPU stays usable.
__global__ void wait_timeout_selftest_kernel(uint32_t* status, unsigned long long limit_ns) {
  griddep_enter();
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(smem_addr(&bar), 1);
  fence_mbar_init();
  mbar_wait_bounded(smem_addr(&bar), 0u, &abort_flag, status, 99u, limit_ns);
}

// ------------------------------------------------------------------------------ fp32 path
// Tiles of 32 rows (a) x 32 columns (b); thread (ty, tx) owns row a0 + ty and the four
// consecutive columns b0 + 4 tx .. b0 + 4 tx + 3, so one Philox block feeds its noise.
constexpr int kF32Tile = 32;

// norm2[i] += sum over this tile of G_i[a, b]^2, G_i = X_i^T dY_i accumulated in fp64.
__global__ void __launch_bounds__(256) f32_norm_kernel(const float* __restrict__ X,
                                                       const float* __restrict__ dY, int T, int m,
                                                       int n, double* __restrict__ norm2) {
  griddep_enter();
  __shared__ float xs[kF32Tile][kF32Tile + 1];  // [t][a]
  __shared__ float ds[kF32Tile][kF32Tile + 1];  // [t][b]
  __shared__ double red[8];
  const int i = blockIdx.z;
  const int a0 = blockIdx.y * kF32Tile, b0 = blockIdx.x * kF32Tile;
  const int tx = threadIdx.x % 8, ty = threadIdx.x / 8;
  const float* Xi = X + static_cast<long long>(i) * T * m;
  const float* Di = dY + static_cast<long long>(i) * T * n;
  double acc[4] = {0, 0, 0, 0};
  for (int t0 = 0; t0 < T; t0 += kF32Tile) {
    for (int e = threadIdx.x; e < kF32Tile * kF32Tile; e += 256) {
      const int tt = e / kF32Tile, cc = e % kF32Tile;
      const int t = t0 + tt;
      xs[tt][cc] = (t < T && a0 + cc < m) ? Xi[static_cast<long long>(t) * m + a0 + cc] : 0.f;
      ds[tt][cc] = (t < T && b0 + cc < n) ? Di[static_cast<long long>(t) * n + b0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < kF32Tile; ++tt) {
      const double x = xs[tt][ty];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fma(x, static_cast<double>(ds[tt][4 * tx + q]), acc[q]);
    }
    __syncthreads();
  }
  double ss = acc[0] * acc[0] + acc[1] * acc[1] + acc[2] * acc[2] + acc[3] * acc[3];
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0;
    for (int w = 0; w < 8; ++w) s += red[w];
    atomicAdd(norm2 + i, s);
  }
}

// S[a, b] = sum_t c_{t / T} X[t, a] dY[t, b] over all N = B*T tokens (fp64 accumulation),
// then out = fp32(S + std * z) (mode store) or out += fp32(S) (mode add).
__global__ void __launch_bounds__(256) f32_clipsum_kernel(
    const float* __restrict__ X, const float* __restrict__ dY, long long N, int T, int m, int n,
    NormSource src, float C, float* __restrict__ out, int add_mode, double noise_std, PhiloxKey key,
    uint32_t layer_id, StepRef step) {
  griddep_enter();
  const uint32_t step_lo = step.get();
  __shared__ float xs[kF32Tile][kF32Tile + 1];
  __shared__ float ds[kF32Tile][kF32Tile + 1];
  __shared__ float cs[kF32Tile];
  const int a0 = blockIdx.y * kF32Tile, b0 = blockIdx.x * kF32Tile;
  const int tx = threadIdx.x % 8, ty = threadIdx.x / 8;
  double acc[4] = {0, 0, 0, 0};
  for (long long t0 = 0; t0 < N; t0 += kF32Tile) {
    if (threadIdx.x < kF32Tile) {
      const long long t = t0 + threadIdx.x;
      cs[threadIdx.x] = (t < N) ? clip_factor(src.norm(static_cast<int>(t / T)), C) : 0.f;
    }
    for (int e = threadIdx.x; e < kF32Tile * kF32Tile; e += 256) {
      const int tt = e / kF32Tile, cc = e % kF32Tile;
      const long long t = t0 + tt;
      xs[tt][cc] = (t < N && a0 + cc < m) ? X[t * m + a0 + cc] : 0.f;
      ds[tt][cc] = (t < N && b0 + cc < n) ? dY[t * n + b0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < kF32Tile; ++tt) {
      const double x = static_cast<double>(cs[tt]) * static_cast<double>(xs[tt][ty]);
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fma(x, static_cast<double>(ds[tt][4 * tx + q]), acc[q]);
    }
    __syncthreads();
  }
  const int a = a0 + ty, b = b0 + 4 * tx;
  if (a >= m || b >= n) return;  // n is a multiple of 4: the four columns are all in range
  float* dst = out + static_cast<long long>(a) * n + b;
  if (add_mode) {
    for (int q = 0; q < 4; ++q) dst[q] += static_cast<float>(acc[q]);
    return;
  }
  if (noise_std != 0.0) {
    const unsigned long long k = static_cast<unsigned long long>(a) * n + b;
    double z[4];
    normals4(static_cast<uint32_t>(k >> 2), layer_id, step_lo, kStreamNoise, key, z, NoiseTablesGlobal{}, noise_std);
    for (int q = 0; q < 4; ++q) acc[q] += z[q];
  }
  for (int q = 0; q < 4; ++q) dst[q] = static_cast<float>(acc[q]);
}

// Z[t, j] = fp32(sum_b dY[t, b] P[b, j]) in fp64, one thread per output.
__global__ void f32_project_kernel(const float* __restrict__ dY, const float* __restrict__ P,
                                   float* __restrict__ Z, long long N, int n, int r) {
  griddep_enter();
  const long long total = N * r;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = e / r;
    const int j = static_cast<int>(e % r);
    double acc = 0;
    for (int b = 0; b < n; ++b)
      acc = fma(static_cast<double>(dY[t * n + b]), static_cast<double>(P[static_cast<long long>(b) * r + j]), acc);
    Z[e] = static_cast<float>(acc);
  }
}

}  // namespace dpclip
