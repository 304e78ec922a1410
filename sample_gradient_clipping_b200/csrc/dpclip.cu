// Host side of the C ABI declared in include/dpclip.h: argument checks, workspace layout,
// TMA tensor-map encoding, norm-method selection and the launches that make up each call.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "dpclip.h"
#include "launch_profiler.h"
#include "nvtx_range.h"
#include "rng.cuh"
#include "simt.cuh"
#include "umma_gemm.cuh"
#include "umma_gemm_2sm.cuh"

using namespace dpclip;

namespace {

thread_local char g_cuda_error[256] = "";

dp_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return DP_ERR_CUDA;
}

#define DP_CUDA(call)                                  \
  do {                                                 \
    cudaError_t e_ = (call);                           \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

// Every kernel is launched with programmatic stream serialization: it may be scheduled while
// the previous kernel in the stream drains, runs its local prologue, and waits for that kernel
// (griddep_wait in ptx.cuh) before its first access to global memory.  This hides most of the
// launch gap between the short kernels of a step.
// Host-side fault injection (dp_selftest_fail_launches): launches to let through before the
// injected failures, the failures left, and the error they report.  Nothing is enqueued for a
// failed launch, as when the runtime refuses one.
std::atomic<long long> g_inject_skip{0};
std::atomic<long long> g_inject_count{0};
std::atomic<int> g_inject_error{0};

cudaError_t injected_launch_error() {
  if (g_inject_count.load(std::memory_order_relaxed) <= 0) return cudaSuccess;
  if (g_inject_skip.fetch_sub(1) > 0) return cudaSuccess;
  if (g_inject_count.fetch_sub(1) <= 0) return cudaSuccess;
  return static_cast<cudaError_t>(g_inject_error.load());
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args&&... args) {
  const cudaError_t injected = injected_launch_error();
  if (injected != cudaSuccess) return injected;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define DP_LAUNCH(what, ...)                             \
  do {                                                   \
    cudaError_t e_ = launch_kernel(__VA_ARGS__);         \
    if (e_ == cudaSuccess) e_ = cudaGetLastError();      \
    if (e_ != cudaSuccess) return cuda_fail(e_, what);   \
  } while (0)

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    counts[dev] = c;
  }
  return counts[dev];
}

// ---------------------------------------------------------------- shape rules
struct Shape {
  int B, T, m, n, r;  // r = 0: unprojected
  dp_dtype dt;
  long long N() const { return static_cast<long long>(B) * T; }
  int ne() const { return r > 0 ? r : n; }  // width of the clip-space gradient
};

bool valid_dtype(dp_dtype dt) { return dt == DP_F32 || dt == DP_BF16; }

bool valid_shape(const Shape& s) {
  if (!valid_dtype(s.dt)) return false;
  if (s.B < 1 || s.T < 1 || s.m < 1 || s.n < 1 || s.r < 0) return false;
  const int q = (s.dt == DP_BF16) ? 8 : 4;
  if (s.m % q || s.n % q || s.r % q) return false;
  if (s.N() >= (1ll << 31)) return false;
  if (static_cast<long long>(s.m) * s.ne() > (1ll << 34)) return false;
  if (s.dt == DP_F32 && s.B > 65535) return false;
  return true;
}

struct WsLayout {
  size_t status = 0, norm2 = 0, c = 0, partials = 0, scaled = 0, z = 0, p = 0, gs = 0, total = 0;
  size_t fixup = 0;     // a clipped sum split over K: its split partials (0: none)
  int fixup_splits = 0;  // splits that region holds
  int partial_stride = 0;  // floats per sample
};

// Per-warp norm partial slots per sample: 4 per unit of the explicit (128-wide tiles at most)
// or ghost (upper-triangular 128-token pairs) norm kernel, whichever has more units.
int partial_slots(const Shape& s) {
  const long long expl = 4ll * ((s.m + 127) / 128) * ((s.ne() + 127) / 128);
  const long long pair = 8ll * ((s.m + 255) / 256) * ((s.ne() + 255) / 256);  // two-SM tiles
  const long long tt = (s.T + 127) / 128;
  const long long ghost = 4 * tt * (tt + 1) / 2;
  long long most = expl > ghost ? expl : ghost;
  if (pair > most) most = pair;
  return static_cast<int>(most);
}

// The ghost units (one per sample and upper-triangular pair of 128-token blocks) that are cut
// in parts, and how.  The ghost kernel is persistent, so the units of the last, partial wave
// on the SMs would run alone while the other SMs wait; each of them is cut into parts over the
// K of the deeper Gram (X over d_in, or dY over the clip-space width) when that Gram is at
// least twice as deep as the other (each part still forms the other Gram whole).  With fewer
// units than SMs every unit is such a tail unit.  A function of the shape alone (and the SM
// count): every launch that forms this linear's ghost norm (alone, grouped with other linears,
// or sharing its X Gram) cuts the same units the same way and writes the same partials, so the
// norms are bitwise the same whichever entry point formed them.  At most
// partial_slots(s) / (4 pairs) parts, so the partials fit every workspace layout.
struct GhostSplit {
  int full;     // units [0, full) whole
  int parts;    // parts of each later unit (1: none)
  bool over_x;  // parts of the X Gram's K (else of the dY Grams')
};
GhostSplit ghost_split(const Shape& s) {
  const int t_tiles = (s.T + 127) / 128;
  const int pairs = t_tiles * (t_tiles + 1) / 2;
  const int units = s.B * pairs;
  const int kx = (s.m + 63) / 64, k1 = (s.ne() + 63) / 64;
  const int sms = sm_count();
  const int tail = units % sms;
  const bool over_x = kx >= 2 * k1;
  if (tail == 0 || !(over_x || k1 >= 2 * kx)) return GhostSplit{units, 1, false};
  const int kd = over_x ? kx : k1;
  int parts = std::min(sms / tail, std::min(kd, partial_slots(s) / (4 * pairs)));
  if (parts < 2) return GhostSplit{units, 1, false};
  parts = ceil_div(kd, ceil_div(kd, parts));  // every part non-empty
  return GhostSplit{units - tail, parts, over_x};
}

// Units of a ghost launch for one linear under its split, and its partial slots per sample.
int ghost_units(const GhostSplit& g, int units) { return g.parts > 1 ? g.full + (units - g.full) * g.parts : units; }

struct ClipSumPlan {
  bool pair;
  int bn, m_tiles, n_tiles, k_blocks, k_blocks_per_split, splits;
};

ClipSumPlan clipsum_plan(const Shape& s) {
  ClipSumPlan c;
  const int ne = s.ne();
  c.bn = ne <= 128 ? 128 : 256;
  // 256 x 256 tiles on SM pairs when both output dimensions fill them: half the operand
  // traffic per SM of a 128 x 256 one-SM tile.
  c.pair = (s.m >= 256 && ne >= 256);
  c.m_tiles = c.pair ? ceil_div(s.m, 256) : ceil_div(s.m, 128);
  c.n_tiles = ceil_div(ne, c.bn);
  c.k_blocks = ceil_div(s.N(), 64);
  // Measured and left out for GPT-2's 768x3072 output (58 us with 256x256 pair tiles split in
  // two): unsplit 256x128 pair tiles (72 on 74 pairs) 96 us, unsplit one-SM 128x128 tiles (144
  // on 148 SMs) 99 us.  Both read 1.5-2x the operand bytes per flop from L2.
  const int slots = c.pair ? sm_count() / 2 : sm_count();  // CTAs (or pairs) that run at once
  const int tiles = c.m_tiles * c.n_tiles;
  int splits = 1;
  if (tiles < slots) {
    splits = slots / tiles;
    const int max_splits = c.k_blocks / 4 > 0 ? c.k_blocks / 4 : 1;
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) splits = 1;
  }
  c.k_blocks_per_split = ceil_div(c.k_blocks, splits);
  c.splits = ceil_div(c.k_blocks, c.k_blocks_per_split);  // every split non-empty
  return c;
}

// Whether a clipped sum takes its noise from the row-scaling launch before it (which writes
// the noise into the output, each value rounded to fp32 once) instead of from its epilogue or
// its combining launch: when all its units run in one unsplit wave, where the epilogue's fp64
// noise would run after every tile with nothing to hide it (measured on unsplit 256x128 tiles
// of GPT-2's output: 100 against 96 us), or when it is split over K into more splits than the
// workspace holds partials for (`fixup_splits`), so that its splits add by atomics.  The sum
// is then added to the noise.  A sum split over K with its split partials takes its noise in
// the combining launch, on the finished sum.
bool sum_prefills_noise(const ClipSumPlan& c, int fixup_splits) {
  const int slots = c.pair ? sm_count() / 2 : sm_count();
  if (c.splits > 1) return c.splits > fixup_splits;
  return c.m_tiles * c.n_tiles <= slots;
}

// Where a clipped sum split over K keeps its split partials (kOutSplitPartials).
struct FixupRef {
  float* scratch;  // [splits][m][ne] fp32
  int max_splits;  // splits the scratch holds
};

WsLayout ws_layout(const Shape& s, dp_norm_method method) {
  WsLayout L;
  size_t off = 256;  // status word(s)
  // A bf16 clipped sum split over K keeps its split partials at the end.  Every method's
  // layout holds them, so that the gradients-once layout stays the largest
  // (dp_clip_accumulate runs the clipped sum whatever method sized the workspace).
  const ClipSumPlan cp = clipsum_plan(s);
  const bool fix = s.dt == DP_BF16 && cp.splits > 1;
  L.norm2 = off;
  off += align256(static_cast<size_t>(s.B) * 8);
  L.c = off;
  off += align256(static_cast<size_t>(s.B) * 4);
  const size_t e = (s.dt == DP_BF16) ? 2 : 4;
  if (s.dt == DP_BF16) {
    L.partial_stride = partial_slots(s);
    L.partials = off;
    off += align256(static_cast<size_t>(s.B) * L.partial_stride * 4);
  }
  if (s.dt == DP_BF16) {
    L.scaled = off;
    off += align256(static_cast<size_t>(s.N()) * static_cast<size_t>(s.m < s.ne() ? s.m : s.ne()) * 2);
  }
  if (s.r > 0) {
    L.z = off;
    off += align256(static_cast<size_t>(s.N()) * s.r * e);
    L.p = off;
    off += align256(static_cast<size_t>(s.n) * s.r * e);
  }
  if (method == DP_NORM_ONCE && s.dt == DP_BF16) {
    L.gs = off;  // per-sample gradient tiles, bf16 [B][d_in][ne]
    off += align256(static_cast<size_t>(s.B) * s.m * s.ne() * 2);
  }
  if (fix) {
    L.fixup = off;
    L.fixup_splits = cp.splits;
    off += align256(static_cast<size_t>(cp.splits) * s.m * s.ne() * 4);
  }
  L.total = off;
  return L;
}

// Cost model of one step for each norm method (seconds), a roofline with four corrections
// calibrated on this B200 build:
//   * per-sample tensor-core kernels run over a sample's T tokens per tile; below ~1024
//     tokens their fixed cost per tile shows (measured: half rate at T = 512);
//   * the clipped-sum contraction with its noise epilogue runs at about 65% of the rate of
//     the per-sample pair kernel;
//   * the gradients-once tile stores stream at ~3 TB/s, and its reduce is bound by the HBM
//     stream or by the noise (~2.5e11 normals/s), whichever is slower;
//   * each launch costs ~4 us, which decides the small shapes.
constexpr double kModelFlops = 1.4e15;       // bf16 tensor flop/s (sustained)
constexpr double kModelBytes = 6.5e12;       // HBM byte/s
constexpr double kModelStoreBytes = 3.0e12;  // per-sample tile stores, byte/s
constexpr double kModelNormals = 2.5e11;     // normals/s in the reduce
constexpr double kModelClipSumEff = 0.65;
constexpr double kModelLaunch = 4e-6;        // s per kernel launch

double model_cost(const Shape& s, dp_norm_method m) {
  const double N = static_cast<double>(s.N()), d = s.m, ne = s.ne(), B = s.B;
  const double contraction = 2.0 * N * d * ne / kModelFlops;
  const double per_sample = contraction / std::min(1.0, s.T / 1024.0);
  const double clip_sum = contraction / kModelClipSumEff;
  const double scale_pass = N * (d < ne ? d : ne) * 4.0 / kModelBytes;
  if (m == DP_NORM_GHOST) {
    const double tt = std::ceil(s.T / 128.0);
    return B * tt * (tt + 1) / 2 * 2.0 * 128 * 128 * (d + ne) / kModelFlops + scale_pass + clip_sum +
           4 * kModelLaunch;
  }
  if (m == DP_NORM_EXPLICIT) return per_sample + clip_sum + scale_pass + 4 * kModelLaunch;
  const double store = B * d * ne * 2.0 / kModelStoreBytes;  // written while the MMAs run
  const double reduce = std::max((B * d * ne * 2.0 + d * ne * 4.0) / kModelBytes, d * ne / kModelNormals);
  return std::max(per_sample, store) + reduce + 3 * kModelLaunch;
}

// DPCLIP_NORM=ghost|explicit|once in the environment overrides the cost model for bf16 calls
// with DP_NORM_AUTO (read at every call, so a workspace size query and the call that uses it
// see the same setting); any other value, or none, leaves the choice to the model.
bool env_norm_method(dp_norm_method* out) {
  const char* v = getenv("DPCLIP_NORM");
  if (!v) return false;
  if (!strcmp(v, "ghost")) *out = DP_NORM_GHOST;
  else if (!strcmp(v, "explicit")) *out = DP_NORM_EXPLICIT;
  else if (!strcmp(v, "once")) *out = DP_NORM_ONCE;
  else return false;
  return true;
}

dp_norm_method auto_method(const Shape& s) {
  if (s.dt == DP_F32) return DP_NORM_EXPLICIT;
  dp_norm_method forced;
  if (env_norm_method(&forced)) return forced;
  dp_norm_method best = DP_NORM_GHOST;
  for (dp_norm_method m : {DP_NORM_EXPLICIT, DP_NORM_ONCE})
    if (model_cost(s, m) < model_cost(s, best)) best = m;
  return best;
}

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

dp_status get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    snprintf(g_cuda_error, sizeof(g_cuda_error), "cuTensorMapEncodeTiled unavailable");
    return DP_ERR_CUDA;
  }
  return DP_OK;
}

// bf16 tensor [outer..., inner] with a box of {64 (inner), box_rows, 1...}, 128-byte swizzle.
dp_status encode_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      uint32_t box_rows) {
  cuuint64_t gdim[3], gstride[2];
  cuuint32_t box[3], estr[3] = {1, 1, 1};
  for (int d = 0; d < rank; ++d) gdim[d] = dims[d];
  uint64_t stride = dims[0] * 2;
  for (int d = 1; d < rank; ++d) {
    gstride[d - 1] = stride;
    stride *= dims[d];
  }
  box[0] = 64;
  box[1] = box_rows;
  if (rank == 3) box[2] = 1;
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gdim,
                        gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    snprintf(g_cuda_error, sizeof(g_cuda_error), "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return DP_ERR_CUDA;
  }
  return DP_OK;
}

dp_status map_2d(CUtensorMap* m, const void* base, long long rows, int cols, uint32_t box_rows) {
  const uint64_t d[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  return encode_bf16(m, base, 2, d, box_rows);
}
dp_status map_3d(CUtensorMap* m, const void* base, int B, int T, int cols, uint32_t box_rows) {
  const uint64_t d[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(T), static_cast<uint64_t>(B)};
  return encode_bf16(m, base, 3, d, box_rows);
}

// ---------------------------------------------------------------- engine launches
// Two-SM launch: clusters of 2 CTAs (compile-time cluster dims), one pair per 2 SMs.
template <class Cfg>
dp_status launch_umma_pair(const UmmaParams& p, cudaStream_t stream) {
  static bool configured[64] = {false};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    DP_CUDA(cudaFuncSetAttribute(umma_pair_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES));
    configured[dev] = true;
  }
  if (p.num_units <= 0) return DP_OK;
  const int pairs_avail = sm_count() / 2;
  const int pairs = p.num_units < pairs_avail ? p.num_units : pairs_avail;
  constexpr int kind = Cfg::EPI == kEpiExplicitStore ? kKindExplicitStore
                       : Cfg::EPI == kEpiClipSum     ? kKindClipSum
                                                     : kKindExplicitNorm;
  LaunchScope scope(kind, stream);
  DP_LAUNCH("umma_pair_kernel", umma_pair_kernel<Cfg>, 2 * pairs, Cfg::THREADS, Cfg::SMEM_BYTES, stream, p);
  return DP_OK;
}

template <class Cfg>
dp_status launch_umma(const UmmaParams& p, cudaStream_t stream) {
  static bool configured[64] = {false};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    DP_CUDA(cudaFuncSetAttribute(umma_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES));
    configured[dev] = true;
  }
  if (p.num_units <= 0) return DP_OK;
  const int grid = p.num_units < sm_count() ? p.num_units : sm_count();
  constexpr int kind = Cfg::EPI == kEpiClipSum         ? kKindClipSum
                       : Cfg::EPI == kEpiExplicitNorm  ? kKindExplicitNorm
                       : Cfg::EPI == kEpiExplicitStore ? kKindExplicitStore
                       : Cfg::EPI == kEpiGhostNorm     ? kKindGhostNorm
                       : Cfg::EPI == kEpiAxpy          ? kKindAxpy
                       : Cfg::EPI == kEpiGhostShared   ? kKindGhostShared
                                                       : kKindProject;
  LaunchScope scope(kind, stream);
  DP_LAUNCH("umma_kernel", umma_kernel<Cfg>, grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream, p);
  return DP_OK;
}

template <class Cfg>
dp_status launch_umma_group(const UmmaParams& p, const UmmaGroup& g, cudaStream_t stream) {
  static bool configured[64] = {false};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    DP_CUDA(cudaFuncSetAttribute(umma_group_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 Cfg::SMEM_BYTES));
    configured[dev] = true;
  }
  if (p.num_units <= 0) return DP_OK;
  const int grid = p.num_units < sm_count() ? p.num_units : sm_count();
  LaunchScope scope(Cfg::EPI == kEpiClipSum ? kKindClipSum : Cfg::EPI == kEpiGhostNorm ? kKindGhostNorm : kKindProject,
                    stream);
  DP_LAUNCH("umma_group_kernel", umma_group_kernel<Cfg>, grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream, p, g);
  return DP_OK;
}

UmmaParams base_params(uint32_t* status) {
  UmmaParams p;
  memset(&p, 0, sizeof(p));
  p.status = status;
  return p;
}

int stream_grid(unsigned long long work_items, int threads) {
  const unsigned long long blocks = (work_items + threads - 1) / threads;
  const unsigned long long cap = static_cast<unsigned long long>(sm_count()) * 8;
  return static_cast<int>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

// Per-warp partials of ||X_i^T Z_i||^2 (bf16 operands; Z is dY or the projected dY, ne
// columns) into `partials` ([B][stride]); `count` receives the slots used per sample.  With
// `store`, the explicit tiles of every G_i are also written there in bf16 ([B][d_in][ne]).
dp_status bf16_norms(const Shape& s, const void* X, const void* Z, dp_norm_method method,
                     float* partials, int stride, int* count, uint32_t* status, cudaStream_t stream,
                     __nv_bfloat16* store = nullptr) {
  UmmaParams p = base_params(status);
  p.partials = partials;
  p.partial_stride = stride;
  p.partials_elems = static_cast<long long>(s.B) * stride;
  const int ne = s.ne();
  if (store) p.out_elems = static_cast<long long>(s.B) * s.m * ne;
  if (method == DP_NORM_GHOST) {
    using Cfg = UmmaConfig<128, kEpiGhostNorm>;
    dp_status st;
    if ((st = map_3d(&p.tmA0, X, s.B, s.T, s.m, 128)) != DP_OK) return st;
    p.tmB0 = p.tmA0;
    if ((st = map_3d(&p.tmA1, Z, s.B, s.T, ne, 128)) != DP_OK) return st;
    p.tmB1 = p.tmA1;
    p.t_tiles = ceil_div(s.T, 128);
    p.pairs_per_sample = p.t_tiles * (p.t_tiles + 1) / 2;
    p.k_blocks = ceil_div(s.m, 64);
    p.k_blocks1 = ceil_div(ne, 64);
    const GhostSplit g = ghost_split(s);
    p.split_full_units = g.full;
    p.split_parts = g.parts;
    p.split_over_x = g.over_x ? 1 : 0;
    p.num_units = ghost_units(g, s.B * p.pairs_per_sample);
    *count = 4 * p.pairs_per_sample * g.parts;
    return launch_umma<Cfg>(p, stream);
  }
  dp_status st;
  if ((st = map_3d(&p.tmA0, X, s.B, s.T, s.m, 64)) != DP_OK) return st;
  if ((st = map_3d(&p.tmB0, Z, s.B, s.T, ne, 64)) != DP_OK) return st;
  p.k_blocks = ceil_div(s.T, 64);
  p.out_rows = s.m;
  p.out_cols = ne;
  p.out_bf16 = store;
  if (s.m >= 256 && ne >= 256) {
    // 256 x 256 tiles on SM pairs: half the operand traffic per SM of a 128 x 256 tile.
    p.m_tiles = ceil_div(s.m, 256);
    p.n_tiles = ceil_div(ne, 256);
    p.num_units = s.B * p.m_tiles * p.n_tiles;
    *count = 8 * p.m_tiles * p.n_tiles;
    if (store) return launch_umma_pair<Umma2Config<kEpiExplicitStore>>(p, stream);
    return launch_umma_pair<Umma2Config<kEpiExplicitNorm>>(p, stream);
  }
  p.m_tiles = ceil_div(s.m, 128);
  const int bn = ne <= 128 ? 128 : 256;
  p.n_tiles = ceil_div(ne, bn);
  p.num_units = s.B * p.m_tiles * p.n_tiles;
  *count = 4 * p.m_tiles * p.n_tiles;
  if (store) {
    if (bn == 128) return launch_umma<UmmaConfig<128, kEpiExplicitStore>>(p, stream);
    return launch_umma<UmmaConfig<256, kEpiExplicitStore>>(p, stream);
  }
  if (bn == 128) return launch_umma<UmmaConfig<128, kEpiExplicitNorm>>(p, stream);
  return launch_umma<UmmaConfig<256, kEpiExplicitNorm>>(p, stream);
}

// Ghost-norm partials of k <= 3 linears that read the same X ([B, T, m]) with dY operands
// Zs[j] of equal width ne: one X Gram per token-block pair serves all of them.  Operand j's
// partials go to partials + j * op_stride, laid out as for bf16_norms.
dp_status bf16_norms_ghost_shared(const Shape& s, const void* X, const void* const* Zs, int k,
                                  float* partials, int stride, long long op_stride, int* count,
                                  uint32_t* status, cudaStream_t stream) {
  if (k < 1 || k > kGhostSharedMaxOps) return DP_ERR_INVALID_ARG;
  UmmaParams p = base_params(status);
  p.partials = partials;
  p.partial_stride = stride;
  p.partial_op_stride = op_stride;
  p.partials_elems = (k - 1) * op_stride + static_cast<long long>(s.B) * stride;
  p.ghost_ops = k;
  const int ne = s.ne();
  dp_status st;
  if ((st = map_3d(&p.tmA0, X, s.B, s.T, s.m, 128)) != DP_OK) return st;
  CUtensorMap* maps[kGhostSharedMaxOps] = {&p.tmB0, &p.tmA1, &p.tmB1};
  for (int j = 0; j < k; ++j)
    if ((st = map_3d(maps[j], Zs[j], s.B, s.T, ne, 128)) != DP_OK) return st;
  p.t_tiles = ceil_div(s.T, 128);
  p.pairs_per_sample = p.t_tiles * (p.t_tiles + 1) / 2;
  p.k_blocks = ceil_div(s.m, 64);
  p.k_blocks1 = ceil_div(ne, 64);
  const GhostSplit g = ghost_split(s);  // the split of one member alone: the members' partials are theirs
  p.split_full_units = g.full;
  p.split_parts = g.parts;
  p.split_over_x = g.over_x ? 1 : 0;
  p.num_units = ghost_units(g, s.B * p.pairs_per_sample);
  *count = 4 * p.pairs_per_sample * g.parts;
  return launch_umma<UmmaConfig<128, kEpiGhostShared>>(p, stream);
}

dp_status launch_noise(float* G, unsigned long long total, double std_dev, unsigned long long seed,
                       StepRef step, unsigned layer_id, cudaStream_t stream);

// The combining launch of clipped sums split over K (combine_splits_kernel).
dp_status launch_combine(const CombineBatch& b, cudaStream_t stream) {
  if (b.count == 0) return DP_OK;
  unsigned long long vecs = 0;
  for (int q = 0; q < b.count; ++q) vecs += b.seg[q].elems / 4;
  LaunchScope scope(kKindCombine, stream);
  // One wave of resident blocks (4 per SM at 64 registers): a short launch whose second wave
  // would start after the first one's tail.
  const int grid = std::min(stream_grid(vecs, 256), sm_count() * 4);
  DP_LAUNCH("combine_splits_kernel", combine_splits_kernel, grid, 256, 0, stream, b);
  return DP_OK;
}

// out (+)= A^T Bm over all N rows (A: [N, m], Bm: [N, ne], both bf16, one already scaled by
// c_i), plus noise when noise_std != 0.  `accumulate` = 0 overwrites out.
// With `defer` (a block step), noise that neither the epilogue nor a combining launch adds
// (splits added by atomics) is queued there instead of launched.  With `preset`, out already
// holds the noise (written by the row-scaling launch) and the sum is added to it.
// Split over K with `fx`: each split stores its partial sum, and a combining launch adds the
// noise and them, in split order, to out's contents (accumulate or preset) in fp64 and rounds
// once (kOutSplitPartials).  Without it, the splits add their partial sums into out by fp32
// atomics and the noise follows.
dp_status bf16_clipsum(const Shape& s, const void* A, const void* Bm, float* out, int accumulate,
                       double noise_std, unsigned long long seed, StepRef step,
                       unsigned layer_id, uint32_t* status, cudaStream_t stream,
                       NoiseBatch* defer = nullptr, bool preset = false, const FixupRef* fx = nullptr) {
  UmmaParams p = base_params(status);
  const int ne = s.ne();
  const ClipSumPlan plan = clipsum_plan(s);
  const int BN = plan.bn;
  const bool pair = plan.pair;
  dp_status st;
  if ((st = map_2d(&p.tmA0, A, s.N(), s.m, 64)) != DP_OK) return st;
  if ((st = map_2d(&p.tmB0, Bm, s.N(), ne, 64)) != DP_OK) return st;
  p.m_tiles = plan.m_tiles;
  p.n_tiles = plan.n_tiles;
  p.k_blocks = plan.k_blocks;
  const int tiles = p.m_tiles * p.n_tiles;
  const int splits = plan.splits;
  p.k_blocks_per_split = plan.k_blocks_per_split;
  p.k_splits = splits;
  p.num_units = tiles * splits;
  p.out_rows = s.m;
  p.out_cols = ne;
  p.out_f32 = out;
  p.out_elems = static_cast<long long>(s.m) * ne;
  if (preset && accumulate) return DP_ERR_INVALID_ARG;  // the callers never ask this
  const bool split_partials = splits > 1 && fx && fx->scratch && splits <= fx->max_splits;
  if (split_partials) {
    p.out_mode = kOutSplitPartials;
    p.split_scratch = fx->scratch;
  } else if (splits > 1 || accumulate || preset) {
    p.out_mode = (splits > 1) ? kOutAtomicAdd : kOutAdd;
    if (!accumulate && !preset)
      DP_CUDA(cudaMemsetAsync(out, 0, static_cast<size_t>(s.m) * ne * sizeof(float), stream));
  } else {
    p.out_mode = kOutStore;
  }
  // With `preset` the noise is already in out.  Otherwise an unsplit sum adds it in its
  // epilogue (fp64, rounded once), and a split one after the sum is complete.
  if (preset) noise_std = 0.0;
  const bool fused_noise = (splits == 1);
  p.noise_std = fused_noise ? noise_std : 0.0;
  const PhiloxKey key = philox_key_from_seed(seed);
  p.key0 = key.k0;
  p.key1 = key.k1;
  p.layer_id = layer_id;
  p.step_lo = step.lo;
  p.step_dev = step.dev;
  dp_status st2 = pair        ? launch_umma_pair<Umma2Config<kEpiClipSum>>(p, stream)
                  : (BN == 128) ? launch_umma<UmmaConfig<128, kEpiClipSum>>(p, stream)
                                : launch_umma<UmmaConfig<256, kEpiClipSum>>(p, stream);
  if (st2 == DP_OK && split_partials) {
    CombineBatch cb;
    memset(&cb, 0, sizeof(cb));
    cb.count = 1;
    cb.key = key;
    cb.step = step;
    cb.seg[0] = CombineSegment{out, fx->scratch, static_cast<unsigned long long>(s.m) * ne, splits,
                               (accumulate || preset) ? 1 : 0, noise_std, static_cast<uint32_t>(layer_id)};
    return launch_combine(cb, stream);
  }
  if (st2 != DP_OK || fused_noise || noise_std == 0.0) return st2;
  if (defer && defer->count < kMaxNoiseSegments) {
    defer->seg[defer->count++] = NoiseSegment{out, static_cast<unsigned long long>(s.m) * ne, noise_std,
                                              static_cast<uint32_t>(layer_id)};
    return DP_OK;
  }
  return launch_noise(out, static_cast<unsigned long long>(s.m) * ne, noise_std, seed, step, layer_id,
                      stream);
}

dp_status launch_noise_batch(const NoiseBatch& b, unsigned long long seed, StepRef step, cudaStream_t stream) {
  if (b.count == 0) return DP_OK;
  unsigned long long nblk = 0;
  for (int q = 0; q < b.count; ++q) nblk += (b.seg[q].total + 3) / 4;
  LaunchScope scope(kKindNoise, stream);
  DP_LAUNCH("noise_add_batch_kernel", noise_add_batch_kernel, stream_grid(nblk, 256), 256, 0, stream, b,
            philox_key_from_seed(seed), step);
  return DP_OK;
}

dp_status launch_noise(float* G, unsigned long long total, double std_dev, unsigned long long seed,
                       StepRef step, unsigned layer_id, cudaStream_t stream) {
  LaunchScope scope(kKindNoise, stream);
  // Large G: a persistent grid whose blocks stage the 32 KB of Box-Muller tables once each.
  const PhiloxKey key = philox_key_from_seed(seed);
  if (total >= (1ull << 22)) {
    const int grid = std::min(stream_grid((total + 3) / 4, 256), sm_count() * 4);
    DP_LAUNCH("noise_add_kernel", noise_add_kernel<true>, grid, 256, 0, stream, G, total, std_dev, key,
              layer_id, step);
  } else {
    DP_LAUNCH("noise_add_kernel", noise_add_kernel<false>, stream_grid((total + 3) / 4, 256), 256, 0, stream,
              G, total, std_dev, key, layer_id, step);
  }
  return DP_OK;
}

// Z[N, r] = dY[N, n] P[n, r], bf16 out.
dp_status bf16_project(const Shape& s, const void* dY, const void* P, void* Z, uint32_t* status,
                       cudaStream_t stream) {
  UmmaParams p = base_params(status);
  dp_status st;
  if ((st = map_2d(&p.tmA0, dY, s.N(), s.n, 128)) != DP_OK) return st;
  if ((st = map_2d(&p.tmB0, P, s.n, s.r, 64)) != DP_OK) return st;
  p.m_tiles = ceil_div(s.N(), 128);
  p.k_blocks = ceil_div(s.n, 64);
  p.k_blocks_per_split = p.k_blocks;
  p.k_splits = 1;
  p.out_rows = static_cast<int>(s.N());
  p.out_cols = s.r;
  p.out_bf16 = static_cast<__nv_bfloat16*>(Z);
  p.out_elems = s.N() * s.r;
  if (s.r <= 64 || (s.r <= 128 && p.m_tiles * 2 <= sm_count())) {
    // 128 x 64 tiles when 128 x 128 tiles would leave more than half the SMs idle (e.g.
    // N = 8192 tokens, r = 128: 64 tiles; 128 with this split).  The two CTAs of a row block
    // read the same dY tile at about the same time, so the second read comes from L2.
    p.n_tiles = ceil_div(s.r, 64);
    p.num_units = p.m_tiles * p.n_tiles;
    return launch_umma<UmmaConfig<64, kEpiStoreBf16>>(p, stream);
  }
  if (s.r <= 128) {
    p.n_tiles = ceil_div(s.r, 128);
    p.num_units = p.m_tiles * p.n_tiles;
    return launch_umma<UmmaConfig<128, kEpiStoreBf16>>(p, stream);
  }
  p.n_tiles = ceil_div(s.r, 256);
  p.num_units = p.m_tiles * p.n_tiles;
  return launch_umma<UmmaConfig<256, kEpiStoreBf16>>(p, stream);
}

dp_status launch_projection(void* P, dp_dtype dt, int d_out, int r, unsigned long long seed,
                            unsigned layer_id, cudaStream_t stream) {
  const unsigned long long total = static_cast<unsigned long long>(d_out) * r;
  const int grid = stream_grid((total + 3) / 4, 256);
  const PhiloxKey key = philox_key_from_seed(seed);
  LaunchScope scope(kKindProjection, stream);
  if (dt == DP_BF16)
    DP_LAUNCH("projection_kernel", projection_kernel<true>, grid, 256, 0, stream, P, total, r, key, layer_id);
  else
    DP_LAUNCH("projection_kernel", projection_kernel<false>, grid, 256, 0, stream, P, total, r, key,
              layer_id);
  return DP_OK;
}

dp_status launch_norm_partials(const float* partials, int stride, int count, int B, float C,
                               float* norm2, float* norms_out, float* c_out, cudaStream_t stream);

// With `partials` (B samples), the scaling kernel forms the clip factors of the samples each
// of its blocks covers, unless a block would cover too many samples or partial slots; then the
// partials kernel runs first.
// Blocks of a row-scaling kernel that are resident on one SM at once.  The scaling launches
// are short (tens of microseconds): a grid of exactly one wave of resident blocks keeps every
// block's prologue (its samples' clip factors) off the critical path of a second wave.
int scale_blocks_per_sm(bool batch) {
  static int cached[2][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  int& c = cached[batch ? 1 : 0][dev & 63];
  if (c == 0) {
    int n = 0;
    const cudaError_t e =
        batch ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, scale_rows_bf16_batch_kernel, 256, 1024)
              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, scale_rows_bf16_kernel, 256, 1024);
    c = (e == cudaSuccess && n > 0) ? n : 4;
  }
  return c;
}

dp_status launch_scale(const void* in, void* out, long long rows, int cols, int T, NormSource src,
                       float C, cudaStream_t stream, const PartialsRef* partials = nullptr, int B = 0,
                       const NoiseFill* fill = nullptr, unsigned long long seed = 0, StepRef step = StepRef{0u, nullptr}) {
  const unsigned long long vecs = static_cast<unsigned long long>(rows) * (cols / 8);
  const int grid = std::min(stream_grid(vecs, 256), sm_count() * scale_blocks_per_sm(false));
  PartialsRef pr{nullptr, 0, 0, nullptr, nullptr, nullptr};
  size_t smem = 0;
  if (partials) {
    // A block's contiguous range of `per` vectors touches at most this many samples.
    const unsigned long long per = (vecs + grid - 1) / grid;
    const unsigned long long sample_vecs = static_cast<unsigned long long>(T) * (cols / 8);
    const long long smax = static_cast<long long>(std::min<unsigned long long>((per - 1) / sample_vecs + 2, B));
    if (smax <= kScaleFusedMaxSamples && smax * partials->count <= kScaleFusedPartialSlots) {
      pr = *partials;
      smem = static_cast<size_t>(smax) * sizeof(float);
    } else {
      dp_status st = launch_norm_partials(partials->partials, partials->stride, partials->count, B, C,
                                          partials->norm2, partials->norms_out, partials->c_out, stream);
      if (st != DP_OK) return st;
      src = NormSource{partials->norm2, nullptr, nullptr};
    }
  }
  LaunchScope scope(kKindScale, stream);
  const NoiseFill nf = fill ? *fill : NoiseFill{nullptr, 0, 0.0, 0u};
  DP_LAUNCH("scale_rows_bf16_kernel", scale_rows_bf16_kernel, grid, 256, smem, stream,
            static_cast<const __nv_bfloat16*>(in), static_cast<__nv_bfloat16*>(out), rows, cols, T, src, pr,
            C, nf, philox_key_from_seed(seed), step);
  return DP_OK;
}

dp_status launch_norm_partials(const float* partials, int stride, int count, int B, float C,
                               float* norm2, float* norms_out, float* c_out, cudaStream_t stream) {
  LaunchScope scope(kKindFinalize, stream);
  DP_LAUNCH("reduce_norm_partials_kernel", reduce_norm_partials_kernel, ceil_div(B, 8), 256, 0, stream,
            partials, stride, count, B, C, norm2, norms_out, c_out);
  return DP_OK;
}

dp_status launch_finalize(NormSource src, int B, float C, float* norms_out, float* c_out,
                          cudaStream_t stream) {
  LaunchScope scope(kKindFinalize, stream);
  DP_LAUNCH("finalize_norms_kernel", finalize_norms_kernel, ceil_div(B, 256), 256, 0, stream, src, B, C,
            norms_out, c_out);
  return DP_OK;
}

// The plain reduce: staged tables and a runtime sample loop (B > 8), or, beside a tensor-core
// pass, tables through the cache and the sample loop unrolled for B <= 8.
template <int BU>
dp_status reduce_plain_launch(int grid, size_t smem, cudaStream_t stream, const __nv_bfloat16* gs, int B,
                              long long mn, NormSource src, const PartialsRef& pr, float C, float* out,
                              double noise_std, PhiloxKey key, unsigned layer_id, StepRef step) {
  constexpr bool kStaged = (BU == 0);
  DP_LAUNCH("clip_reduce_kernel", clip_reduce_kernel<kStaged, BU>, grid, 256, smem, stream, gs, B, mn,
            src, pr, C, out, noise_std, key, layer_id, step);
  return DP_OK;
}

// `pr` is used by the unrolled form only (its blocks sum the partials themselves).
dp_status reduce_kernel_launch(int grid, size_t smem, cudaStream_t stream, const __nv_bfloat16* gs, int B,
                          long long mn, NormSource src, const PartialsRef& pr, float C, float* out,
                          double noise_std, PhiloxKey key, unsigned layer_id, StepRef step, bool staged) {
  const PartialsRef none{nullptr, 0, 0, nullptr, nullptr, nullptr};
#define DP_REDUCE_PLAIN(BU_, PR_) \
  reduce_plain_launch<BU_>(grid, smem, stream, gs, B, mn, src, PR_, C, out, noise_std, key, layer_id, step)
  if (staged) return DP_REDUCE_PLAIN(0, none);
  switch (B) {  // coresident: B <= 8 (larger batches keep the staged runtime loop)
    case 1: return DP_REDUCE_PLAIN(1, pr);
    case 2: return DP_REDUCE_PLAIN(2, pr);
    case 3: return DP_REDUCE_PLAIN(3, pr);
    case 4: return DP_REDUCE_PLAIN(4, pr);
    case 5: return DP_REDUCE_PLAIN(5, pr);
    case 6: return DP_REDUCE_PLAIN(6, pr);
    case 7: return DP_REDUCE_PLAIN(7, pr);
    default: return DP_REDUCE_PLAIN(8, pr);
  }
#undef DP_REDUCE_PLAIN
}

template <int BU>
dp_status reduce_tma_launch(cudaStream_t stream, const __nv_bfloat16* gs, long long mn, NormSource src,
                            const PartialsRef& pr, float C, float* out, double noise_std, PhiloxKey key,
                            unsigned layer_id, StepRef step, uint32_t* status) {
  using Cfg = ReduceTmaConfig<BU>;
  static bool configured[64] = {false};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    DP_CUDA(cudaFuncSetAttribute(clip_reduce_tma_kernel<BU>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    configured[dev] = true;
  }
  const long long chunks = (mn + kReduceChunk - 1) / kReduceChunk;
  const int grid = static_cast<int>(chunks < sm_count() ? chunks : sm_count());
  DP_LAUNCH("clip_reduce_tma_kernel", clip_reduce_tma_kernel<BU>, grid, Cfg::THREADS,
            Cfg::SMEM_BYTES, stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status);
  return DP_OK;
}

dp_status launch_reduce(const __nv_bfloat16* gs, int B, long long mn, NormSource src, float C,
                        float* out, double noise_std, unsigned long long seed, StepRef step,
                        unsigned layer_id, cudaStream_t stream, uint32_t* status,
                        const PartialsRef* partials = nullptr, bool coresident = false) {
  // With `partials`, the clip factors come from the per-warp norm partials: the bulk-copy
  // reduce sums them in its prologue (and block 0 writes norm2 / norms_out / c_out); the
  // other reduce needs them summed first.
  // `coresident`: the reduce runs beside a tensor-core pass (the overlapped block step), so it
  // takes the plain kernel with its tables read through the cache, whose blocks fit on an SM
  // next to a tensor-core CTA; the bulk-copy kernel fills a whole SM's shared memory.
  if (B <= 8 && !coresident) {
    // Warp-specialised bulk-copy reduce: noise generation overlaps the HBM stream.
    const PhiloxKey key = philox_key_from_seed(seed);
    const PartialsRef pr = partials ? *partials : PartialsRef{nullptr, 0, 0, nullptr, nullptr, nullptr};
    LaunchScope scope(kKindReduce, stream);
    dp_status st;
    switch (B) {
      case 1: st = reduce_tma_launch<1>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 2: st = reduce_tma_launch<2>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 3: st = reduce_tma_launch<3>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 4: st = reduce_tma_launch<4>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 5: st = reduce_tma_launch<5>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 6: st = reduce_tma_launch<6>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      case 7: st = reduce_tma_launch<7>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
      default: st = reduce_tma_launch<8>(stream, gs, mn, src, pr, C, out, noise_std, key, layer_id, step, status); break;
    }
    if (st != DP_OK) return st;
    return DP_OK;
  }
  const bool unrolled = coresident && B <= 8;
  PartialsRef pr{nullptr, 0, 0, nullptr, nullptr, nullptr};
  if (partials && unrolled) {
    pr = *partials;  // the unrolled reduce sums them in its prologue
  } else if (partials) {
    dp_status st = launch_norm_partials(partials->partials, partials->stride, partials->count, B, C,
                                        partials->norm2, partials->norms_out, partials->c_out, stream);
    if (st != DP_OK) return st;
    src = NormSource{partials->norm2, nullptr, nullptr};
  }
  const int cached = B < kReduceCachedSamples ? B : kReduceCachedSamples;
  // Beside a tensor-core pass one block per SM: two would take more registers than an SM has
  // next to a tensor-core CTA, and the next pass would wait for them.
  const int grid = std::min(stream_grid(static_cast<unsigned long long>(mn / 8), 256),
                            coresident ? sm_count() : sm_count() * 2);
  const size_t smem = (unrolled ? 0 : kNoiseSharedBytes) + cached * sizeof(float);
  const PhiloxKey key = philox_key_from_seed(seed);
  LaunchScope scope(kKindReduce, stream);
  return reduce_kernel_launch(grid, smem, stream, gs, B, mn, src, pr, C, out, noise_std, key, layer_id, step,
                              !unrolled);
}

// ---------------------------------------------------------------- common front end
struct Call {
  Shape s;
  WsLayout L;
  uint8_t* ws;
  cudaStream_t stream;
  uint32_t* status() const { return reinterpret_cast<uint32_t*>(ws + L.status); }
  float* norm2_f32() const { return reinterpret_cast<float*>(ws + L.norm2); }
  double* norm2_f64() const { return reinterpret_cast<double*>(ws + L.norm2); }
  float* c() const { return reinterpret_cast<float*>(ws + L.c); }
  float* partials() const { return reinterpret_cast<float*>(ws + L.partials); }
};

dp_status check_common(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B,
                       int T, int d_in, int d_out, void* workspace, size_t ws_bytes, bool p_from_seed,
                       dp_norm_method method, Call* call) {
  if (!X || !dY || !workspace) return DP_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(dY) || (P && !aligned16(P))) return DP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DP_ERR_INVALID_ARG;
  if (P && r < 1) return DP_ERR_INVALID_ARG;
  if (!P && r != 0 && !p_from_seed) return DP_ERR_INVALID_ARG;
  call->s = Shape{B, T, d_in, d_out, r, dt};
  if (!valid_shape(call->s)) return DP_ERR_INVALID_ARG;
  call->L = ws_layout(call->s, method == DP_NORM_AUTO ? auto_method(call->s) : method);
  if (ws_bytes < call->L.total) return DP_ERR_WORKSPACE;
  call->ws = static_cast<uint8_t*>(workspace);
  return DP_OK;
}

// Projection front end shared by the calls: returns the clip-space operand (dY or Z = dY P).
dp_status clip_space_operand(Call& c, const void* dY, const void* P, bool p_from_seed,
                             unsigned long long seed, unsigned layer_id, const void** Zout) {
  if (c.s.r == 0) {
    *Zout = dY;
    return DP_OK;
  }
  const void* Pd = P;
  dp_status st;
  if (!P && p_from_seed) {
    if ((st = launch_projection(c.ws + c.L.p, c.s.dt, c.s.n, c.s.r, seed, layer_id, c.stream)) != DP_OK)
      return st;
    Pd = c.ws + c.L.p;
  }
  void* Z = c.ws + c.L.z;
  if (c.s.dt == DP_BF16) {
    if ((st = bf16_project(c.s, dY, Pd, Z, c.status(), c.stream)) != DP_OK) return st;
  } else {
    const long long total = c.s.N() * c.s.r;
    LaunchScope scope(kKindF32Project, c.stream);
    DP_LAUNCH("f32_project_kernel", f32_project_kernel, stream_grid(total, 256), 256, 0, c.stream,
              static_cast<const float*>(dY), static_cast<const float*>(Pd), static_cast<float*>(Z), c.s.N(),
              c.s.n, c.s.r);
  }
  *Zout = Z;
  return DP_OK;
}

// Per-sample squared norms into the workspace's norm2[B]; for bf16 also norms_out and c
// when given (the fp32 path writes those in launch_finalize).
dp_status norms_into_ws(Call& c, const void* X, const void* Z, dp_norm_method method, float C,
                        float* norms_out, bool store_tiles = false) {
  if (c.s.dt == DP_F32) {
    dim3 grid(ceil_div(c.s.ne(), kF32Tile), ceil_div(c.s.m, kF32Tile), c.s.B);
    LaunchScope scope(kKindF32Norm, c.stream);
    DP_LAUNCH("f32_norm_kernel", f32_norm_kernel, grid, 256, 0, c.stream, static_cast<const float*>(X),
              static_cast<const float*>(Z), c.s.T, c.s.m, c.s.ne(), c.norm2_f64());
    return DP_OK;
  }
  int count = 0;
  dp_status st = bf16_norms(c.s, X, Z, method, c.partials(), c.L.partial_stride, &count, c.status(),
                            c.stream, store_tiles ? reinterpret_cast<__nv_bfloat16*>(c.ws + c.L.gs) : nullptr);
  if (st != DP_OK) return st;
  return launch_norm_partials(c.partials(), c.L.partial_stride, count, c.s.B, C, c.norm2_f32(), norms_out,
                              norms_out ? c.c() : nullptr, c.stream);
}

NormSource ws_norm_source(const Call& c) {
  NormSource src{nullptr, nullptr, nullptr};
  if (c.s.dt == DP_F32)
    src.norm2_f64 = c.norm2_f64();
  else
    src.norm2_f32 = c.norm2_f32();
  return src;
}

// G_out (+)= sum_i c_i X_i^T Z_i (+ noise) for norms given by `src`.
dp_status clipped_sum(Call& c, const void* X, const void* Z, NormSource src, float C, float* out,
                      int accumulate, double noise_std, unsigned long long seed,
                      StepRef step, unsigned layer_id, NoiseBatch* defer = nullptr,
                      const PartialsRef* partials = nullptr, bool prefill_noise = false) {
  // prefill_noise (a clipped sum that adds itself to out, accumulate = 0): the row-scaling
  // launch also writes the noise into out, and the contraction adds its sum to it.
  const Shape& s = c.s;
  if (s.dt == DP_F32) {
    dim3 grid(ceil_div(s.ne(), kF32Tile), ceil_div(s.m, kF32Tile));
    const PhiloxKey key = philox_key_from_seed(seed);
    LaunchScope scope(kKindF32ClipSum, c.stream);
    DP_LAUNCH("f32_clipsum_kernel", f32_clipsum_kernel, grid, 256, 0, c.stream, static_cast<const float*>(X),
              static_cast<const float*>(Z), s.N(), s.T, s.m, s.ne(), src, C, out, accumulate, noise_std, key,
              layer_id, step);
    return DP_OK;
  }
  // Fold c_i into the narrower operand: one extra read + write of N * min(m, ne) bf16.
  void* scaled = c.ws + c.L.scaled;
  dp_status st;
  const NoiseFill fill{out, static_cast<unsigned long long>(s.m) * s.ne(), noise_std, layer_id};
  const NoiseFill* nf = prefill_noise ? &fill : nullptr;
  // The layout's split-sum regions, when it has them (a shape whose clipped sum splits over K).
  const FixupRef fx{c.L.fixup ? reinterpret_cast<float*>(c.ws + c.L.fixup) : nullptr, c.L.fixup_splits};
  if (s.ne() <= s.m) {
    if ((st = launch_scale(Z, scaled, s.N(), s.ne(), s.T, src, C, c.stream, partials, s.B, nf, seed, step)) != DP_OK)
      return st;
    return bf16_clipsum(s, X, scaled, out, accumulate, noise_std, seed, step, layer_id, c.status(), c.stream,
                        defer, prefill_noise, &fx);
  }
  if ((st = launch_scale(X, scaled, s.N(), s.m, s.T, src, C, c.stream, partials, s.B, nf, seed, step)) != DP_OK)
    return st;
  return bf16_clipsum(s, scaled, Z, out, accumulate, noise_std, seed, step, layer_id, c.status(), c.stream,
                      defer, prefill_noise, &fx);
}

dp_status resolve_method(const Shape& s, dp_norm_method method, dp_norm_method* out) {
  if (method == DP_NORM_AUTO) {
    *out = auto_method(s);
    return DP_OK;
  }
  if (method != DP_NORM_GHOST && method != DP_NORM_EXPLICIT && method != DP_NORM_ONCE)
    return DP_ERR_INVALID_ARG;
  if (s.dt == DP_F32 && method != DP_NORM_EXPLICIT) return DP_ERR_UNSUPPORTED;
  *out = method;
  return DP_OK;
}

// ---------------------------------------------------------------- block step
// One call for the linears of a block.  Linears that read the same X with the same shape and
// take the ghost norm are grouped (up to three: q/k/v, gate/up), and one X Gram per
// token-block pair serves the whole group.  Every other linear is a group of one.
//
// Workspace: one status word; the flat squared norms [B]; every layer's squared norms [L][B]
// (fp64 slots, fp32 used for bf16); c[B]; the norm partial slots (three sets when some group
// shares an X Gram) and the scaled-operand copy, each sized for the largest layer; and the
// bf16 per-sample tiles of the gradients-once layers.  Flat clipping needs every such layer's
// tiles at once; per-layer clipping finishes each layer before the next, so one region sized
// for the largest serves them all.
struct BlockLayout {
  size_t flat = 0, norm2 = 0, c = 0, partials = 0, scaled = 0, total = 0;
  std::vector<size_t> z;                 // per layer: its projected operand Z = dY P, or 0
  int partial_stride = 0;
  long long partial_op_stride = 0;       // floats between the partial sets of a shared group
  std::vector<size_t> tiles;             // per layer; 0 when the layer does not keep tiles
  std::vector<dp_norm_method> methods;   // resolved per layer
  std::vector<std::vector<int>> groups;  // layers grouped as described above, in processing order
  // Per-layer mode with two or more gradients-once layers: the reduce of one such layer runs on
  // a second stream beside the next layer's tensor-core pass, so consecutive gradients-once
  // layers alternate between two tile regions and two norm-partial sets.
  bool overlap = false;
  size_t tiles_alt = 0;                  // the second tile region (overlap only)
  // Per-layer mode, bf16, two or more ghost/explicit layers whose scaled copies fit
  // kBatchScaleBytes: every such layer's norm pass first (each into its own norm-partial set),
  // then one row-scaling launch for all of them (each into its own scaled copy), then their
  // clipped sums.  One launch replaces one per layer.
  bool batched_scale = false;
  std::vector<size_t> scaled_l;          // per layer: its scaled copy (batched schedule), or 0
  std::vector<long long> partial_set;    // per layer: its norm-partial set (batched schedule)
  bool z_grouped = false;                // bf16 projected layers: every Z formed in grouped launches
  // Clipped sums split over K: per layer its split partials (0: none).
  std::vector<size_t> fixup;
  std::vector<int> fixup_splits;         // per layer: splits its partials region holds
};

constexpr size_t kBatchScaleBytes = size_t(256) << 20;

// Whether a per-layer block step overlaps each gradients-once reduce with the next layer's
// tensor-core pass.  Off unless the environment sets DPCLIP_OVERLAP_REDUCE=1: measured on the
// Llama blocks, the reduce beside the pass slows the pass by 7-17% (they share issue slots
// and L2), which cancels the hidden reduce time (7B 5.59 against 5.61 ms serial, 13B 4.80
// against 4.60 ms).  Read at every call, so a workspace size query and the step that uses it
// must see the same setting.
bool overlap_reduce_enabled() {
  const char* v = getenv("DPCLIP_OVERLAP_REDUCE");
  return v && v[0] == '1';
}

Shape layer_shape(const dp_layer& l, int B, int T, dp_dtype dt) {
  return Shape{B, T, l.d_in, l.d_out, l.P ? l.r : 0, dt};
}

// The second stream of the current device on which overlapped reduces run, created on the
// first call that needs it (non-blocking, so it never waits on the legacy default stream).
dp_status side_stream(cudaStream_t* out) {
  static std::mutex mu;
  static cudaStream_t streams[64] = {nullptr};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return DP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(mu);
  if (!streams[dev]) DP_CUDA(cudaStreamCreateWithFlags(&streams[dev], cudaStreamNonBlocking));
  *out = streams[dev];
  return DP_OK;
}

// Ordering events of one host thread on the current device, reused round-robin.  A stream's
// wait on an event takes the event's state when the wait is enqueued, so reuse is safe once
// every wait on the earlier record has been enqueued (a block step waits at most two layers
// after a record, far fewer than the ring's size).
class EventRing {
 public:
  dp_status next(cudaEvent_t* out) {
    int dev = 0;
    DP_CUDA(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return DP_ERR_UNSUPPORTED;
    auto& ring = rings_[dev];
    if (ring.empty()) {
      ring.resize(kSize, nullptr);
      for (auto& e : ring) DP_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    }
    *out = ring[pos_[dev]];
    pos_[dev] = (pos_[dev] + 1) % kSize;
    return DP_OK;
  }

 private:
  static constexpr int kSize = 64;
  std::vector<cudaEvent_t> rings_[64];
  int pos_[64] = {0};
};

EventRing& event_ring() {
  static thread_local EventRing ring;
  return ring;
}

// Makes `waiter` wait for everything enqueued on `signaller` so far.
dp_status stream_after(cudaStream_t waiter, cudaStream_t signaller, cudaEvent_t* recorded = nullptr) {
  cudaEvent_t e;
  dp_status st = event_ring().next(&e);
  if (st != DP_OK) return st;
  DP_CUDA(cudaEventRecord(e, signaller));
  DP_CUDA(cudaStreamWaitEvent(waiter, e, 0));
  if (recorded) *recorded = e;
  return DP_OK;
}

dp_status block_methods(const dp_layer* layers, int L, int B, int T, dp_dtype dt, dp_norm_method method,
                        std::vector<dp_norm_method>* out) {
  out->clear();
  for (int l = 0; l < L; ++l) {
    const Shape s = layer_shape(layers[l], B, T, dt);
    if (!valid_shape(s)) return DP_ERR_INVALID_ARG;
    dp_norm_method m;
    dp_status st = resolve_method(s, method, &m);
    if (st != DP_OK) return st;
    out->push_back(m);
  }
  return DP_OK;
}

std::vector<std::vector<int>> block_groups(const dp_layer* layers, int L, dp_dtype dt,
                                           const std::vector<dp_norm_method>& methods) {
  std::vector<std::vector<int>> groups;
  std::vector<bool> taken(L, false);
  for (int l = 0; l < L; ++l) {
    if (taken[l]) continue;
    groups.push_back({l});
    taken[l] = true;
    if (dt != DP_BF16 || methods[l] != DP_NORM_GHOST) continue;
    for (int j = l + 1; j < L && static_cast<int>(groups.back().size()) < kGhostSharedMaxOps; ++j) {
      if (!taken[j] && methods[j] == DP_NORM_GHOST && layers[j].X == layers[l].X &&
          layers[j].d_in == layers[l].d_in &&
          (layers[j].P ? layers[j].r : layers[j].d_out) == (layers[l].P ? layers[l].r : layers[l].d_out)) {
        groups.back().push_back(j);
        taken[j] = true;
      }
    }
  }
  return groups;
}

// Whether the clipped sums of the layers in `ls` can run as grouped launches: every one on the
// one-SM engine with the same tile width (no SM-pair tiles), up to kMaxGroup a launch.
bool clipsums_groupable(const dp_layer* layers, const std::vector<int>& ls, int B, int T, dp_dtype dt) {
  if (ls.size() < 2) return false;
  int bn = 0;
  for (int l : ls) {
    const ClipSumPlan c = clipsum_plan(layer_shape(layers[l], B, T, dt));
    if (c.pair || (bn && c.bn != bn)) return false;
    bn = c.bn;
  }
  return true;
}

// The K split of each grouped launch of clipped sums over the layers `ls` (chunks of up to
// kMaxGroup in order), per layer of `ls`: one split for a whole launch, chosen so that its
// units fill the GPU about once.  The layout sizes each layer's split partials with it.
std::vector<int> group_sum_splits(const dp_layer* layers, const std::vector<int>& ls, int B, int T, dp_dtype dt) {
  std::vector<int> out;
  for (size_t c0 = 0; c0 < ls.size(); c0 += kMaxGroup) {
    const int count = static_cast<int>(std::min<size_t>(kMaxGroup, ls.size() - c0));
    const ClipSumPlan plan0 = clipsum_plan(layer_shape(layers[ls[c0]], B, T, dt));
    int tiles = 0;
    for (int q = 0; q < count; ++q) tiles += ceil_div(layers[ls[c0 + q]].d_in, 128) * plan0.n_tiles;
    int splits = std::max(1, sm_count() / std::max(1, tiles));
    splits = std::min(splits, std::max(1, plan0.k_blocks / 4));
    splits = ceil_div(plan0.k_blocks, ceil_div(plan0.k_blocks, splits));  // every split non-empty
    for (int q = 0; q < count; ++q) out.push_back(splits);
  }
  return out;
}

BlockLayout block_layout(const dp_layer* layers, int L, int B, int T, dp_dtype dt, dp_clip_mode mode,
                         const std::vector<dp_norm_method>& methods) {
  BlockLayout Lb;
  Lb.methods = methods;
  Lb.groups = block_groups(layers, L, dt, methods);
  int once_groups = 0;
  for (const auto& g : Lb.groups) once_groups += (dt == DP_BF16 && methods[g[0]] == DP_NORM_ONCE) ? 1 : 0;
  Lb.overlap = (mode == DP_CLIP_PER_LAYER && once_groups >= 2 && overlap_reduce_enabled());
  if (Lb.overlap) {
    // Gradients-once layers first, largest reduce first, so that the one reduce no tensor-core
    // pass follows is the smallest; then the other groups.  Per-layer clipping makes the layers
    // independent, so the order changes no result.
    auto size_of = [&](const std::vector<int>& g) {
      const Shape s = layer_shape(layers[g[0]], B, T, dt);
      return static_cast<long long>(s.m) * s.ne();
    };
    auto is_once = [&](const std::vector<int>& g) { return methods[g[0]] == DP_NORM_ONCE; };
    std::stable_sort(Lb.groups.begin(), Lb.groups.end(), [&](const std::vector<int>& a, const std::vector<int>& b) {
      if (is_once(a) != is_once(b)) return is_once(a);
      return is_once(a) && size_of(a) > size_of(b);
    });
  }
  size_t off = 256;
  Lb.flat = off;
  off += align256(static_cast<size_t>(B) * 8);
  Lb.norm2 = off;
  off += align256(static_cast<size_t>(L) * B * 8);
  Lb.c = off;
  off += align256(static_cast<size_t>(B) * 4);
  size_t scaled = 0, tiles_most = 0;
  for (int l = 0; l < L; ++l) {
    const Shape s = layer_shape(layers[l], B, T, dt);
    if (dt == DP_BF16) {
      const int ps = partial_slots(s);
      if (ps > Lb.partial_stride) Lb.partial_stride = ps;
      const size_t sc = static_cast<size_t>(s.N()) * static_cast<size_t>(s.m < s.ne() ? s.m : s.ne()) * 2;
      if (methods[l] != DP_NORM_ONCE && sc > scaled) scaled = sc;
      if (methods[l] == DP_NORM_ONCE)
        tiles_most = std::max(tiles_most, static_cast<size_t>(B) * s.m * s.ne() * 2);
    }
  }
  int sets = Lb.overlap ? 2 : 1;
  for (const auto& g : Lb.groups) sets = std::max(sets, static_cast<int>(g.size()));
  // The batched row-scaling schedule (see BlockLayout).
  size_t scaled_all = 0;
  int scaled_layers = 0;
  for (const auto& g : Lb.groups) {
    if (dt != DP_BF16 || methods[g[0]] == DP_NORM_ONCE) continue;
    for (int l : g) {
      const Shape s = layer_shape(layers[l], B, T, dt);
      scaled_all += align256(static_cast<size_t>(s.N()) * static_cast<size_t>(std::min(s.m, s.ne())) * 2);
      ++scaled_layers;
    }
  }
  Lb.batched_scale = (mode == DP_CLIP_PER_LAYER && scaled_layers >= 2 && scaled_layers <= kMaxScaleSegments &&
                      scaled_all <= kBatchScaleBytes);
  Lb.partial_set.assign(L, 0);
  if (Lb.batched_scale) {
    int next = 2;  // sets 0 and 1 serve the gradients-once layers
    for (const auto& g : Lb.groups) {
      if (methods[g[0]] == DP_NORM_ONCE) continue;
      for (int l : g) Lb.partial_set[l] = next++;
    }
    sets = std::max(sets, next);
  }
  Lb.partial_op_stride = static_cast<long long>(align256(static_cast<size_t>(B) * Lb.partial_stride * 4) / 4);
  Lb.partials = off;
  off += static_cast<size_t>(sets) * Lb.partial_op_stride * 4;
  Lb.scaled = off;
  off += align256(scaled);
  Lb.tiles.assign(L, 0);
  if (mode == DP_CLIP_PER_LAYER) {
    if (tiles_most) {
      for (int l = 0; l < L; ++l)
        if (dt == DP_BF16 && methods[l] == DP_NORM_ONCE) Lb.tiles[l] = off;
      off += align256(tiles_most);
      if (Lb.overlap) {
        Lb.tiles_alt = off;
        off += align256(tiles_most);
      }
    }
  } else {
    for (int l = 0; l < L; ++l) {
      if (dt == DP_BF16 && methods[l] == DP_NORM_ONCE) {
        Lb.tiles[l] = off;
        off += align256(static_cast<size_t>(B) * layers[l].d_in * layer_shape(layers[l], B, T, dt).ne() * 2);
      }
    }
  }
  Lb.scaled_l.assign(L, 0);
  if (Lb.batched_scale) {
    for (const auto& g : Lb.groups) {
      if (methods[g[0]] == DP_NORM_ONCE) continue;
      for (int l : g) {
        const Shape s = layer_shape(layers[l], B, T, dt);
        Lb.scaled_l[l] = off;
        off += align256(static_cast<size_t>(s.N()) * static_cast<size_t>(std::min(s.m, s.ne())) * 2);
      }
    }
  }
  // Each projected layer keeps its Z = dY P from its norms to its clipped sum.
  Lb.z.assign(L, 0);
  Lb.z_grouped = false;
  for (int l = 0; l < L; ++l) Lb.z_grouped = Lb.z_grouped || (dt == DP_BF16 && layers[l].P);
  for (int l = 0; l < L; ++l) {
    if (layers[l].P) {
      Lb.z[l] = off;
      off += align256(static_cast<size_t>(B) * T * layers[l].r * (dt == DP_BF16 ? 2 : 4));
    }
  }
  // Split partials of each bf16 ghost or explicit layer whose clipped sum splits over K: with
  // the split of its grouped launch (batched schedule, groupable sums), else its own.
  Lb.fixup.assign(L, 0);
  Lb.fixup_splits.assign(L, 0);
  if (dt == DP_BF16) {
    std::vector<int> splits(L, 1);
    for (int l = 0; l < L; ++l)
      if (methods[l] != DP_NORM_ONCE) splits[l] = clipsum_plan(layer_shape(layers[l], B, T, dt)).splits;
    if (Lb.batched_scale) {
      std::vector<int> batch_all;
      for (const auto& g : Lb.groups)
        if (methods[g[0]] != DP_NORM_ONCE) batch_all.insert(batch_all.end(), g.begin(), g.end());
      if (clipsums_groupable(layers, batch_all, B, T, dt)) {
        const std::vector<int> gs = group_sum_splits(layers, batch_all, B, T, dt);
        for (size_t i = 0; i < batch_all.size(); ++i) splits[batch_all[i]] = gs[i];
      }
    }
    for (int l = 0; l < L; ++l) {
      if (splits[l] < 2) continue;
      const Shape s = layer_shape(layers[l], B, T, dt);
      Lb.fixup[l] = off;
      Lb.fixup_splits[l] = splits[l];
      off += align256(static_cast<size_t>(splits[l]) * s.m * s.ne() * 4);
    }
  }
  Lb.total = off;
  return Lb;
}

// Layer l's clip-space operand: dY, or Z = dY P formed into the workspace when `form` is set
// (the norms pass forms it; the clipped sum reuses it).
dp_status block_operand(const dp_layer* layers, int l, dp_dtype dt, int B, int T, const BlockLayout& Lb,
                        uint8_t* ws, cudaStream_t stream, bool form, const void** Z) {
  const dp_layer& y = layers[l];
  if (!y.P) {
    *Z = y.dY;
    return DP_OK;
  }
  void* z = ws + Lb.z[l];
  *Z = z;
  if (!form || Lb.z_grouped) return DP_OK;  // grouped: formed at the start of the step
  const Shape s = layer_shape(y, B, T, dt);
  if (dt == DP_BF16) return bf16_project(s, y.dY, y.P, z, reinterpret_cast<uint32_t*>(ws), stream);
  const long long total = s.N() * s.r;
  LaunchScope scope(kKindF32Project, stream);
  DP_LAUNCH("f32_project_kernel", f32_project_kernel, stream_grid(total, 256), 256, 0, stream,
            static_cast<const float*>(y.dY), static_cast<const float*>(y.P), static_cast<float*>(z), s.N(),
            s.n, s.r);
  return DP_OK;
}

// Z_l = dY_l P_l of every bf16 projected layer, in one grouped tensor-core launch per chunk of
// up to kMaxGroup layers with the same r (the DP-GRAPE projection of a block, formed once).
dp_status block_projections(const dp_layer* layers, int L, dp_dtype dt, int B, int T, const BlockLayout& Lb,
                            uint8_t* ws, cudaStream_t stream) {
  if (!Lb.z_grouped) return DP_OK;
  std::vector<bool> done(L, false);
  const long long N = static_cast<long long>(B) * T;
  const int m_tiles = ceil_div(N, 128);
  for (int l0 = 0; l0 < L; ++l0) {
    if (done[l0] || !layers[l0].P) continue;
    const int r = layers[l0].r;
    std::vector<int> chunk;
    for (int l = l0; l < L && static_cast<int>(chunk.size()) < kMaxGroup; ++l)
      if (!done[l] && layers[l].P && layers[l].r == r) chunk.push_back(l);
    const int count = static_cast<int>(chunk.size());
    // 128 x 64 tiles when 128 x 128 tiles would leave more than half the SMs idle.
    const int bn = (r <= 64 || (r <= 128 && count * m_tiles * 2 <= sm_count())) ? 64 : (r <= 128 ? 128 : 256);
    UmmaParams p = base_params(reinterpret_cast<uint32_t*>(ws));
    UmmaGroup g;
    memset(&g, 0, sizeof(g));
    g.count = count;
    p.m_tiles = m_tiles;
    p.n_tiles = ceil_div(r, bn);
    p.k_splits = 1;
    p.out_rows = static_cast<int>(N);
    p.out_cols = r;
    p.out_elems = N * r;
    int units = 0;
    dp_status st;
    for (int q = 0; q < count; ++q) {
      const dp_layer& y = layers[chunk[q]];
      if ((st = map_2d(&g.tmA[q], y.dY, N, y.d_out, 128)) != DP_OK) return st;
      if ((st = map_2d(&g.tmB[q], y.P, y.d_out, r, 64)) != DP_OK) return st;
      g.out_bf16[q] = reinterpret_cast<__nv_bfloat16*>(ws + Lb.z[chunk[q]]);
      g.k_blocks[q] = ceil_div(y.d_out, 64);
      g.unit_begin[q] = units;
      units += p.m_tiles * p.n_tiles;
      done[chunk[q]] = true;
    }
    g.unit_begin[count] = units;
    p.num_units = units;
    if (bn == 64) st = launch_umma_group<UmmaConfig<64, kEpiStoreBf16, true>>(p, g, stream);
    else if (bn == 128) st = launch_umma_group<UmmaConfig<128, kEpiStoreBf16, true>>(p, g, stream);
    else st = launch_umma_group<UmmaConfig<256, kEpiStoreBf16, true>>(p, g, stream);
    if (st != DP_OK) return st;
  }
  return DP_OK;
}

// Ghost-norm partials of single (unshared) ghost layers `ls` in grouped launches of up to
// kMaxGroup problems, each with its own X and dY (or Z) maps, partial set and unit split.
dp_status launch_ghost_group(const dp_layer* layers, const std::vector<int>& ls, dp_dtype dt, int B, int T,
                             const BlockLayout& Lb, uint8_t* ws, cudaStream_t stream, std::vector<int>* counts) {
  dp_status st;
  const int t_tiles = ceil_div(T, 128);
  const int pairs = t_tiles * (t_tiles + 1) / 2;
  for (size_t c0 = 0; c0 < ls.size(); c0 += kMaxGroup) {
    const int count = static_cast<int>(std::min<size_t>(kMaxGroup, ls.size() - c0));
    UmmaParams p = base_params(reinterpret_cast<uint32_t*>(ws));
    UmmaGroup g;
    memset(&g, 0, sizeof(g));
    g.count = count;
    p.t_tiles = t_tiles;
    p.pairs_per_sample = pairs;
    p.partial_stride = Lb.partial_stride;
    int units = 0;
    for (int q = 0; q < count; ++q) {
      const int l = ls[c0 + q];
      const Shape s = layer_shape(layers[l], B, T, dt);
      const void* Z;
      if ((st = block_operand(layers, l, dt, B, T, Lb, ws, stream, false, &Z)) != DP_OK) return st;
      if ((st = map_3d(&g.tmA[q], layers[l].X, B, T, s.m, 128)) != DP_OK) return st;
      if ((st = map_3d(&g.tmB[q], Z, B, T, s.ne(), 128)) != DP_OK) return st;
      g.k_blocks[q] = ceil_div(s.m, 64);
      g.k_blocks1[q] = ceil_div(s.ne(), 64);
      g.partials[q] = reinterpret_cast<float*>(ws + Lb.partials) + Lb.partial_set[l] * Lb.partial_op_stride;
      g.unit_begin[q] = units;
      const GhostSplit gs = ghost_split(s);
      g.split_full_units[q] = gs.full;
      g.split_parts[q] = gs.parts;
      g.split_over_x[q] = gs.over_x ? 1 : 0;
      units += ghost_units(gs, B * pairs);
      (*counts)[c0 + q] = 4 * pairs * gs.parts;
    }
    g.unit_begin[count] = units;
    p.num_units = units;
    if ((st = launch_umma_group<UmmaConfig<128, kEpiGhostNorm, true>>(p, g, stream)) != DP_OK) return st;
  }
  return DP_OK;
}

// Squared norms of the layers of one group into their [B] rows of the norm2 block, and each
// layer's norms_out when given (gradients-once layers also keep their tiles).
dp_status block_group_norms(const dp_layer* layers, const std::vector<int>& g, dp_dtype dt, int B, int T,
                            const BlockLayout& Lb, uint8_t* ws, cudaStream_t stream, int* count_out = nullptr,
                            float* partials_base = nullptr) {
  dp_status st;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  const dp_layer& y0 = layers[g[0]];
  const Shape s = layer_shape(y0, B, T, dt);
  const void* Zs[kGhostSharedMaxOps] = {};
  for (size_t j = 0; j < g.size(); ++j)
    if ((st = block_operand(layers, g[j], dt, B, T, Lb, ws, stream, true, &Zs[j])) != DP_OK) return st;
  if (dt == DP_F32) {
    double* n2 = reinterpret_cast<double*>(ws + Lb.norm2) + static_cast<size_t>(g[0]) * B;
    dim3 grid(ceil_div(s.ne(), kF32Tile), ceil_div(s.m, kF32Tile), B);
    {
      LaunchScope scope(kKindF32Norm, stream);
      DP_LAUNCH("f32_norm_kernel", f32_norm_kernel, grid, 256, 0, stream, static_cast<const float*>(y0.X),
                static_cast<const float*>(Zs[0]), T, s.m, s.ne(), n2);
    }
    if (y0.norms_out) {
      NormSource src{nullptr, n2, nullptr};
      if ((st = launch_finalize(src, B, INFINITY, y0.norms_out, nullptr, stream)) != DP_OK) return st;
    }
    return DP_OK;
  }
  float* partials = partials_base ? partials_base : reinterpret_cast<float*>(ws + Lb.partials);
  int count = 0;
  if (g.size() > 1) {
    if ((st = bf16_norms_ghost_shared(s, y0.X, Zs, static_cast<int>(g.size()), partials, Lb.partial_stride,
                                      Lb.partial_op_stride, &count, status, stream)) != DP_OK)
      return st;
  } else {
    const bool once = (Lb.methods[g[0]] == DP_NORM_ONCE);
    if ((st = bf16_norms(s, y0.X, Zs[0], once ? DP_NORM_EXPLICIT : Lb.methods[g[0]], partials,
                         Lb.partial_stride, &count, status, stream,
                         once ? reinterpret_cast<__nv_bfloat16*>(ws + Lb.tiles[g[0]]) : nullptr)) != DP_OK)
      return st;
  }
  if (count_out) {  // the caller sums the partials later (in the row-scaling kernel)
    *count_out = count;
    return DP_OK;
  }
  for (size_t j = 0; j < g.size(); ++j) {
    const dp_layer& y = layers[g[j]];
    float* n2 = reinterpret_cast<float*>(ws + Lb.norm2) + static_cast<size_t>(g[j]) * B;
    if ((st = launch_norm_partials(partials + j * Lb.partial_op_stride, Lb.partial_stride, count, B, INFINITY,
                                   n2, y.norms_out, nullptr, stream)) != DP_OK)
      return st;
  }
  return DP_OK;
}

// Layer l's clipped sum with the clip factors of `src` and bound C, plus noise of std sigma C.
dp_status block_layer_sum(const dp_layer* layers, int l, dp_dtype dt, int B, int T, NormSource src, float C,
                          float sigma, unsigned long long seed, StepRef step, const BlockLayout& Lb,
                          uint8_t* ws, cudaStream_t stream, NoiseBatch* defer,
                          const PartialsRef* partials = nullptr) {
  const dp_layer& y = layers[l];
  const Shape s = layer_shape(y, B, T, dt);
  const double noise_std = (sigma == 0.0f) ? 0.0 : static_cast<double>(sigma) * static_cast<double>(C);
  if (dt == DP_BF16 && Lb.methods[l] == DP_NORM_ONCE)
    return launch_reduce(reinterpret_cast<const __nv_bfloat16*>(ws + Lb.tiles[l]), B,
                         static_cast<long long>(s.m) * s.ne(), src, C, y.G_out, noise_std, seed, step, y.layer_id,
                         stream, reinterpret_cast<uint32_t*>(ws));
  Call c;
  c.s = s;
  c.L = WsLayout();
  c.L.scaled = Lb.scaled;
  c.L.fixup = Lb.fixup[l];
  c.L.fixup_splits = Lb.fixup_splits[l];
  c.ws = ws;
  c.stream = stream;
  const void* Z;
  dp_status st = block_operand(layers, l, dt, B, T, Lb, ws, stream, false, &Z);  // formed by the norms
  if (st != DP_OK) return st;
  // A bf16 sum that adds itself to its output: its row-scaling launch writes the noise first
  // (as in one linear).
  const bool prefill =
      (dt == DP_BF16 && noise_std != 0.0 && sum_prefills_noise(clipsum_plan(s), Lb.fixup_splits[l]));
  return clipped_sum(c, y.X, Z, src, C, y.G_out, 0, noise_std, seed, step, y.layer_id, defer, partials,
                     prefill);
}

NormSource layer_norm_source(const BlockLayout& Lb, uint8_t* ws, int l, int B, dp_dtype dt) {
  NormSource src{nullptr, nullptr, nullptr};
  if (dt == DP_F32)
    src.norm2_f64 = reinterpret_cast<double*>(ws + Lb.norm2) + static_cast<size_t>(l) * B;
  else
    src.norm2_f32 = reinterpret_cast<float*>(ws + Lb.norm2) + static_cast<size_t>(l) * B;
  return src;
}

// The clipped sums of the layers in `ls` (batched schedule, groupable) in grouped launches of
// up to kMaxGroup problems.  One K split for the whole launch (group_sum_splits), chosen so
// that its units fill the GPU about once.  The splits store their partial sums and one
// combining launch forms every output from its noise (std sigma C_l) and its partials, in
// split order (kOutSplitPartials).  Without the layout's split partials the outputs are zeroed,
// the splits add by atomics, and the noise is queued in `deferred`.
dp_status launch_clipsum_groups(const dp_layer* layers, const std::vector<int>& ls, dp_dtype dt, int B, int T,
                                const BlockLayout& Lb, uint8_t* ws, float sigma, unsigned long long seed,
                                StepRef step, NoiseBatch* deferred, cudaStream_t stream) {
  dp_status st;
  for (size_t c0 = 0; c0 < ls.size(); c0 += kMaxGroup) {
    const int count = static_cast<int>(std::min<size_t>(kMaxGroup, ls.size() - c0));
    UmmaParams p = base_params(reinterpret_cast<uint32_t*>(ws));
    UmmaGroup g;
    memset(&g, 0, sizeof(g));
    g.count = count;
    const ClipSumPlan plan0 = clipsum_plan(layer_shape(layers[ls[c0]], B, T, dt));
    bool fix = true;
    for (int q = 0; q < count; ++q) {
      const Shape s = layer_shape(layers[ls[c0 + q]], B, T, dt);
      g.m_tiles[q] = ceil_div(s.m, 128);
      fix = fix && Lb.fixup[ls[c0 + q]] != 0;
    }
    const int k_blocks = plan0.k_blocks;
    int splits = group_sum_splits(layers, std::vector<int>(ls.begin() + c0, ls.begin() + c0 + count), B, T, dt)[0];
    g.k_blocks_per_split = ceil_div(k_blocks, splits);
    splits = ceil_div(k_blocks, g.k_blocks_per_split);
    for (int q = 0; q < count; ++q) fix = fix && splits <= Lb.fixup_splits[ls[c0 + q]];
    int units = 0;
    for (int q = 0; q < count; ++q) {
      const int l = ls[c0 + q];
      const dp_layer& y = layers[l];
      const Shape s = layer_shape(y, B, T, dt);
      const void* Z;
      if ((st = block_operand(layers, l, dt, B, T, Lb, ws, stream, false, &Z)) != DP_OK) return st;
      const void* scaled = ws + Lb.scaled_l[l];
      const void* A = s.ne() <= s.m ? y.X : scaled;
      const void* Bm = s.ne() <= s.m ? scaled : Z;
      if ((st = map_2d(&g.tmA[q], A, s.N(), s.m, 64)) != DP_OK) return st;
      if ((st = map_2d(&g.tmB[q], Bm, s.N(), s.ne(), 64)) != DP_OK) return st;
      g.out_f32[q] = y.G_out;
      g.split_scratch[q] = fix ? reinterpret_cast<float*>(ws + Lb.fixup[l]) : nullptr;
      g.out_rows[q] = s.m;
      g.k_blocks[q] = k_blocks;
      g.unit_begin[q] = units;
      units += g.m_tiles[q] * plan0.n_tiles * splits;
    }
    g.unit_begin[count] = units;
    p.num_units = units;
    p.n_tiles = plan0.n_tiles;
    p.k_blocks = k_blocks;
    p.k_splits = splits;
    p.out_cols = layer_shape(layers[ls[c0]], B, T, dt).ne();
    p.out_mode = fix ? kOutSplitPartials : kOutAtomicAdd;
    p.noise_std = 0.0;  // added to the finished sums
    if (!fix)
      for (int q = 0; q < count; ++q) {
        const Shape s = layer_shape(layers[ls[c0 + q]], B, T, dt);
        DP_CUDA(cudaMemsetAsync(g.out_f32[q], 0, static_cast<size_t>(s.m) * s.ne() * sizeof(float), stream));
      }
    if (plan0.bn == 128) st = launch_umma_group<UmmaConfig<128, kEpiClipSum, true>>(p, g, stream);
    else st = launch_umma_group<UmmaConfig<256, kEpiClipSum, true>>(p, g, stream);
    if (st != DP_OK) return st;
    CombineBatch cb;
    memset(&cb, 0, sizeof(cb));
    cb.key = philox_key_from_seed(seed);
    cb.step = step;
    for (int q = 0; q < count; ++q) {
      const dp_layer& y = layers[ls[c0 + q]];
      const Shape s = layer_shape(y, B, T, dt);
      const unsigned long long elems = static_cast<unsigned long long>(s.m) * s.ne();
      const double std_dev = sigma == 0.0f ? 0.0 : static_cast<double>(sigma) * static_cast<double>(y.C);
      if (fix) {
        cb.seg[cb.count++] = CombineSegment{g.out_f32[q], g.split_scratch[q], elems, splits, 0, std_dev, y.layer_id};
      } else if (std_dev != 0.0 && deferred->count < kMaxNoiseSegments) {
        deferred->seg[deferred->count++] = NoiseSegment{g.out_f32[q], elems, std_dev, y.layer_id};
      } else if (std_dev != 0.0 && (st = launch_noise(g.out_f32[q], elems, std_dev, seed, step, y.layer_id, stream)) != DP_OK) {
        return st;
      }
    }
    if (fix && (st = launch_combine(cb, stream)) != DP_OK) return st;
  }
  return DP_OK;
}

// One launch of the row scalings of the layers in `ls` (batched schedule): layer l's narrower
// operand (Z, or X when X is narrower) scaled by its clip factors into its own copy.  Each
// layer's blocks sum their samples' norm partials themselves, unless a block would cover too
// many samples or slots; that layer's partials are then summed first.
dp_status launch_scale_batch(const dp_layer* layers, const std::vector<int>& ls, const std::vector<int>& counts,
                             dp_dtype dt, int B, int T, const BlockLayout& Lb, uint8_t* ws, cudaStream_t stream,
                             const std::vector<NoiseFill>& fills, unsigned long long seed, StepRef step) {
  ScaleBatch b;
  memset(&b, 0, sizeof(b));
  b.T = T;
  b.count = static_cast<int>(ls.size());
  b.fills = static_cast<int>(fills.size());
  for (int q = 0; q < b.fills; ++q) b.fill[q] = fills[q];
  b.key = philox_key_from_seed(seed);
  b.step = step;
  unsigned long long total_vecs = 0;
  std::vector<unsigned long long> vecs(ls.size());
  for (size_t q = 0; q < ls.size(); ++q) {
    const Shape s = layer_shape(layers[ls[q]], B, T, dt);
    vecs[q] = static_cast<unsigned long long>(s.N()) * (std::min(s.m, s.ne()) / 8);
    total_vecs += vecs[q];
  }
  const int grid = std::min(stream_grid(total_vecs, 256), sm_count() * scale_blocks_per_sm(true));
  int first = 0;
  size_t smem = 0;
  dp_status st;
  for (size_t q = 0; q < ls.size(); ++q) {
    const int l = ls[q];
    const dp_layer& y = layers[l];
    const Shape s = layer_shape(y, B, T, dt);
    const void* Z;
    if ((st = block_operand(layers, l, dt, B, T, Lb, ws, stream, false, &Z)) != DP_OK) return st;
    ScaleSegment& sg = b.seg[q];
    sg.in = static_cast<const __nv_bfloat16*>(s.ne() <= s.m ? Z : y.X);
    sg.out = reinterpret_cast<__nv_bfloat16*>(ws + Lb.scaled_l[l]);
    sg.rows = s.N();
    sg.cols = std::min(s.m, s.ne());
    sg.C = y.C;
    sg.first_block = first;
    sg.blocks = static_cast<int>(std::max<unsigned long long>(1, (vecs[q] * grid + total_vecs - 1) / total_vecs));
    first += sg.blocks;
    float* partials = reinterpret_cast<float*>(ws + Lb.partials) + Lb.partial_set[l] * Lb.partial_op_stride;
    float* n2 = reinterpret_cast<float*>(ws + Lb.norm2) + static_cast<size_t>(l) * B;
    const unsigned long long per = (vecs[q] + sg.blocks - 1) / sg.blocks;
    const unsigned long long sample_vecs = static_cast<unsigned long long>(T) * (sg.cols / 8);
    const long long smax = static_cast<long long>(std::min<unsigned long long>((per - 1) / sample_vecs + 2, B));
    if (smax <= kScaleFusedMaxSamples && smax * counts[q] <= kScaleFusedPartialSlots) {
      sg.pr = PartialsRef{partials, Lb.partial_stride, counts[q], n2, y.norms_out, nullptr};
      smem = std::max(smem, static_cast<size_t>(smax) * sizeof(float));
    } else {
      // Too many samples or slots for one block: sum this layer's partials first.
      if ((st = launch_norm_partials(partials, Lb.partial_stride, counts[q], B, y.C, n2, y.norms_out, nullptr,
                                     stream)) != DP_OK)
        return st;
      sg.pr = PartialsRef{nullptr, 0, 0, nullptr, nullptr, nullptr};
      sg.src = NormSource{n2, nullptr, nullptr};
    }
  }
  LaunchScope scope(kKindScale, stream);
  DP_LAUNCH("scale_rows_bf16_batch_kernel", scale_rows_bf16_batch_kernel, first, 256, smem, stream, b);
  return DP_OK;
}

dp_status block_step(const dp_layer* layers, int L, dp_dtype dt, int B, int T, dp_clip_mode mode, float C,
                     float sigma, unsigned long long seed, StepRef step, const BlockLayout& Lb,
                     float* flat_norms_out, uint8_t* ws, cudaStream_t stream) {
  dp_status st;
  // Status word, and the fp32 path's atomic norm accumulators, start at zero.
  DP_CUDA(cudaMemsetAsync(ws, 0, Lb.c, stream));
  // Every projected layer's Z = dY P, grouped (bf16).
  if ((st = block_projections(layers, L, dt, B, T, Lb, ws, stream)) != DP_OK) return st;
  // Noise of split-K clipped sums that no row-scaling launch writes (past the batched launch's
  // segment table), added in one launch at the end of the step.
  NoiseBatch deferred;
  deferred.count = 0;
  if (mode == DP_CLIP_PER_LAYER) {
    // Overlap: gradients-once layer k's reduce runs on the side stream beside layer k+1's
    // tensor-core pass.  Layer k alternates between tile region / partial set k mod 2, and the
    // pass of layer k+2, which reuses them, waits for reduce k.  The side stream joins the
    // caller's stream before the call returns, so the call keeps plain stream semantics (and a
    // CUDA graph captured around it stays one fork-join).
    cudaStream_t side = stream;
    if (Lb.overlap && (st = side_stream(&side)) != DP_OK) return st;
    cudaEvent_t reduce_done[2] = {nullptr, nullptr};
    int once_k = 0, once_n = 0;
    for (const auto& g : Lb.groups) once_n += (dt == DP_BF16 && Lb.methods[g[0]] == DP_NORM_ONCE) ? 1 : 0;
    bool side_pending = false;  // reduces on the side stream the caller's stream has not joined
    std::vector<int> batch_layers, batch_counts;  // batched schedule: layers waiting for their sums
    std::vector<int> ghost_single, ghost_single_at;  // batched schedule: single ghost layers, their slots
    // Batched schedule: the noise of every clipped sum that adds itself to its output (one
    // unsplit wave, or splits without their partials' workspace) is written into that output by
    // the batched row-scaling launch.  Grouped sums, and sums split with their partials, take
    // their noise in the combining launch.
    std::vector<bool> preset(L, false);
    std::vector<NoiseFill> fills;
    std::vector<int> batch_all;
    if (Lb.batched_scale)
      for (const auto& g : Lb.groups)
        if (Lb.methods[g[0]] != DP_NORM_ONCE) batch_all.insert(batch_all.end(), g.begin(), g.end());
    const bool grouped_sums = Lb.batched_scale && dt == DP_BF16 && clipsums_groupable(layers, batch_all, B, T, dt);
    if (Lb.batched_scale && sigma != 0.0f && !grouped_sums) {
      for (int l : batch_all) {
        const Shape s = layer_shape(layers[l], B, T, dt);
        if (sum_prefills_noise(clipsum_plan(s), Lb.fixup_splits[l]) && static_cast<int>(fills.size()) < kMaxScaleSegments) {
          fills.push_back(NoiseFill{layers[l].G_out, static_cast<unsigned long long>(s.m) * s.ne(),
                                    static_cast<double>(sigma) * static_cast<double>(layers[l].C), layers[l].layer_id});
          preset[l] = true;
        }
      }
    }
    // Each group: its norms, then each member's clipped sum with its own bound and noise.
    for (const auto& g : Lb.groups) {
      if (dt == DP_BF16 && Lb.methods[g[0]] == DP_NORM_ONCE) {
        // Gradients once: tiles and norm partials, then the reduce that sums the partials.
        const dp_layer& y = layers[g[0]];
        const Shape s = layer_shape(y, B, T, dt);
        const int par = Lb.overlap ? (once_k & 1) : 0;
        float* partials = reinterpret_cast<float*>(ws + Lb.partials) + par * Lb.partial_op_stride;
        __nv_bfloat16* tiles = reinterpret_cast<__nv_bfloat16*>(ws + (par ? Lb.tiles_alt : Lb.tiles[g[0]]));
        if (reduce_done[par]) DP_CUDA(cudaStreamWaitEvent(stream, reduce_done[par], 0));
        const void* Z;
        if ((st = block_operand(layers, g[0], dt, B, T, Lb, ws, stream, true, &Z)) != DP_OK) return st;
        int count = 0;
        if ((st = bf16_norms(s, y.X, Z, DP_NORM_EXPLICIT, partials, Lb.partial_stride, &count,
                             reinterpret_cast<uint32_t*>(ws), stream, tiles)) != DP_OK)
          return st;
        float* n2 = reinterpret_cast<float*>(ws + Lb.norm2) + static_cast<size_t>(g[0]) * B;
        const PartialsRef pr{partials, Lb.partial_stride, count, n2, y.norms_out, nullptr};
        const double noise_std = (sigma == 0.0f) ? 0.0 : static_cast<double>(sigma) * static_cast<double>(y.C);
        // The last gradients-once reduce has no tensor-core pass beside it: it takes the whole
        // GPU, on the caller's stream, with the bulk-copy kernel.
        const bool beside = Lb.overlap && once_k + 1 < once_n;
        if (beside && (st = stream_after(side, stream)) != DP_OK) return st;
        if ((st = launch_reduce(tiles, B, static_cast<long long>(s.m) * s.ne(), layer_norm_source(Lb, ws, g[0], B, dt),
                                y.C, y.G_out, noise_std, seed, step, y.layer_id, beside ? side : stream,
                                reinterpret_cast<uint32_t*>(ws), &pr, beside)) != DP_OK)
          return st;
        if (beside) {
          if ((st = event_ring().next(&reduce_done[par])) != DP_OK) return st;
          DP_CUDA(cudaEventRecord(reduce_done[par], side));
          side_pending = true;
        }
        ++once_k;
        continue;
      }
      // The other groups reuse the norm-partial sets: join the side stream first.
      if (side_pending) {
        if ((st = stream_after(stream, side)) != DP_OK) return st;
        side_pending = false;
      }
      if (Lb.batched_scale) {
        // Batched schedule: this group's norm pass now (single ghost layers: all in one grouped
        // launch after the loop), its row scaling and clipped sums after every norm pass.
        if (dt == DP_BF16 && g.size() == 1 && Lb.methods[g[0]] == DP_NORM_GHOST) {
          ghost_single.push_back(g[0]);
          ghost_single_at.push_back(static_cast<int>(batch_layers.size()));
          batch_layers.push_back(g[0]);
          batch_counts.push_back(0);  // set by the grouped launch
          continue;
        }
        int count = 0;
        float* base = reinterpret_cast<float*>(ws + Lb.partials) + Lb.partial_set[g[0]] * Lb.partial_op_stride;
        if ((st = block_group_norms(layers, g, dt, B, T, Lb, ws, stream, &count, base)) != DP_OK) return st;
        for (int l : g) {
          batch_layers.push_back(l);
          batch_counts.push_back(count);
        }
        continue;
      }
      // bf16: the row-scaling kernel of each member's clipped sum sums its norm partials.
      int count = 0;
      if ((st = block_group_norms(layers, g, dt, B, T, Lb, ws, stream, dt == DP_BF16 ? &count : nullptr)) !=
          DP_OK)
        return st;
      for (size_t j = 0; j < g.size(); ++j) {
        const int l = g[j];
        const NormSource src = layer_norm_source(Lb, ws, l, B, dt);
        const PartialsRef pr{reinterpret_cast<float*>(ws + Lb.partials) + j * Lb.partial_op_stride,
                             Lb.partial_stride, count, reinterpret_cast<float*>(ws + Lb.norm2) + static_cast<size_t>(l) * B,
                             layers[l].norms_out, nullptr};
        if ((st = block_layer_sum(layers, l, dt, B, T, src, layers[l].C, sigma, seed, step, Lb, ws, stream,
                                  &deferred, dt == DP_BF16 ? &pr : nullptr)) != DP_OK)
          return st;
      }
    }
    if (!ghost_single.empty()) {
      std::vector<int> counts(ghost_single.size(), 0);
      if ((st = launch_ghost_group(layers, ghost_single, dt, B, T, Lb, ws, stream, &counts)) != DP_OK) return st;
      for (size_t i = 0; i < ghost_single.size(); ++i) batch_counts[ghost_single_at[i]] = counts[i];
    }
    if (!batch_layers.empty()) {
      if ((st = launch_scale_batch(layers, batch_layers, batch_counts, dt, B, T, Lb, ws, stream, fills, seed,
                                   step)) != DP_OK)
        return st;
      if (grouped_sums && (st = launch_clipsum_groups(layers, batch_layers, dt, B, T, Lb, ws, sigma, seed, step,
                                                      &deferred, stream)) != DP_OK)
        return st;
      for (int l : grouped_sums ? std::vector<int>() : batch_layers) {
        const dp_layer& y = layers[l];
        const Shape s = layer_shape(y, B, T, dt);
        const void* Z;
        if ((st = block_operand(layers, l, dt, B, T, Lb, ws, stream, false, &Z)) != DP_OK) return st;
        const void* scaled = ws + Lb.scaled_l[l];
        const double noise_std = (sigma == 0.0f) ? 0.0 : static_cast<double>(sigma) * static_cast<double>(y.C);
        const FixupRef fx{Lb.fixup[l] ? reinterpret_cast<float*>(ws + Lb.fixup[l]) : nullptr, Lb.fixup_splits[l]};
        if ((st = bf16_clipsum(s, s.ne() <= s.m ? y.X : scaled, s.ne() <= s.m ? scaled : Z, y.G_out, 0, noise_std,
                               seed, step, y.layer_id, reinterpret_cast<uint32_t*>(ws), stream, &deferred,
                               preset[l], &fx)) != DP_OK)
          return st;
      }
    }
    if (side_pending && (st = stream_after(stream, side)) != DP_OK) return st;  // join
    return launch_noise_batch(deferred, seed, step, stream);
  }
  // 1. Every layer's per-sample norms (gradients-once layers also keep their tiles).
  for (const auto& g : Lb.groups)
    if ((st = block_group_norms(layers, g, dt, B, T, Lb, ws, stream)) != DP_OK) return st;
  // 2. The flat squared norms, summed over the layers in order.
  NormSource src{nullptr, nullptr, nullptr};
  {
    LaunchScope scope(kKindFinalize, stream);
    if (dt == DP_F32) {
      double* flat = reinterpret_cast<double*>(ws + Lb.flat);
      DP_LAUNCH("flat_norm2_kernel", flat_norm2_kernel<double>, ceil_div(B, 256), 256, 0, stream,
                reinterpret_cast<const double*>(ws + Lb.norm2), L, B, flat, flat_norms_out);
      src.norm2_f64 = flat;
    } else {
      float* flat = reinterpret_cast<float*>(ws + Lb.flat);
      DP_LAUNCH("flat_norm2_kernel", flat_norm2_kernel<float>, ceil_div(B, 256), 256, 0, stream,
                reinterpret_cast<const float*>(ws + Lb.norm2), L, B, flat, flat_norms_out);
      src.norm2_f32 = flat;
    }
  }
  // 3. Every layer's clipped sum with the shared clip factors, plus its own noise.
  for (int l = 0; l < L; ++l)
    if ((st = block_layer_sum(layers, l, dt, B, T, src, C, sigma, seed, step, Lb, ws, stream, &deferred)) !=
        DP_OK)
      return st;
  return launch_noise_batch(deferred, seed, step, stream);
}

// ---------------------------------------------------------------- allocation-free norms
// Scratch of dp_per_sample_norms_static: a fixed device array instead of a caller workspace.
// Every GPU that loads this library holds these 1 MiB until the process exits.
constexpr size_t kStaticScratchBytes = size_t(1) << 20;
static __device__ __align__(256) unsigned char g_norms_scratch[kStaticScratchBytes];

// Unique ID of the CUDA context current on this thread (cuCtxGetId: IDs are never reused in a
// process, unlike context handles), or 0 when it cannot be read.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(fn);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_norms_scratch in the current context.  In host code the array's name is
// only a host-side stand-in, so the address must come from cudaGetSymbolAddress, resolved with
// the device current.  It is looked up once per device and context: a device reset, or another
// context made current, gives a new context ID, and the address is looked up again (the module,
// and so the array, is loaded anew in every context).  Without a readable context ID it is
// looked up on every call.
dp_status static_scratch(unsigned char** out) {
  static std::mutex mu;
  static unsigned char* addr[64] = {nullptr};
  static unsigned long long ctx_id[64] = {0};
  int dev = 0;
  DP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return DP_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> g(mu);
  const unsigned long long id = current_context_id();
  if (!addr[dev] || id == 0 || id != ctx_id[dev]) {
    void* p = nullptr;
    DP_CUDA(cudaGetSymbolAddress(&p, g_norms_scratch));
    addr[dev] = static_cast<unsigned char*>(p);
    ctx_id[dev] = current_context_id();  // the lookup makes the primary context current if none was
  }
  *out = addr[dev];
  return DP_OK;
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

size_t dp_workspace_size(int B, int T, int d_in, int d_out, int r, dp_dtype dt) {
  const Shape s{B, T, d_in, d_out, r, dt};
  if (!valid_shape(s)) return 0;
  return ws_layout(s, auto_method(s)).total;
}

size_t dp_workspace_size_for(int B, int T, int d_in, int d_out, int r, dp_dtype dt,
                             dp_norm_method method) {
  const Shape s{B, T, d_in, d_out, r, dt};
  if (!valid_shape(s)) return 0;
  if (method != DP_NORM_AUTO && method != DP_NORM_GHOST && method != DP_NORM_EXPLICIT &&
      method != DP_NORM_ONCE)
    return 0;
  return ws_layout(s, method == DP_NORM_AUTO ? auto_method(s) : method).total;
}

dp_norm_method dp_auto_norm_method(int B, int T, int d_in, int d_out, int r, dp_dtype dt) {
  const Shape s{B < 1 ? 1 : B, T, d_in, d_out, r, dt};
  return auto_method(s);
}

dp_status dp_per_sample_norms(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B,
                              int T, int d_in, int d_out, dp_norm_method method, float* norms,
                              void* workspace, size_t ws_bytes, void* stream) {
  DP_NVTX_RANGE();
  Call c;
  dp_status st = check_common(X, dY, P, r, dt, B, T, d_in, d_out, workspace, ws_bytes, false,
                              DP_NORM_GHOST, &c);
  if (st != DP_OK) return st;
  if (!norms) return DP_ERR_INVALID_ARG;
  dp_norm_method m;
  if ((st = resolve_method(c.s, method, &m)) != DP_OK) return st;
  if (m == DP_NORM_ONCE) m = DP_NORM_EXPLICIT;  // nothing to reuse: the norms are the result
  if ((st = get_encoder()) != DP_OK && dt == DP_BF16) return st;
  c.stream = static_cast<cudaStream_t>(stream);
  DP_CUDA(cudaMemsetAsync(c.ws, 0, c.L.c, c.stream));  // status word + norm accumulators
  const void* Z;
  if ((st = clip_space_operand(c, dY, P, false, 0, 0, &Z)) != DP_OK) return st;
  if ((st = norms_into_ws(c, X, Z, m, INFINITY, dt == DP_BF16 ? norms : nullptr)) != DP_OK) return st;
  if (dt == DP_BF16) return DP_OK;
  return launch_finalize(ws_norm_source(c), B, INFINITY, norms, nullptr, c.stream);
}

dp_status dp_clip_accumulate(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B,
                             int T, int d_in, int d_out, const float* norms, float C, float* G_sum,
                             void* workspace, size_t ws_bytes, void* stream) {
  DP_NVTX_RANGE();
  Call c;
  dp_status st = check_common(X, dY, P, r, dt, B, T, d_in, d_out, workspace, ws_bytes, false,
                              DP_NORM_GHOST, &c);
  if (st != DP_OK) return st;
  if (!norms || !G_sum || !aligned16(G_sum)) return DP_ERR_INVALID_ARG;
  if (!(C > 0.0f)) return DP_ERR_INVALID_ARG;  // also rejects NaN
  if ((st = get_encoder()) != DP_OK && dt == DP_BF16) return st;
  c.stream = static_cast<cudaStream_t>(stream);
  DP_CUDA(cudaMemsetAsync(c.ws, 0, 256, c.stream));  // status word
  const void* Z;
  if ((st = clip_space_operand(c, dY, P, false, 0, 0, &Z)) != DP_OK) return st;
  NormSource src{nullptr, nullptr, norms};
  return clipped_sum(c, X, Z, src, C, G_sum, 1, 0.0, 0, step_value(0), 0);
}

dp_status dp_add_noise(float* G, long long rows, long long cols, float std, unsigned long long seed,
                       unsigned long long step, unsigned layer_id, void* stream) {
  DP_NVTX_RANGE();
  if (!G || !aligned16(G) || rows < 1 || cols < 1) return DP_ERR_INVALID_ARG;
  if (!(std >= 0.0f) || std::isinf(std)) return DP_ERR_INVALID_ARG;
  if (rows > (1ll << 34) / cols) return DP_ERR_INVALID_ARG;
  const unsigned long long total = static_cast<unsigned long long>(rows) * static_cast<unsigned long long>(cols);
  if (std == 0.0f) return DP_OK;
  return launch_noise(G, total, static_cast<double>(std), seed, step_value(step), layer_id,
                      static_cast<cudaStream_t>(stream));
}

dp_status dp_projection_matrix(void* P, dp_dtype dt, int d_out, int r, unsigned long long seed,
                               unsigned layer_id, void* stream) {
  DP_NVTX_RANGE();
  if (!P || !aligned16(P) || !valid_dtype(dt) || d_out < 1 || r < 1) return DP_ERR_INVALID_ARG;
  const int q = (dt == DP_BF16) ? 8 : 4;
  if (d_out % q || r % q) return DP_ERR_INVALID_ARG;
  if (static_cast<long long>(d_out) * r > (1ll << 34)) return DP_ERR_INVALID_ARG;
  return launch_projection(P, dt, d_out, r, seed, layer_id, static_cast<cudaStream_t>(stream));
}

dp_status linear_step(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B, int T, int d_in,
                      int d_out, float C, float sigma, unsigned long long seed, StepRef step, unsigned layer_id,
                      dp_norm_method method, float* norms_out, float* G_out, void* workspace, size_t ws_bytes,
                      void* stream) {
  Call c;
  if (method < DP_NORM_AUTO || method > DP_NORM_ONCE) return DP_ERR_INVALID_ARG;
  dp_status st = check_common(X, dY, P, r, dt, B, T, d_in, d_out, workspace, ws_bytes, true,
                              method, &c);
  if (st != DP_OK) return st;
  if (!G_out || !aligned16(G_out)) return DP_ERR_INVALID_ARG;
  if (!(C > 0.0f) || !(sigma >= 0.0f) || std::isinf(sigma)) return DP_ERR_INVALID_ARG;
  if (std::isinf(C) && sigma != 0.0f) return DP_ERR_INVALID_ARG;  // std = sigma * C would be inf
  dp_norm_method m;
  if ((st = resolve_method(c.s, method, &m)) != DP_OK) return st;
  if ((st = get_encoder()) != DP_OK && dt == DP_BF16) return st;
  c.stream = static_cast<cudaStream_t>(stream);
  DP_CUDA(cudaMemsetAsync(c.ws, 0, c.L.c, c.stream));  // status word + norm accumulators
  const void* Z;
  if ((st = clip_space_operand(c, dY, P, true, seed, layer_id, &Z)) != DP_OK) return st;
  const bool once = (m == DP_NORM_ONCE);
  // sigma = 0 means no noise, also for C = +inf (where sigma * C would be NaN).
  const double noise_std = (sigma == 0.0f) ? 0.0 : static_cast<double>(sigma) * static_cast<double>(C);
  const long long mn = static_cast<long long>(c.s.m) * c.s.ne();
  if (once) {
    // Each G_i tile is formed once: squared on chip into per-warp partials and stored in bf16.
    // The reduce sums the partials itself, then streams the tiles: sum_i c_i G_i + noise.
    __nv_bfloat16* tiles = reinterpret_cast<__nv_bfloat16*>(c.ws + c.L.gs);
    int count = 0;
    if ((st = bf16_norms(c.s, X, Z, DP_NORM_EXPLICIT, c.partials(), c.L.partial_stride, &count, c.status(),
                         c.stream, tiles)) != DP_OK)
      return st;
    const PartialsRef pr{c.partials(), c.L.partial_stride, count, c.norm2_f32(), norms_out,
                         norms_out ? c.c() : nullptr};
    return launch_reduce(tiles, B, mn, ws_norm_source(c), C, G_out, noise_std, seed, step, layer_id, c.stream,
                         c.status(), &pr);
  }
  if (dt == DP_BF16) {
    // A clipped sum that adds itself to G_out (one unsplit wave, or splits without their
    // partials' workspace) finds its noise there, written by the row-scaling launch before it.
    const bool prefill = (noise_std != 0.0 && sum_prefills_noise(clipsum_plan(c.s), c.L.fixup_splits));
    // The norm partials are summed by the row-scaling kernel of the clipped sum.
    int count = 0;
    if ((st = bf16_norms(c.s, X, Z, m, c.partials(), c.L.partial_stride, &count, c.status(), c.stream)) !=
        DP_OK)
      return st;
    const PartialsRef pr{c.partials(), c.L.partial_stride, count, c.norm2_f32(), norms_out,
                         norms_out ? c.c() : nullptr};
    return clipped_sum(c, X, Z, ws_norm_source(c), C, G_out, 0, noise_std, seed, step, layer_id, nullptr, &pr,
                       prefill);
  }
  if ((st = norms_into_ws(c, X, Z, m, C, nullptr)) != DP_OK) return st;
  const NormSource src = ws_norm_source(c);
  if (dt == DP_F32 && norms_out && (st = launch_finalize(src, B, C, norms_out, c.c(), c.stream)) != DP_OK)
    return st;
  return clipped_sum(c, X, Z, src, C, G_out, 0, noise_std, seed, step, layer_id);
}

dp_status dp_linear_step(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B, int T,
                         int d_in, int d_out, float C, float sigma, unsigned long long seed,
                         unsigned long long step, unsigned layer_id, dp_norm_method method,
                         float* norms_out, float* G_out, void* workspace, size_t ws_bytes, void* stream) {
  DP_NVTX_RANGE();
  return linear_step(X, dY, P, r, dt, B, T, d_in, d_out, C, sigma, seed, step_value(step), layer_id, method,
                     norms_out, G_out, workspace, ws_bytes, stream);
}

dp_status dp_linear_step_dev_step(const void* X, const void* dY, const void* P, int r, dp_dtype dt, int B,
                                  int T, int d_in, int d_out, float C, float sigma, unsigned long long seed,
                                  const unsigned long long* step_dev, unsigned layer_id, dp_norm_method method,
                                  float* norms_out, float* G_out, void* workspace, size_t ws_bytes,
                                  void* stream) {
  DP_NVTX_RANGE();
  if (!step_dev || (reinterpret_cast<uintptr_t>(step_dev) & 7u) != 0) return DP_ERR_INVALID_ARG;
  return linear_step(X, dY, P, r, dt, B, T, d_in, d_out, C, sigma, seed, StepRef{0u, step_dev}, layer_id,
                     method, norms_out, G_out, workspace, ws_bytes, stream);
}

dp_status dp_philox_blocks(unsigned* out, unsigned long long nblocks, unsigned long long seed,
                           unsigned long long step, unsigned layer_id, unsigned stream_id,
                           void* stream) {
  DP_NVTX_RANGE();
  if (!out || !aligned16(out) || nblocks < 1 || nblocks > (1ull << 32)) return DP_ERR_INVALID_ARG;
  LaunchScope scope(kKindPhilox, static_cast<cudaStream_t>(stream));
  DP_LAUNCH("philox_blocks_kernel", philox_blocks_kernel, stream_grid(nblocks, 256), 256, 0,
            static_cast<cudaStream_t>(stream), reinterpret_cast<uint4*>(out), nblocks,
            philox_key_from_seed(seed), layer_id, static_cast<uint32_t>(step & 0xFFFFFFFFull), stream_id);
  return DP_OK;
}

dp_status dp_box_muller(const unsigned* words, long long npairs, double* z, void* stream) {
  DP_NVTX_RANGE();
  if (!words || !z || !aligned16(words) || !aligned16(z) || npairs < 1 || npairs > (1ll << 40))
    return DP_ERR_INVALID_ARG;
  LaunchScope scope(kKindNoise, static_cast<cudaStream_t>(stream));
  const unsigned long long n = static_cast<unsigned long long>(npairs);
  DP_LAUNCH("box_muller_words_kernel", box_muller_words_kernel, stream_grid(n, 256), 256, 0,
            static_cast<cudaStream_t>(stream), reinterpret_cast<const uint2*>(words),
            reinterpret_cast<double2*>(z), n);
  return DP_OK;
}

dp_status dp_per_sample_norms_static(const void* X, const void* dY, dp_dtype dt, int B, int T,
                                     int d_in, int d_out, dp_norm_method method, float* norms,
                                     void* stream) {
  DP_NVTX_RANGE();
  if (!X || !dY || !norms || !aligned16(X) || !aligned16(dY)) return DP_ERR_INVALID_ARG;
  const Shape s{B, T, d_in, d_out, 0, dt};
  if (!valid_shape(s)) return DP_ERR_INVALID_ARG;
  dp_norm_method m;
  dp_status st = resolve_method(s, method, &m);
  if (st != DP_OK) return st;
  if (m == DP_NORM_ONCE) m = DP_NORM_EXPLICIT;
  // Layout inside the fixed array: status word, fp64 or fp32 norm accumulators, per-warp
  // norm partials (bf16).  Anything larger than the array is refused before any launch.
  const size_t norm2_off = 256;
  const size_t partials_off = norm2_off + align256(static_cast<size_t>(B) * 8);
  const int stride = (dt == DP_BF16) ? partial_slots(s) : 0;
  const size_t total = partials_off + align256(static_cast<size_t>(B) * stride * 4);
  if (total > kStaticScratchBytes) {
    snprintf(g_cuda_error, sizeof(g_cuda_error),
             "dp_per_sample_norms_static: needs %zu bytes of scratch, the fixed array holds %zu", total,
             kStaticScratchBytes);
    return DP_ERR_WORKSPACE;
  }
  if (dt == DP_BF16 && (st = get_encoder()) != DP_OK) return st;
  unsigned char* scratch = nullptr;
  if ((st = static_scratch(&scratch)) != DP_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  // The status word and the fp32 path's atomic accumulators must start at zero.
  DP_CUDA(cudaMemsetAsync(scratch, 0, partials_off, cs));
  uint32_t* status = reinterpret_cast<uint32_t*>(scratch);
  if (dt == DP_F32) {
    double* norm2 = reinterpret_cast<double*>(scratch + norm2_off);
    dim3 grid(ceil_div(d_out, kF32Tile), ceil_div(d_in, kF32Tile), B);
    {
      LaunchScope scope(kKindF32Norm, cs);
      DP_LAUNCH("f32_norm_kernel", f32_norm_kernel, grid, 256, 0, cs, static_cast<const float*>(X),
                static_cast<const float*>(dY), T, d_in, d_out, norm2);
    }
    NormSource src{nullptr, norm2, nullptr};
    return launch_finalize(src, B, INFINITY, norms, nullptr, cs);
  }
  float* partials = reinterpret_cast<float*>(scratch + partials_off);
  float* norm2 = reinterpret_cast<float*>(scratch + norm2_off);
  int count = 0;
  if ((st = bf16_norms(s, X, dY, m, partials, stride, &count, status, cs)) != DP_OK) return st;
  return launch_norm_partials(partials, stride, count, B, INFINITY, norm2, norms, nullptr, cs);
}

size_t dp_block_workspace_size(const dp_layer* layers, int L, int B, int T, dp_dtype dt,
                               dp_clip_mode mode, dp_norm_method method) {
  if (!layers || L < 1) return 0;
  std::vector<dp_norm_method> methods;
  if (method < DP_NORM_AUTO || method > DP_NORM_ONCE) return 0;
  if (mode != DP_CLIP_PER_LAYER && mode != DP_CLIP_FLAT) return 0;
  if (block_methods(layers, L, B, T, dt, method, &methods) != DP_OK) return 0;
  return block_layout(layers, L, B, T, dt, mode, methods).total;
}

dp_status block_step_entry(const dp_layer* layers, int L, dp_dtype dt, int B, int T, dp_clip_mode mode,
                           float C, float sigma, unsigned long long seed, StepRef step, dp_norm_method method,
                           float* flat_norms_out, void* workspace, size_t ws_bytes, void* stream) {
  if (!layers || L < 1 || !workspace) return DP_ERR_INVALID_ARG;
  if (mode != DP_CLIP_PER_LAYER && mode != DP_CLIP_FLAT) return DP_ERR_INVALID_ARG;
  if (method < DP_NORM_AUTO || method > DP_NORM_ONCE) return DP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DP_ERR_INVALID_ARG;
  if (!(sigma >= 0.0f) || std::isinf(sigma)) return DP_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l) {
    const dp_layer& y = layers[l];
    if (!y.X || !y.dY || !y.G_out || !aligned16(y.X) || !aligned16(y.dY) || !aligned16(y.G_out))
      return DP_ERR_INVALID_ARG;
    // A projection is given with its width; r without P is refused (P is not regenerated).
    if ((y.P && (y.r < 1 || !aligned16(y.P))) || (!y.P && y.r != 0)) return DP_ERR_INVALID_ARG;
    if (mode == DP_CLIP_PER_LAYER && (!(y.C > 0.0f) || (std::isinf(y.C) && sigma != 0.0f)))
      return DP_ERR_INVALID_ARG;
  }
  std::vector<dp_norm_method> methods;
  dp_status st = block_methods(layers, L, B, T, dt, method, &methods);
  if (st != DP_OK) return st;
  if (mode == DP_CLIP_FLAT && (!(C > 0.0f) || (std::isinf(C) && sigma != 0.0f))) return DP_ERR_INVALID_ARG;
  const BlockLayout Lb = block_layout(layers, L, B, T, dt, mode, methods);
  if (ws_bytes < Lb.total) return DP_ERR_WORKSPACE;
  if (dt == DP_BF16 && (st = get_encoder()) != DP_OK) return st;
  return block_step(layers, L, dt, B, T, mode, C, sigma, seed, step, Lb, flat_norms_out,
                    static_cast<uint8_t*>(workspace), static_cast<cudaStream_t>(stream));
}

dp_status dp_block_step(const dp_layer* layers, int L, dp_dtype dt, int B, int T, dp_clip_mode mode,
                        float C, float sigma, unsigned long long seed, unsigned long long step,
                        dp_norm_method method, float* flat_norms_out, void* workspace, size_t ws_bytes,
                        void* stream) {
  DP_NVTX_RANGE();
  return block_step_entry(layers, L, dt, B, T, mode, C, sigma, seed, step_value(step), method, flat_norms_out,
                          workspace, ws_bytes, stream);
}

dp_status dp_block_step_dev_step(const dp_layer* layers, int L, dp_dtype dt, int B, int T, dp_clip_mode mode,
                                 float C, float sigma, unsigned long long seed,
                                 const unsigned long long* step_dev, dp_norm_method method,
                                 float* flat_norms_out, void* workspace, size_t ws_bytes, void* stream) {
  DP_NVTX_RANGE();
  if (!step_dev || (reinterpret_cast<uintptr_t>(step_dev) & 7u) != 0) return DP_ERR_INVALID_ARG;
  return block_step_entry(layers, L, dt, B, T, mode, C, sigma, seed, StepRef{0u, step_dev}, method,
                          flat_norms_out, workspace, ws_bytes, stream);
}

size_t dp_adam_workspace_size(int d_in, int r) {
  if (d_in < 1 || r < 1 || r % 8) return 0;
  return 256 + align256(static_cast<size_t>(d_in) * r * 2);
}

dp_status dp_projected_adam_step(float* W, const float* R, float* m, float* v, const void* P, dp_dtype dt,
                                 int d_in, int d_out, int r, float lr, float beta1, float beta2, float eps,
                                 float grad_scale, int t, void* workspace, size_t ws_bytes, void* stream) {
  DP_NVTX_RANGE();
  if (!W || !R || !m || !v || !P || !workspace) return DP_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(R) || !aligned16(m) || !aligned16(v) || !aligned16(P)) return DP_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DP_ERR_INVALID_ARG;
  if (!valid_dtype(dt)) return DP_ERR_INVALID_ARG;
  if (d_in < 1 || d_out < 1 || r < 1 || d_in % 8 || d_out % 8 || r % 8) return DP_ERR_INVALID_ARG;
  if (static_cast<long long>(d_in) * d_out > (1ll << 34)) return DP_ERR_INVALID_ARG;
  if (t < 1 || !(lr >= 0.0f) || std::isinf(lr) || !(beta1 >= 0.0f && beta1 < 1.0f) ||
      !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps >= 0.0f) || std::isinf(grad_scale) || grad_scale != grad_scale)
    return DP_ERR_INVALID_ARG;
  if (dt != DP_BF16) return DP_ERR_UNSUPPORTED;  // the back-projection runs on bf16 tensor cores
  if (ws_bytes < dp_adam_workspace_size(d_in, r)) return DP_ERR_WORKSPACE;
  dp_status st;
  if ((st = get_encoder()) != DP_OK) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DP_CUDA(cudaMemsetAsync(ws, 0, 256, cs));  // status word
  __nv_bfloat16* U = reinterpret_cast<__nv_bfloat16*>(ws + 256);
  const long long n = static_cast<long long>(d_in) * r;
  const float bc1 = 1.0f - static_cast<float>(std::pow(static_cast<double>(beta1), t));
  const float bc2 = 1.0f - static_cast<float>(std::pow(static_cast<double>(beta2), t));
  {
    LaunchScope scope(kKindAdam, cs);
    DP_LAUNCH("adam_rspace_kernel", adam_rspace_kernel,
              stream_grid(static_cast<unsigned long long>(n / 4), 256), 256, 0, cs, R, m, v, U, n, grad_scale,
              beta1, beta2, eps, bc1, bc2);
  }
  if (lr == 0.0f) return DP_OK;
  UmmaParams p = base_params(reinterpret_cast<uint32_t*>(ws));
  if ((st = map_2d(&p.tmA0, U, d_in, r, 128)) != DP_OK) return st;
  if ((st = map_2d(&p.tmB0, P, d_out, r, 256)) != DP_OK) return st;
  p.m_tiles = ceil_div(d_in, 128);
  p.n_tiles = ceil_div(d_out, 256);
  p.k_blocks = ceil_div(r, 64);
  p.k_blocks_per_split = p.k_blocks;
  p.k_splits = 1;
  p.num_units = p.m_tiles * p.n_tiles;
  p.out_rows = d_in;
  p.out_cols = d_out;
  p.out_f32 = W;
  p.out_elems = static_cast<long long>(d_in) * d_out;
  p.alpha = -lr;
  return launch_umma<UmmaConfig<256, kEpiAxpy>>(p, cs);
}

dp_status dp_selftest_fail_launches(long long skip, long long count, int cuda_error) {
  if (skip < 0 || count < 0 || (count > 0 && cuda_error <= 0)) return DP_ERR_INVALID_ARG;
  g_inject_count.store(0);
  g_inject_skip.store(skip);
  g_inject_error.store(cuda_error);
  g_inject_count.store(count);
  return DP_OK;
}

dp_status dp_selftest_wait_timeout(void* workspace, unsigned long long limit_ns, void* stream) {
  DP_NVTX_RANGE();
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DP_ERR_INVALID_ARG;
  if (limit_ns < 1000ull || limit_ns > kWaitLimitNs) return DP_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  DP_CUDA(cudaMemsetAsync(workspace, 0, 256, cs));
  DP_LAUNCH("wait_timeout_selftest_kernel", wait_timeout_selftest_kernel, 1, 32, 0, cs,
            static_cast<uint32_t*>(workspace), limit_ns);
  return DP_OK;
}

dp_status dp_workspace_status(const void* workspace, void* stream) {
  DP_NVTX_RANGE();
  if (!workspace) return DP_ERR_INVALID_ARG;
  DP_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  uint32_t word = 0;
  DP_CUDA(cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost));
#ifdef DPCLIP_DEBUG
  // Checks of kernels without a workspace status word land in the module's debug word only.
  uint32_t dbg = 0;
  DP_CUDA(cudaMemcpyFromSymbol(&dbg, g_debug_word, sizeof(dbg)));
  if (dbg >= kDebugCheckBase) {
    snprintf(g_cuda_error, sizeof(g_cuda_error), "device-side check %u failed", dbg - kDebugCheckBase);
    return DP_ERR_DEVICE_CHECK;
  }
#endif
  if (word >= kDebugCheckBase) {
    snprintf(g_cuda_error, sizeof(g_cuda_error), "device-side check %u failed", word - kDebugCheckBase);
    return DP_ERR_DEVICE_CHECK;
  }
  return word ? DP_ERR_TIMEOUT : DP_OK;
}

const char* dp_status_string(dp_status s) {
  switch (s) {
    case DP_OK: return "ok";
    case DP_ERR_INVALID_ARG: return "invalid argument";
    case DP_ERR_UNSUPPORTED: return "unsupported";
    case DP_ERR_WORKSPACE: return "workspace too small";
    case DP_ERR_CUDA: return "CUDA error";
    case DP_ERR_TIMEOUT: return "in-kernel wait timed out";
    case DP_ERR_DEVICE_CHECK: return "device-side check failed (debug build)";
  }
  return "unknown status";
}

const char* dp_last_cuda_error(void) { return g_cuda_error; }

dp_status dp_profiling_enable(int on) {
  LaunchProfiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  for (auto& r : p.recs) {
    p.give(r.a);
    p.give(r.b);
  }
  p.recs.clear();
  p.enabled = (on != 0);
  return DP_OK;
}

int dp_profiling_kinds(void) { return kNumKinds; }

const char* dp_profiling_kind_name(int kind) { return kernel_kind_name(kind); }

dp_status dp_profiling_collect(double* total_ms, long long* launches) {
  if (!total_ms || !launches) return DP_ERR_INVALID_ARG;
  LaunchProfiler& p = profiler();
  std::lock_guard<std::mutex> g(p.mu);
  for (int k = 0; k < kNumKinds; ++k) {
    total_ms[k] = 0.0;
    launches[k] = 0;
  }
  dp_status st = DP_OK;
  for (auto& r : p.recs) {
    float ms = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "dp_profiling_collect");
    } else {
      total_ms[r.kind] += ms;
      launches[r.kind] += 1;
    }
    p.give(r.a);
    p.give(r.b);
  }
  p.recs.clear();
  return st;
}

long long dp_kernel_launches(void) { return profiler().launches.load(); }

}  // extern "C"
