/*
 * dpclip.h -- C ABI of the B200 (sm_100a) per-sample gradient clipping library.
 *
 * The library privatises the weight gradient of one linear layer Y = X W, as DP-SGD does per
 * layer.  X[B,T,d_in] is the layer input saved by the forward pass and dY[B,T,d_out] the
 * output gradient.  Sample i's weight gradient is G_i = X_i^T dY_i.  A call of the library
 * computes, per sample, the Frobenius norm n_i = ||G_i||, clips with c_i = min(1, C / n_i),
 * sums S = sum_i c_i G_i and adds Gaussian noise of std sigma*C.  Sources:
 *   - "FlashDP: Private Training Large Language Models with Efficient DP-SGD", Abstract:
 *     per-sample gradient clipping is the costly step of DP-SGD.  FlashDP computes each
 *     per-sample gradient once, in one fused task per layer, and matches per-layer clipped
 *     DP-SGD.
 *   - "Memory-Efficient Differentially Private Training with Gradient Random Projection"
 *     (DP-GRAPE), Problem Statement: per-sample gradients are clipped before noise is added.
 *     Methodology, "Random Projection over SVD" and "Order of Operations": the raw per-sample
 *     gradient is projected by a random Gaussian matrix regenerated from a seed, and only
 *     then clipped and noised.
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller.  Tensors are row-major and
 *     contiguous, with 16-byte aligned base addresses.
 *   - X is [B, T, d_in] and dY is [B, T, d_out], both in dtype `dt`.  Token t of sample i
 *     is row i*T + t.
 *   - P is [d_out, r] in dtype `dt`.  Every output is fp32.
 *   - Work is enqueued asynchronously on `stream`, a cudaStream_t passed as void*; NULL is
 *     the legacy default stream.  Kernels are launched with programmatic dependent launch: a
 *     kernel may be scheduled while the work before it on the stream finishes, but it touches
 *     no memory until that work has completed, so stream order holds as for plain launches.
 *   - The library allocates no device memory.  Scratch comes from the caller's `workspace`,
 *     sized by dp_workspace_size.
 *   - Arguments are checked on the host before anything is enqueued.  On failure nothing on
 *     the device is touched and a non-zero dp_status is returned.  Launch failures return
 *     DP_ERR_CUDA.
 *   - No kernel traps.  Every wait inside a kernel is bounded: when it runs out, the kernel
 *     records it in the workspace's status word and returns, and dp_workspace_status then
 *     reports DP_ERR_TIMEOUT.
 *   - Shapes:
 *       B, T, d_in, d_out >= 1;
 *       d_in, d_out and r are multiples of 8 for bf16 and of 4 for fp32 (rows of 16 bytes);
 *       B*T < 2^31;
 *       an output of rows*cols elements has rows*cols <= 2^34, since one Philox counter
 *       word numbers its blocks of four.
 *   - Random numbers: Philox4x32-10 (Salmon et al., "Parallel random numbers: as easy as
 *     1, 2, 3", SC'11), then Box-Muller (1958) in fp64:
 *       key = (seed mod 2^32, seed >> 32);
 *       counter = (j, layer_id, step mod 2^32, stream);
 *       stream 0 = gradient noise, stream 1 = projection;
 *       u1 = (x_even + 1) 2^-32 and u2 = x_odd 2^-32;
 *       z_even = sqrt(-2 ln u1) cos(2 pi u2) and z_odd = sqrt(-2 ln u1) sin(2 pi u2).
 *     Flat element k = row*cols + col of a buffer takes z_{k mod 4} of block j = k div 4.
 */
#ifndef DPCLIP_H
#define DPCLIP_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DP_OK = 0,
    DP_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misalignment, C <= 0, sigma < 0 ... */
    DP_ERR_UNSUPPORTED = 2,   /* valid request the library does not implement (e.g. fp32 ghost) */
    DP_ERR_WORKSPACE = 3,     /* workspace smaller than dp_workspace_size() */
    DP_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed; see dp_last_cuda_error */
    DP_ERR_TIMEOUT = 5,       /* a bounded in-kernel wait ran out (reported by dp_workspace_status) */
    DP_ERR_DEVICE_CHECK = 6   /* a device-side index check of a DPCLIP_DEBUG build failed; the access
                                 was skipped (reported by dp_workspace_status) */
} dp_status;

typedef enum { DP_F32 = 0, DP_BF16 = 1 } dp_dtype;

/* How n_i is computed.  Both methods give the same value up to rounding:
 *   GHOST    : n_i^2 = sum_{t,s} (x_t . x_s)(dy_t . dy_s), from the two T x T Gram matrices of
 *              sample i.  This is the ghost-norm identity behind the implicit methods the
 *              FlashDP Abstract names (GhostClip).
 *   EXPLICIT : n_i^2 = sum of squares of the tiles of G_i = X_i^T dY_i, formed on chip and
 *              never stored.
 *   ONCE     : EXPLICIT, and each tile of G_i is also kept in the workspace in bf16.  The
 *              clipped sum is then sum_i c_i G_i over those stored tiles, not a second
 *              contraction, so each per-sample gradient is formed exactly once (FlashDP
 *              Abstract: "calculating gradients only once").  It needs B*d_in*ne bf16 of
 *              extra workspace, where ne = d_out, or r with projection.  bf16 only.
 *   AUTO     : the cheapest of the three by a roofline cost model: flops at 1.4e15/s and
 *              bytes at 6.5e12/s (ghost: B ceil(T/128)(ceil(T/128)+1)/2 128x128 Gram tile
 *              pairs plus one scaling pass; explicit: twice the contraction; once: the
 *              contraction plus the stored tiles read back).  fp32 inputs always use
 *              EXPLICIT. */
typedef enum {
    DP_NORM_AUTO = 0,
    DP_NORM_GHOST = 1,
    DP_NORM_EXPLICIT = 2,
    DP_NORM_ONCE = 3
} dp_norm_method;

/* Bytes of workspace needed by every call below for these shapes when the norm method is
 * DP_NORM_AUTO.  r = 0 means unprojected.  Returns 0 when the shape is invalid.  The workspace
 * must be 256-byte aligned (any cudaMalloc or torch allocation is). */
size_t dp_workspace_size(int B, int T, int d_in, int d_out, int r, dp_dtype dt);

/* The same for an explicit norm method (DP_NORM_ONCE needs the most). */
size_t dp_workspace_size_for(int B, int T, int d_in, int d_out, int r, dp_dtype dt,
                             dp_norm_method method);

/* Per-sample gradient norms n_i = ||X_i^T dY_i||_F, or ||X_i^T dY_i P||_F when P != NULL.
 * (FlashDP Abstract: per-sample gradient clipping needs each sample's gradient; DP-GRAPE
 * Methodology: the norm is taken after projection.)
 *   P      : NULL, or DEVICE [d_out, r] in dtype dt.
 *   norms  : DEVICE fp32 [B], overwritten. */
dp_status dp_per_sample_norms(const void* X, const void* dY, const void* P, int r, dp_dtype dt,
                              int B, int T, int d_in, int d_out, dp_norm_method method,
                              float* norms, void* workspace, size_t ws_bytes, void* stream);

/* G_sum += sum_i c_i X_i^T dY_i [P], where c_i = 1 if norms[i] <= C and C / norms[i] otherwise.
 * (FlashDP Abstract: per-layer clipped DP-SGD.)  No noise is added.
 *   norms  : DEVICE fp32 [B].  These may be this layer's norms, or flat norms
 *            sqrt(sum_l n_{i,l}^2) that the caller computed over several layers.
 *   C      : > 0.  +INF means no clipping.
 *   G_sum  : DEVICE fp32 [d_in, P ? r : d_out], accumulated into, so that several
 *            microbatches can be summed. */
dp_status dp_clip_accumulate(const void* X, const void* dY, const void* P, int r, dp_dtype dt,
                             int B, int T, int d_in, int d_out, const float* norms, float C,
                             float* G_sum, void* workspace, size_t ws_bytes, void* stream);

/* G[k] += std * z_k for k < rows*cols, with z from Philox stream 0 under (seed, step,
 * layer_id).  This is the Gaussian noise that follows clipping (DP-GRAPE Problem Statement
 * and Methodology).  Each element is added in fp64 and rounded once to fp32.
 *   G    : DEVICE fp32 [rows, cols], updated in place.
 *   std  : >= 0 and finite; it is sigma * C for a DP-SGD step. */
dp_status dp_add_noise(float* G, long long rows, long long cols, float std,
                       unsigned long long seed, unsigned long long step, unsigned layer_id,
                       void* stream);

/* P[b, j] = z_{b*r + j} / sqrt(r), with z from Philox stream 1 under (seed, step 0,
 * layer_id): a Gaussian matrix with N(0, 1/r) entries, regenerated from the seed, one per
 * layer (DP-GRAPE Methodology, "Random Projection over SVD").  The value is formed in fp64,
 * rounded to fp32, then for bf16 rounded to nearest even.
 *   P : DEVICE [d_out, r] in dtype dt, overwritten. */
dp_status dp_projection_matrix(void* P, dp_dtype dt, int d_out, int r,
                               unsigned long long seed, unsigned layer_id, void* stream);

/* One privatised step for one linear layer (FlashDP Abstract: one fused task per layer):
 *   norms_out[i] = n_i,
 *   G_out = sum_i c_i G_i [P] + sigma*C*z (Philox stream 0, (seed, step, layer_id)).
 * Projection: pass P (DEVICE [d_out, r]).  Or pass P = NULL with r > 0 to regenerate P from
 * (seed, layer_id) into the workspace, as dp_projection_matrix does.  r = 0 with P = NULL
 * is the unprojected step.
 *   C          : > 0.  +INF (no clipping) requires sigma = 0.
 *   sigma      : >= 0.
 *   norms_out  : NULL or DEVICE fp32 [B].
 *   G_out      : DEVICE fp32 [d_in, r or d_out], overwritten.  The gradients-once method
 *                rounds sigma*C*z to fp32 before adding it to the fp32 sum (within one ulp
 *                of rounding the fp64 sum once).  A ghost or explicit clipped sum split over
 *                K (small outputs) stores each split's partial sum in the workspace, and a
 *                combining launch adds sigma*C*z and the partials in split order in fp64,
 *                rounding once, so the result does not depend on the order the splits ran
 *                in.  An unsplit sum that runs in one wave gets sigma*C*z rounded to fp32 from
 *                the row-scaling launch before it and adds itself to that.  Otherwise the
 *                epilogue adds the noise in fp64 and rounds once.  bf16 results are the same
 *                bits on every run. */
dp_status dp_linear_step(const void* X, const void* dY, const void* P, int r, dp_dtype dt,
                         int B, int T, int d_in, int d_out, float C, float sigma,
                         unsigned long long seed, unsigned long long step, unsigned layer_id,
                         dp_norm_method method, float* norms_out, float* G_out,
                         void* workspace, size_t ws_bytes, void* stream);

/* dp_linear_step with the step number in device memory, read when the noise kernels run.
 * One CUDA graph captured around this call then serves every training step: the caller
 * advances *step_dev (on the device, or by a copy ordered on the stream) between replays.
 * (The pages have no counterpart; the noise counter is the same (seed, step, layer_id).)
 *   step_dev : DEVICE uint64, 8-byte aligned; only its low 32 bits enter the counter.
 * Capture only after one ordinary call with the same shapes and method on that device: the
 * first call of a kernel configuration sets its shared-memory attribute, which is not a
 * stream operation.  The call itself allocates nothing and does not synchronise. */
dp_status dp_linear_step_dev_step(const void* X, const void* dY, const void* P, int r,
                                  dp_dtype dt, int B, int T, int d_in, int d_out, float C,
                                  float sigma, unsigned long long seed,
                                  const unsigned long long* step_dev, unsigned layer_id,
                                  dp_norm_method method, float* norms_out, float* G_out,
                                  void* workspace, size_t ws_bytes, void* stream);

/* The raw Philox4x32-10 words behind every random number of the library (Salmon et al.,
 * "Parallel random numbers: as easy as 1, 2, 3", SC'11), exposed so that the uint32 stream
 * can be checked bit for bit: out[4 j + q] = word q of block j under counter
 * (j, layer_id, step mod 2^32, stream_id) and key (seed mod 2^32, seed >> 32), j < nblocks.
 *   out : DEVICE uint32 [nblocks, 4], overwritten; nblocks <= 2^32. */
dp_status dp_philox_blocks(unsigned* out, unsigned long long nblocks, unsigned long long seed,
                           unsigned long long step, unsigned layer_id, unsigned stream_id,
                           void* stream);

/* The Gaussian transform behind the gradient noise, exposed so that it can be checked on
 * chosen words (the noise itself reaches it only through Philox output).  Box and Muller
 * (1958) in fp64, evaluated exactly as the noise kernels evaluate it, before the scaling by
 * sigma*C: for q < npairs, with u1 = (words[2q] + 1) 2^-32 and u2 = words[2q+1] 2^-32,
 *   z[2q] = sqrt(-2 ln u1) cos(2 pi u2),  z[2q+1] = sqrt(-2 ln u1) sin(2 pi u2).
 * The evaluation is table-driven and agrees with the exact values to about 2e-12.
 *   words : DEVICE uint32 [npairs, 2]; z : DEVICE fp64 [npairs, 2], overwritten;
 *   both 16-byte aligned; 1 <= npairs <= 2^40. */
dp_status dp_box_muller(const unsigned* words, long long npairs, double* z, void* stream);

/* dp_per_sample_norms without a workspace, for callers that cannot allocate device memory.
 * Some callers cannot: code that runs inside another framework's allocator hook or a memory
 * budget it does not own, or a real-time loop that forbids new device allocations after
 * start-up.  (The pages have no counterpart of this entry point; it is a convenience of
 * this library.)
 *   - Unprojected only (no P), same arguments and results as dp_per_sample_norms.
 *   - Scratch is a fixed 1 MiB device array inside the library.  Every GPU that loads the
 *     library holds it until the process exits.  The call refuses shapes whose scratch would
 *     exceed it with DP_ERR_WORKSPACE (dp_last_cuda_error() gives the sizes).  bf16 needs
 *     about 512 + 8 B + 4 B * slots bytes, where slots is the largest of
 *     4 ceil(d_in/128) ceil(d_out/128), 8 ceil(d_in/256) ceil(d_out/256) and
 *     2 ceil(T/128) (ceil(T/128) + 1); e.g. B <= 63 for 4096 x 4096 linears.
 *   - It calls no cudaMalloc, cudaFree or other allocating routine.  The first call on each
 *     device looks up the array's device address (cudaGetSymbolAddress) with that device
 *     current.  Make that first call before any stream capture.  The address belongs to the
 *     CUDA context it was looked up in; a call in another context (after cudaDeviceReset, or
 *     with another driver context current) looks it up again, so make one such call before
 *     any capture in that context too.
 *   - Every call shares the one array, and each call clears what must start at zero.  Calls
 *     that overlap on the GPU (other streams, other host threads) race on it and give wrong
 *     norms: serialise them.
 *   - An in-kernel wait that times out is recorded only inside the array; use the workspace
 *     entry point when dp_workspace_status is needed. */
dp_status dp_per_sample_norms_static(const void* X, const void* dY, dp_dtype dt, int B, int T,
                                     int d_in, int d_out, dp_norm_method method, float* norms,
                                     void* stream);

/* ------------------------------------------------------------------ block step
 * One call for all the linears of a block that see the same samples (e.g. q, k, v, o, gate,
 * up, down of a transformer block).  Two clipping modes:
 *   DP_CLIP_PER_LAYER : each layer l is clipped with its own bound layers[l].C and gets noise
 *                       of std sigma * layers[l].C.  This is per-layer clipped DP-SGD
 *                       (FlashDP Abstract), the same result as one dp_linear_step per layer.
 *   DP_CLIP_FLAT      : one clip factor per sample for the whole block,
 *                       c_i = min(1, C / sqrt(sum_l n_{i,l}^2)).  The sample's gradient over
 *                       all the block's weights is clipped as one vector, as in textbook
 *                       DP-SGD.  Every layer's output gets noise of std sigma * C.
 * Each layer's noise uses its own layer_id in the Philox counter.  A layer with P clips,
 * sums and noises its projected gradient (the noise then has the [d_in, r] shape); its P is
 * given, not regenerated (make it once with dp_projection_matrix).
 * Layers whose norm method resolves to DP_NORM_GHOST and that point at the same X with the
 * same d_in and the same clip-space width (d_out, or r when projected; q/k/v, gate/up) are
 * grouped, up to three, and share one X Gram per pair of 128-token blocks; their norms are
 * bitwise those of one layer at a time. */
typedef struct {
    const void* X;        /* DEVICE [B, T, d_in] in dtype dt */
    const void* dY;       /* DEVICE [B, T, d_out] in dtype dt */
    int d_in, d_out;
    unsigned layer_id;
    float C;              /* the layer's bound (per-layer mode; ignored in flat mode) */
    float* G_out;         /* DEVICE fp32 [d_in, r or d_out], overwritten */
    float* norms_out;     /* NULL or DEVICE fp32 [B]: the layer's own per-sample norms */
    const void* P;        /* NULL, or DEVICE [d_out, r] in dtype dt: clip and noise the
                             projected gradient G_i P (DP-GRAPE), as dp_linear_step does */
    int r;                /* 0 without P; with P, a multiple of 8 (bf16) or 4 (fp32) */
} dp_layer;

typedef enum { DP_CLIP_PER_LAYER = 0, DP_CLIP_FLAT = 1 } dp_clip_mode;

/* Workspace bytes for dp_block_step with these layers (0 if a layer's shape is invalid).
 * Flat mode with DP_NORM_ONCE keeps every layer's per-sample tiles: sum_l B d_in d_out bf16;
 * per-layer mode finishes each layer first and needs one such region, for the largest. */
size_t dp_block_workspace_size(const dp_layer* layers, int L, int B, int T, dp_dtype dt,
                               dp_clip_mode mode, dp_norm_method method);

/* layers: HOST array of L descriptors; the tensors they point to are DEVICE memory.
 * C: the flat bound (> 0; flat mode only).  flat_norms_out: NULL or DEVICE fp32 [B],
 * sqrt(sum_l n_{i,l}^2) (flat mode only).  Other arguments as for dp_linear_step. */
dp_status dp_block_step(const dp_layer* layers, int L, dp_dtype dt, int B, int T,
                        dp_clip_mode mode, float C, float sigma, unsigned long long seed,
                        unsigned long long step, dp_norm_method method, float* flat_norms_out,
                        void* workspace, size_t ws_bytes, void* stream);

/* dp_block_step with the step number in device memory (see dp_linear_step_dev_step). */
dp_status dp_block_step_dev_step(const dp_layer* layers, int L, dp_dtype dt, int B, int T,
                                 dp_clip_mode mode, float C, float sigma, unsigned long long seed,
                                 const unsigned long long* step_dev, dp_norm_method method,
                                 float* flat_norms_out, void* workspace, size_t ws_bytes,
                                 void* stream);

/* ------------------------------------------------------------------ projected Adam
 * One projected Adam update.  DP-GRAPE page, Methodology, "Projected Optimizer States": the
 * optimizer state lives in the projected space, O(r x layers) instead of O(d).  The page
 * gives neither the averaging nor the map back to the weights; the plainest readings are
 * used:
 *   g = grad_scale * R                          (grad_scale = 1/B averages over the batch)
 *   m <- beta1 m + (1 - beta1) g,  v <- beta2 v + (1 - beta2) g^2
 *   U = (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)        (t >= 1)
 *   W <- W - lr U P^T                           (the r-space update mapped back through P)
 *   W    : DEVICE fp32 [d_in, d_out], updated in place.
 *   R    : DEVICE fp32 [d_in, r], the privatised projected gradient (G_out of a projected
 *          dp_linear_step).
 *   m, v : DEVICE fp32 [d_in, r], updated in place; zeros before the first step.
 *   P    : DEVICE [d_out, r] in dtype dt (bf16: U is rounded to bf16 for the tensor cores).
 *   workspace : DEVICE, 256-byte aligned, >= dp_adam_workspace_size(d_in, r) bytes.
 * d_in, d_out and r are multiples of 8. */
size_t dp_adam_workspace_size(int d_in, int r);
dp_status dp_projected_adam_step(float* W, const float* R, float* m, float* v, const void* P,
                                 dp_dtype dt, int d_in, int d_out, int r, float lr, float beta1,
                                 float beta2, float eps, float grad_scale, int t, void* workspace,
                                 size_t ws_bytes, void* stream);

/* Failure-detection self-test of the bounded in-kernel waits: a one-warp kernel waits on a
 * barrier that nothing arrives at.  After limit_ns nanoseconds (1 us .. 2 s) it gives up,
 * records the timeout in the workspace's status word and returns.  dp_workspace_status then
 * reports DP_ERR_TIMEOUT, and the device stays usable for further calls.
 *   workspace : DEVICE, 256-byte aligned, at least 256 bytes. */
dp_status dp_selftest_wait_timeout(void* workspace, unsigned long long limit_ns, void* stream);

/* Host-side fault injection, for tests of the error paths (no device fault is involved): the
 * library lets the next `skip` kernel launches of this process through, then makes the
 * `count` launches after them fail with `cuda_error` (a cudaError_t value, e.g. 2 for
 * cudaErrorMemoryAllocation) as if the runtime had refused them.  Nothing is enqueued for a
 * failed launch; the call that made it returns DP_ERR_CUDA and dp_last_cuda_error() names the
 * launch and the error.  count = 0 clears any pending injection.  The counters are global to
 * the process and shared by all threads.  Returns DP_ERR_INVALID_ARG for a negative count or
 * skip, or an error code <= 0 with count > 0. */
dp_status dp_selftest_fail_launches(long long skip, long long count, int cuda_error);

/* Synchronises `stream`, then reads the status word that the kernels of earlier calls wrote
 * into `workspace`.  Returns DP_OK, DP_ERR_TIMEOUT (a bounded in-kernel wait ran out; the
 * results of that call are invalid), DP_ERR_DEVICE_CHECK or DP_ERR_CUDA.  The word is cleared
 * at the start of every call that takes a workspace.
 * Debug build: the library compiled with -DDPCLIP_DEBUG (libdpclip_debug.so) checks, before each
 * main-loop store or load of its kernels, that the index lies inside the buffer the host
 * described.  A failed check never traps: it skips the access and records its site, here and
 * in a word of the module that this call also reads (that word is never cleared), and this
 * call then returns DP_ERR_DEVICE_CHECK with the site in dp_last_cuda_error().  In the normal
 * build the checks compile away. */
dp_status dp_workspace_status(const void* workspace, void* stream);

/* Norm method that DP_NORM_AUTO picks for these shapes (GHOST, EXPLICIT or ONCE).  For bf16,
 * the environment variable DPCLIP_NORM=ghost|explicit|once, read at every call, overrides the
 * cost model in every call made with DP_NORM_AUTO (and in dp_workspace_size); other values
 * are ignored.  fp32 always takes EXPLICIT. */
dp_norm_method dp_auto_norm_method(int B, int T, int d_in, int d_out, int r, dp_dtype dt);

/* Launch accounting, for measurement.  dp_kernel_launches() is the number of kernels this
 * library has launched in this process.  Once dp_profiling_enable(1) is called, every later
 * launch is bracketed by two CUDA events recorded on its own stream.
 * dp_profiling_collect(total_ms, launches) waits for those events and fills both arrays,
 * which the caller owns, with dp_profiling_kinds() entries: the device time and launch count
 * per kernel kind.  dp_profiling_kind_name() names a kind.  It then forgets the records.
 * dp_profiling_enable(0) stops recording.  Both calls drop records not yet collected. */
dp_status dp_profiling_enable(int on);
int dp_profiling_kinds(void);
const char* dp_profiling_kind_name(int kind);
dp_status dp_profiling_collect(double* total_ms, long long* launches);
long long dp_kernel_launches(void);

/* Static description of a status code. */
const char* dp_status_string(dp_status s);

/* The last CUDA error string seen by this thread's calls, or "" if none. */
const char* dp_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DPCLIP_H */
