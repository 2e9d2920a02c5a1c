/*
 * srnl_scan.h — C ABI of the B200 (sm_100a) SRNL four-direction chunked scan.
 *
 * The operation is the forward pass of the VisionHOPE operator's memory scan:
 *   - "VisionHOPE" README (github PSRben/VisionHOPE), sections "Overview" and
 *     "SRNL and VisionHOPE operator": image features in, same shape out, a new
 *     memory sequence on every call, head_dim-sized heads, row/column chunks.
 *   - "VisionHOPE Model Overview: Architecture, Benchmarks, and Practical
 *     Limits", sections "How VisionHOPE's Five Memories Work" (three matrix and
 *     two vector memories per head), "Four-Directional Scanning and Spatial
 *     Chunking" (four routes, per-route memories, shared query projection,
 *     boundary generation, restore and channel fusion) and "Why the Stability
 *     Controls Matter" (soft injection cap, spectral clamp).
 *   - "VisionHOPE: Visual Backbones as Self-Modifying Learning Systems"
 *     (summary of arXiv 2609.33325), write-rule, stability and 2D-maps
 *     paragraphs (retained delta gradient write, stabilized key normalisation,
 *     retention clamp, chunks equal to rows or columns).
 *
 * Layout.  Activations are channels-last: x[B][H][W][C] and y[B][H][W][C],
 * dense, row-major, element type act_dtype.  Channel c belongs to head
 * c / d, lane c % d.  Token raster index p = i*W + j.
 *
 * Routes.  r = 0 forward row-major, 1 reverse row-major, 2 forward
 * column-major (t = j*H + i), 3 reverse column-major.  Chunks hold chunk_row
 * (default W) consecutive tokens on routes 0/1 and chunk_col (default H) on
 * routes 2/3; the last chunk of a route may be shorter.
 *
 * Per (batch, head, route) the five memories M_mem, M_k, M_v (d x d) and
 * m_eta, m_alpha (1 x d) start from the route's initial states.  At each
 * chunk boundary they generate, for every token of the chunk,
 *   k~ = M_k x, v = M_v x, a = m_eta x, beta = m_alpha x        (x: head slice)
 * then  k = k~ / sqrt(|k~|^2 + eps),  alpha_t = min(sigmoid(beta), alpha),
 *       eta0 = softplus(a), g = |k - v| |k|,
 *       eta1 = eta0 * phi(eta0 g / (1 - alpha_t)),  phi(z) = tanh(z)/z,
 *       eta  = min(eta1, 2 / |k|^2),
 * and every memory X is written in token order
 *       X <- X alpha_t (I - eta k k^T) - eta (X k - X v) k^T.
 * The readout after token t's write is y_t = M_mem q_t with q = x W_q^T (all
 * C channels, split per head).  Outputs of the four routes are restored to
 * raster order and fused: y[p][c] = sum_r scales[r][c] * y_r[p][c] (r = 0..3).
 *
 * Precision.  Memory states and all recurrence arithmetic are fp32.
 * gen_dtype = SRNL_BF16 computes the boundary generation as a bf16 tensor-core
 * contraction with fp32 accumulation: the four generating memories at a chunk
 * boundary are G Q_b (G their initial states, Q_b the product of the
 * transitions so far), and each token's k~, v, a, beta = G (Q_b x); G and
 * Q_b x are rounded to bfloat16.  It also rounds the query-projection operands
 * (x, W_q) and the stored q to bfloat16, and runs the token-order write in its
 * chunkwise form: within a chunk every row of the state solves one shared
 * triangular system (fp32), and the products around it run on the tensor cores
 * with each fp32 operand split into bf16 high + low parts (about fp32 accuracy).
 * With bf16 activations as well, each route's scaled output is rounded to
 * bfloat16 before the four are summed in fp32 (in the order r0..r3) and
 * rounded once more to y.
 *
 * Errors.  Every entry point returns an srnl_status and never aborts.  On
 * failure the outputs are unspecified and srnl_scan_last_error() describes
 * the cause.  Kernels are asynchronous on the given stream: a CUDA error
 * raised by a kernel surfaces from a later call or a stream synchronisation.
 * No kernel of this library waits on another kernel, rank or flag; the scan
 * kernel's only waits are bounded polls on its own tensor-core completions and
 * on its own TMA copies (the stage tiles of bf16 activations arrive by
 * cp.async.bulk.tensor, without cluster multicast).
 *
 * Threads.  A handle may be used from one host thread at a time; forward
 * calls on one handle must not overlap on the device (they share the
 * handle's workspace).
 */
#ifndef SRNL_SCAN_H_
#define SRNL_SCAN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SRNL_API __attribute__((visibility("default")))
#else
#define SRNL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct srnl_scan srnl_scan; /* opaque; owned by the library */

typedef enum {
  SRNL_OK = 0,
  SRNL_E_INVAL = -1,       /* bad argument: NULL, shape, alignment, range */
  SRNL_E_UNSUPPORTED = -2, /* valid but not built (e.g. a head dim other than 4, 8, 16, 32, 64) */
  SRNL_E_CUDA = -3,        /* a CUDA runtime call failed */
  SRNL_E_NOMEM = -4,       /* device or pinned allocation failed */
  SRNL_E_TIMEOUT = -5      /* a bounded in-kernel wait gave up (see srnl_scan_device_status) */
} srnl_status;

typedef enum { SRNL_F32 = 0, SRNL_BF16 = 1 } srnl_dtype;

/* Injection cap on the proposed step ("VisionHOPE: Visual Backbones as Self-Modifying
 * Learning Systems", stability and results paragraphs): the soft cap
 * eta1 = eta0 tanh(z)/z, z = eta0 g / (1 - alpha_t) (the method), or the hard clamp of its
 * ablation, eta1 = min(eta0, (1 - alpha_t) / g), which is "active" on a token update when
 * eta0 g > 1 - alpha_t. */
typedef enum { SRNL_CAP_SOFT = 0, SRNL_CAP_HARD = 1 } srnl_cap;

typedef struct {
  int B, H, W, C; /* batch, height, width, channels (C = heads * d) */
  int heads, d;   /* heads and head dim: 4, 8, 16, 32 or 64 (below 32 the heads run zero-padded
                     to 32 lanes, which is exact; 64 runs 64-wide SIMT kernels, fp32 products
                     with the bf16 path's roundings when gen_dtype is SRNL_BF16; the
                     no-allocation forward takes 32 only) */
  float alpha;    /* retention cap, 0 < alpha < 1 (0.95 hierarchical, 0.9 plain) */
  float eps;      /* key normalisation epsilon, > 0 (1e-6) */
  int chunk_row;  /* chunk length on routes 0/1; 0 means W (full rows) */
  int chunk_col;  /* chunk length on routes 2/3; 0 means H (full columns) */
  int act_dtype;  /* srnl_dtype of x and y */
  int gen_dtype;  /* srnl_dtype of generation / projection operands */
  int injection_cap; /* srnl_cap; 0 = SRNL_CAP_SOFT */
} srnl_scan_config;

/* Parameters, HOST pointers to dense fp32 arrays.  srnl_scan_create copies and
 * repacks them into device memory owned by the handle; the caller may free
 * them when create returns. */
typedef struct {
  const float* W_q;      /* [C][C]   q = x W_q^T (shared by all routes)      */
  const float* scales;   /* [4][C]   channel fusion scales per route          */
  const float* M_mem0;   /* [4][heads][d][d] initial content memory per route */
  const float* M_k0;     /* [4][heads][d][d] initial key memory               */
  const float* M_v0;     /* [4][heads][d][d] initial value memory             */
  const float* m_eta0;   /* [4][heads][d]    initial step-size memory         */
  const float* m_alpha0; /* [4][heads][d]    initial retention memory         */
} srnl_scan_params;

/* Validate the config, allocate the handle, its device workspace and its
 * packed parameters on the CURRENT CUDA device.  *out is set to NULL on
 * failure.  Allocates with cudaMalloc; synchronous. */
SRNL_API srnl_status srnl_scan_create(srnl_scan** out, const srnl_scan_config* cfg,
                             const srnl_scan_params* params);

/* Forward pass.  x and y are DEVICE pointers on the handle's device, 16-byte
 * aligned, [B][H][W][C] of act_dtype; x and y must not overlap.
 * final_states: optional DEVICE pointer to fp32
 * [4][B][heads][3*d*d + 2*d] receiving the memories after the last token of
 * each route (M_mem, M_k, M_v row-major, then m_eta, m_alpha); NULL skips it.
 * stream: a cudaStream_t (NULL = legacy default stream).  Asynchronous. */
SRNL_API srnl_status srnl_scan_forward(srnl_scan* h, const void* x, void* y,
                              float* final_states, void* stream);

/* Same forward with HOST buffers: copies x host->device, runs the forward and
 * copies y device->host on `stream`, then synchronises the stream.  x/y are
 * host pointers of B*H*W*C act_dtype elements; pinned memory gives full copy
 * bandwidth.  Uses staging buffers owned by the handle. */
SRNL_API srnl_status srnl_scan_forward_host(srnl_scan* h, const void* x_host, void* y_host,
                                   void* stream);

/* Allocation-free forward (the pages have no counterpart: this is an
 * interface for callers, not part of the method).  It is for callers that
 * must not call cudaMalloc: code hosted by a framework that owns all device
 * memory through its own pool, where a raw allocation bypasses its accounting,
 * and latency-critical loops where an allocation may synchronise the device.
 * No handle is created and nothing is allocated or freed; the scratch (packed
 * parameters, projected queries, route partials, a status word) is a
 * file-scope device array of SRNL_NOALLOC_SCRATCH_BYTES that every GPU loading
 * this library holds until the process exits.
 *   cfg    : same rules as srnl_scan_create; head dim d = 32 only.
 *   params : DEVICE (or managed) pointers on the current device, same layouts
 *            as srnl_scan_params, each 4-byte aligned (fp32 arrays).
 *   x, y   : DEVICE (or managed) pointers on the current device as in
 *            srnl_scan_forward, 16-byte aligned, not overlapping.
 * Host pointers, pointers of another device, misaligned pointers and a
 * workload needing more than SRNL_NOALLOC_SCRATCH_BYTES of scratch (about
 * 18 bytes per activation element on the bf16 path, 20 on fp32, plus the
 * parameters) are rejected with SRNL_E_INVAL before anything is launched;
 * the message gives the reason (and both sizes).  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress) and sets
 * the kernels' function attributes with that device current; make that first
 * call before any stream capture.  All calls share the array and it keeps the
 * last call's contents: each call first clears the status word (an
 * asynchronous memset on `stream`), and everything else it reads it writes
 * itself; calls that overlap on the GPU race.  Argument and launch errors come
 * back as the status and through srnl_scan_last_error(NULL); a bounded
 * in-kernel wait that gives up is reported by srnl_scan_noalloc_status.
 * Asynchronous on `stream`. */
#define SRNL_NOALLOC_SCRATCH_BYTES (32u << 20)
SRNL_API srnl_status srnl_scan_forward_noalloc(const srnl_scan_config* cfg,
                                               const srnl_scan_params* params,
                                               const void* x, void* y, void* stream);

/* Device status of the last srnl_scan_forward_noalloc on the current device (no
 * counterpart on the pages either): waits for `stream`, then reads the status word of the
 * shared scratch array.  Returns SRNL_OK, or SRNL_E_TIMEOUT when a bounded in-kernel wait of
 * that forward gave up (its y is then unspecified).  The next no-allocation forward clears
 * the word.  Allocates nothing. */
SRNL_API srnl_status srnl_scan_noalloc_status(void* stream);

/* Test hook: the device computes the route map the scan kernels use and
 * writes out[t] = raster index of the t-th token of `route`, t < H*W, into the
 * DEVICE int32 buffer `out`.  Asynchronous. */
SRNL_API srnl_status srnl_scan_route_index(const srnl_scan* h, int route, int32_t* out,
                                  void* stream);

/* Test hook: xr[b][t][c] = x[b][perm_route(t)][c] on the device (act_dtype,
 * DEVICE pointers, 16-byte aligned).  Asynchronous. */
SRNL_API srnl_status srnl_scan_gather(const srnl_scan* h, int route, const void* x, void* xr,
                             void* stream);

/* Stage timing.  srnl_scan_enable_stage_timing(h, n) with n > 0 makes each
 * later forward record CUDA events on its stream before and after each of its
 * three kernels (query projection, scan, fusion), keeping the events of the
 * last n forwards (n <= 1024); n = 0 turns timing off.  A backward call records
 * its three stages in the same ring (query projection, scan backward, combine:
 * route sums, dx, dW_q and the parameter reductions); time one kind of call per
 * window. 
 * srnl_scan_stage_times waits for those events, writes the mean duration in
 * milliseconds of each kernel over the kept forwards to ms_out[0..2] and the
 * number of forwards averaged to *count (may be NULL), then starts a new
 * window.  Returns SRNL_E_INVAL if timing is off or no forward ran. */
SRNL_API srnl_status srnl_scan_enable_stage_timing(srnl_scan* h, int n);
SRNL_API srnl_status srnl_scan_stage_times(srnl_scan* h, float* ms_out, int* count);

/* Pipelined forward with HOST buffers, for a loop of steps: copies x host->device on
 * an internal copy stream, runs the forward on `stream`, copies y device->host on a
 * second internal copy stream, and returns without waiting.  Two staging slots alternate,
 * so one call's copies overlap the neighbouring calls' forwards.  x_host must stay
 * unchanged and y_host unread until the copies are done: srnl_scan_host_sync(h) waits
 * for them on the host, srnl_scan_host_join(h, stream) makes `stream` wait for them.
 * Pinned host memory is needed for the copies to overlap. */
SRNL_API srnl_status srnl_scan_forward_host_async(srnl_scan* h, const void* x_host, void* y_host,
                                                 void* stream);
SRNL_API srnl_status srnl_scan_host_join(srnl_scan* h, void* stream);
SRNL_API srnl_status srnl_scan_host_sync(srnl_scan* h);

/* Device status of the handle's kernels: synchronously reads the status word
 * the scan kernel sets when one of its bounded waits (for its own tensor-core
 * work) gives up.  Returns SRNL_OK, or SRNL_E_TIMEOUT once that has happened
 * (outputs of that forward are then unspecified). */
SRNL_API srnl_status srnl_scan_device_status(srnl_scan* h);

/* Number of token updates (all routes, batches and heads) of the last forward on which
 * the hard injection clamp was active; 0 under the soft cap.  Synchronises the device.
 * (srnl_scan_forward_noalloc does not count.) */
SRNL_API srnl_status srnl_scan_cap_count(srnl_scan* h, unsigned long long* count);

/* ------------------------------------------------------------------------
 * Backward pass (reverse-mode gradient of the forward above; the layer is trained end to
 * end inside the backbone: "VisionHOPE" README, "SRNL and VisionHOPE operator").
 * For a loss L with upstream gradient dy = dL/dy, it returns dL/dx and the gradients of
 * every parameter of srnl_scan_params, taking the active branch of each clamp (the
 * retention clamp, the hard injection clamp, the spectral clamp).
 *
 * Gradient buffers: DEVICE pointers to dense fp32 arrays in the layouts of
 * srnl_scan_params; each is OVERWRITTEN (not accumulated) and each may be NULL to skip it.
 * ---------------------------------------------------------------------- */
typedef struct {
  float* W_q;      /* [C][C]            */
  float* scales;   /* [4][C]            */
  float* M_mem0;   /* [4][heads][d][d]  */
  float* M_k0;     /* [4][heads][d][d]  */
  float* M_v0;     /* [4][heads][d][d]  */
  float* m_eta0;   /* [4][heads][d]     */
  float* m_alpha0; /* [4][heads][d]     */
} srnl_scan_grads;

/* Backward pass.  x: the forward's input; dy: dL/dy; dx: receives dL/dx.  DEVICE
 * pointers, 16-byte aligned, [B][H][W][C] of act_dtype; dx must not overlap x or dy.
 * grads may be NULL (only dx).  The handle must have gen_dtype SRNL_F32 (otherwise
 * SRNL_E_UNSUPPORTED): all arithmetic is fp32; act_dtype SRNL_BF16 means bf16 x, dy and dx.
 * The forward is recomputed from x (boundary products are kept per chunk and the states
 * inside a chunk recomputed), so no forward state is needed.  The first call allocates the
 * backward workspace (cudaMalloc, synchronous; about 9 fp32 values per activation element,
 * plus per (route, batch, head) sequence (2 w + 8) floats per token and w^2 floats per chunk
 * and per token of its longest chunk, w = 32 or 64 the kernels' head width); later calls
 * reuse it.  Asynchronous on `stream`; shares the handle's workspace with the forward. */
SRNL_API srnl_status srnl_scan_backward(srnl_scan* h, const void* x, const void* dy, void* dx,
                                       const srnl_scan_grads* grads, void* stream);

/* ------------------------------------------------------------------------
 * The VisionHOPE residual block around the operator ("VisionHOPE: Visual Backbones as
 * Self-Modifying Learning Systems", 2D-maps paragraph: a standard two-branch residual,
 * depthwise conv for local context, SRNL for long range, then an FFN; "VisionHOPE Model
 * Overview", "Four-Directional Scanning and Spatial Chunking": projections, normalization,
 * depthwise convolution and a feed-forward network; "VisionHOPE" README, "SRNL and VisionHOPE
 * operator": shape-preserving, mixer_dim sets the internal width).  The pages do not print
 * the wiring; this library reads it as (channels-last, m = mixer_dim)
 *   u   = LN1(x) W_in^T + b_in
 *   mix = DWConv3x3(u) + operator(u)          (3 x 3 per channel, zero padding, bias)
 *   y   = x + mix W_out^T + b_out
 *   out = y + GELU(LN2(y) W_1^T + b_1) W_2^T + b_2      (hidden width 4 dim, GELU v Phi(v))
 * with LayerNorm over channels (scale and shift, epsilon ln_eps).  bf16 activations; the
 * projections run as bf16 tensor-core products with fp32 accumulation and bf16 outputs, the
 * normalisations and the convolution in fp32 arithmetic.
 * ---------------------------------------------------------------------- */
typedef struct srnl_block srnl_block; /* opaque; owned by the library */

typedef struct {
  int B, H, W;        /* batch, height, width                                     */
  int dim;            /* channels of x and y: a multiple of 32, at most 512      */
  int mixer_dim;      /* width of the mixer and the operator: a multiple of 32, at most 512 */
  int head_dim;       /* the operator's head dim (4, 8, 16, 32 or 64)             */
  float alpha, eps;   /* the operator's retention cap and key epsilon              */
  int chunk_row, chunk_col; /* the operator's chunks (0: full rows / columns)    */
  int act_dtype;      /* SRNL_BF16                                                */
  int gen_dtype;      /* the operator's generation dtype                          */
  int injection_cap;  /* srnl_cap of the operator                                 */
  float ln_eps;       /* LayerNorm epsilon, > 0 (1e-6)                            */
} srnl_block_config;

/* HOST pointers to dense fp32 arrays, copied (weights rounded to bf16) at create. */
typedef struct {
  const float *ln1_g, *ln1_b;   /* [dim]                      */
  const float *W_in, *b_in;     /* [m][dim], [m]              */
  const float *dw_w, *dw_b;     /* [m][3][3], [m]             */
  srnl_scan_params op;          /* the operator at width m (C = m, heads = m / head_dim) */
  const float *W_out, *b_out;   /* [dim][m], [dim]            */
  const float *ln2_g, *ln2_b;   /* [dim]                      */
  const float *W_1, *b_1;       /* [4 dim][dim], [4 dim]      */
  const float *W_2, *b_2;       /* [dim][4 dim], [dim]        */
} srnl_block_params;

/* Validate, pack the parameters and allocate the block's workspace (six bf16 buffers of
 * B*H*W rows: dim, m, m, m, dim and 4 dim wide) and its operator handle on the CURRENT
 * device.  cudaMalloc; synchronous.  *out is NULL on failure. */
SRNL_API srnl_status srnl_block_create(srnl_block** out, const srnl_block_config* cfg,
                                       const srnl_block_params* params);
/* out = block(x): DEVICE pointers, bf16 [B][H][W][dim], 16-byte aligned, not overlapping.
 * Asynchronous on `stream` (eight kernels plus the operator's); calls on one handle must not
 * overlap on the device. */
SRNL_API srnl_status srnl_block_forward(srnl_block* h, const void* x, void* y, void* stream);
/* Synchronously reads the status words of the block's and its operator's kernels: SRNL_OK,
 * or SRNL_E_TIMEOUT once a bounded in-kernel wait gave up. */
SRNL_API srnl_status srnl_block_device_status(srnl_block* h);
SRNL_API const char* srnl_block_last_error(const srnl_block* h);
SRNL_API void srnl_block_destroy(srnl_block* h);

/* Self-test of the failure path of the bounded in-kernel waits: on the CURRENT device, runs
 * the scan kernels' bounded mbarrier wait on a barrier that nothing completes, with a
 * wall-time limit of wait_ms milliseconds (1..5000).  Returns SRNL_E_TIMEOUT when the wait
 * gave up as designed (the expected result; the device and context stay usable),
 * SRNL_OK if the wait wrongly completed, SRNL_E_INVAL for wait_ms out of range (no device
 * work), SRNL_E_CUDA on a CUDA error.  Synchronous; the message is srnl_scan_last_error(NULL). */
SRNL_API srnl_status srnl_selftest_wait_timeout(int wait_ms);

/* The same bounded wait on a barrier nothing completes, run asynchronously on `stream`
 * with the no-allocation forward's status word as its status (1 <= wait_ms <= 5000): after
 * it, srnl_scan_noalloc_status returns SRNL_E_TIMEOUT until the next no-allocation forward
 * clears the word.  Tests the no-allocation forward's failure report without a fault.
 * Allocates nothing. */
SRNL_API srnl_status srnl_selftest_noalloc_wait_timeout(int wait_ms, void* stream);

/* Bytes of device workspace the handle holds (packed params excluded). */
SRNL_API size_t srnl_scan_workspace_bytes(const srnl_scan* h);

/* Message for the last failure on this handle; with h == NULL, the last
 * failure of srnl_scan_create on the calling thread.  Never NULL. */
SRNL_API const char* srnl_scan_last_error(const srnl_scan* h);

/* Static name of a status code. */
SRNL_API const char* srnl_status_string(int status);

/* Free the handle and all its device memory.  Accepts NULL.  Synchronises the
 * device before freeing. */
SRNL_API void srnl_scan_destroy(srnl_scan* h);

/* ------------------------------------------------------------------------
 * Standalone SRNL layer on sequences ("VisionHOPE" README, section "SRNL and
 * VisionHOPE operator": a layer on [batch, tokens, dim] returning the same
 * shape; queries of the same shape may be passed, otherwise x is the query;
 * 64-token chunks unless a positive length is given; an incomplete final chunk
 * is allowed; every call starts a new sequence).
 *
 * One pass in token order (no routes, no fusion).  Per (batch, head) the five
 * memories start from the layer's initial states and follow the recurrence
 * above with x_t and q_t the head's d-slices of x and of the queries;
 * y[b][t][h*d + i] = (M_mem q_t)[i] after token t's write.  There is no input
 * or output projection.  Precision paths as above (gen_dtype = SRNL_BF16:
 * bf16 queries and generation, chunkwise write; SRNL_F32: fp32 throughout).
 * ---------------------------------------------------------------------- */
typedef struct srnl_seq srnl_seq; /* opaque; owned by the library */

typedef struct {
  int B, T, D;    /* batch, tokens, dim (D = heads * d) */
  int heads, d;   /* heads and head dim: 4, 8, 16, 32 or 64 (as srnl_scan_config) */
  float alpha;    /* retention cap, 0 < alpha < 1 */
  float eps;      /* key normalisation epsilon, > 0 */
  int chunk;      /* chunk length; 0 means 64 */
  int act_dtype;  /* srnl_dtype of x, the queries and y */
  int gen_dtype;  /* srnl_dtype of generation / query operands */
  int injection_cap; /* srnl_cap; 0 = SRNL_CAP_SOFT */
} srnl_seq_config;

/* Initial states, HOST pointers to dense fp32 arrays, copied by create. */
typedef struct {
  const float* M_mem0;   /* [heads][d][d] */
  const float* M_k0;     /* [heads][d][d] */
  const float* M_v0;     /* [heads][d][d] */
  const float* m_eta0;   /* [heads][d]    */
  const float* m_alpha0; /* [heads][d]    */
} srnl_seq_params;

/* Validate, allocate the handle and its workspace on the CURRENT device.
 * *out is NULL on failure; the message is srnl_seq_last_error(NULL). */
SRNL_API srnl_status srnl_seq_create(srnl_seq** out, const srnl_seq_config* cfg,
                                     const srnl_seq_params* params);

/* Forward pass.  x, q, y: DEVICE pointers, 16-byte aligned, [B][T][D] of
 * act_dtype; q may be NULL (x is then the query); y must not overlap x or q.
 * final_states: optional DEVICE fp32 [B][heads][3*d*d + 2*d] (M_mem, M_k,
 * M_v row-major, m_eta, m_alpha after the last token), NULL skips it.
 * Asynchronous on `stream` (a cudaStream_t, NULL = legacy default stream). */
SRNL_API srnl_status srnl_seq_forward(srnl_seq* h, const void* x, const void* q, void* y,
                                      float* final_states, void* stream);

/* Backward pass of the sequence layer (see srnl_scan_backward): for dy = dL/dy it writes
 * dx = dL/dx and, when q is given and dq is not NULL, dq = dL/dq (DEVICE, 16-byte aligned,
 * [B][T][D] of act_dtype; with q == NULL x is also the query, its gradient is included in
 * dx and dq must be NULL).  grads: DEVICE fp32 buffers in the srnl_seq_params layouts,
 * overwritten, each may be NULL (or grads NULL).  gen_dtype must be SRNL_F32 (else
 * SRNL_E_UNSUPPORTED).  The first call allocates the backward workspace.  Asynchronous. */
typedef struct {
  float* M_mem0;   /* [heads][d][d] */
  float* M_k0;     /* [heads][d][d] */
  float* M_v0;     /* [heads][d][d] */
  float* m_eta0;   /* [heads][d]    */
  float* m_alpha0; /* [heads][d]    */
} srnl_seq_grads;
SRNL_API srnl_status srnl_seq_backward(srnl_seq* h, const void* x, const void* q, const void* dy, void* dx,
                                      void* dq, const srnl_seq_grads* grads, void* stream);

/* Synchronously reads the status word of the handle's kernels (SRNL_OK or
 * SRNL_E_TIMEOUT, as srnl_scan_device_status). */
SRNL_API srnl_status srnl_seq_device_status(srnl_seq* h);

/* Hard-clamp activations of the last forward (see srnl_scan_cap_count). */
SRNL_API srnl_status srnl_seq_cap_count(srnl_seq* h, unsigned long long* count);

/* Message for the last failure on this handle (h == NULL: the calling
 * thread's last srnl_seq_create failure).  Never NULL. */
SRNL_API const char* srnl_seq_last_error(const srnl_seq* h);

/* Free the handle and its device memory.  Accepts NULL.  Synchronises the
 * device before freeing. */
SRNL_API void srnl_seq_destroy(srnl_seq* h);

#ifdef __cplusplus
}
#endif

#endif /* SRNL_SCAN_H_ */
