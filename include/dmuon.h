/*
 * dmuon.h -- C ABI of the B200 (sm_100a) Muon / DMuon optimizer step.
 *
 * One call updates a set of 2-D weight matrices in place.  For every matrix
 * (rows x cols, row-major, contiguous):
 *
 *   B' = mu*B + G                      momentum buffer, in place
 *   U  = G + mu*B'                     Nesterov look-ahead (nesterov = 1)
 *   X  = U, or U^T when rows > cols    iterate on the wide orientation
 *   X0 = X / (||X||_F + eps)
 *   K times:  A = X X^T,  X <- a X + (b A + c A^2) X        (quintic NS)
 *   O  = X_K (transposed back)
 *   W' = (1 - lr*wd) W - lr * 0.2*sqrt(max(rows, cols)) * O
 *
 * Sources (page title, section):
 *   "DeepSpeed 現已支援 Muon Optimizer" (setupai.cc), 技術深入: Muon
 *     orthogonalises the momentum-based update of 2-D weights by
 *     Newton-Schulz iterations, with decoupled weight decay and a
 *     per-parameter scale chosen by RMS matching so AdamW's lr/wd carry over.
 *   DMuon release article (wjxwpt.net), section 2 "shape-adaptive execution
 *     stack": the NS iteration may run in the m x m Gram space, small
 *     matrices are grouped to fill the GPU, and the math form and kernel are
 *     chosen per shape; section 3: each shape group's full computation is
 *     measured once and the measured costs drive the work order.
 *   DMuon announcement (m.zaocj.com), "自變量三招": on a new shape the
 *     candidate kernels are timed, the best is kept and reused for that shape.
 * The pages fix neither the coefficients nor eps; the defaults are
 * (a, b, c) = (3.4445, -4.7750, 2.0315), eps = 1e-7, K = 5.
 * Precision: with bf16 parameters the iterate and the m x m matrices are
 * rounded to bf16 between tensor-core products (fp32 accumulation, fp32
 * epilogues), except that an iterate of at most 5 rows (min(rows, cols) <= 5)
 * stays fp32 throughout on the CUDA cores: with so few, nearly equal
 * singular values bf16 roundings would move O by several percent.  fp32
 * parameters: fp32 throughout.
 *
 * Conventions for every entry point:
 *   - Device pointers are CUDA device memory of the current device; the
 *     pointer ARRAYS (params, grads, ...) and `shapes` are HOST memory, read
 *     during the call only.  The caller owns every buffer it passes.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     asynchronous on it.  The first call that meets a new shape group
 *     autotunes it and synchronises `stream` (see dmuon_step).
 *   - Return 0 on success, a negative DMUON_ERR_* code on failure;
 *     dmuon_last_error() gives a message (thread-local).  Any error detected
 *     before the first launch leaves every caller buffer untouched.
 *   - Aliasing between params, grads and momenta of any matrices is
 *     undefined.  NaN/Inf in a gradient propagates into that matrix only.
 *   - Calls are serialised per device inside the library; GPU work of two
 *     calls is ordered through an internal event, so calls on different
 *     streams are safe.
 */
#ifndef DMUON_H
#define DMUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DMUON_VERSION 1

/* Status codes. */
#define DMUON_OK 0
#define DMUON_ERR_INVALID (-1)        /* null pointer, bad shape/count/steps, non-finite hyperparameter;
                                         a side above 2^20 or more than 2^31 elements in one matrix */
#define DMUON_ERR_DTYPE (-2)          /* unsupported dtype combination */
#define DMUON_ERR_CUDA (-3)           /* a CUDA runtime/driver call failed */
#define DMUON_ERR_OOM (-4)            /* workspace allocation failed or caller workspace too small */
#define DMUON_ERR_DEVICE_TIMEOUT (-5) /* a bounded device-side wait ran out (pipeline stalled) */

/* Element types. */
typedef enum dmuon_dtype { DMUON_BF16 = 0, DMUON_F32 = 1 } dmuon_dtype;

/* Newton-Schulz form.  AUTO lets the per-shape autotuner choose. */
typedef enum dmuon_variant {
  DMUON_VARIANT_AUTO = 0,
  DMUON_VARIANT_DIRECT = 1,  /* iterate on X (m x n): 5 x (m^2 n + m^3 + m^2 n) GEMMs */
  DMUON_VARIANT_GRAM = 2,    /* iterate on Q (m x m), one m x m x n product at the end */
  DMUON_VARIANT_BATCHED = 3  /* resident, every step in one launch.  bf16, m <= 128, n <= 512: up
                                to 8 small matrices per CTA, iterate, A and P in shared memory for
                                all steps.  bf16, other m <= 256, n <= 1024 with 4n >= 5m: one CTA
                                pair per matrix, the Gram-space chain (A, P, Q, m x m) in shared
                                memory, X read twice.  fp32 iterate (fp32
                                parameters, or at most 5 rows), m <= 1024: one cooperative launch
                                over all SMs, a grid barrier between products.  Other shapes run
                                as AUTO */
} dmuon_variant;

/* Options of dmuon_step_ex.  Zero-initialise, then call dmuon_options_init. */
typedef struct dmuon_options {
  int param_dtype;   /* dmuon_dtype of W   (default DMUON_BF16) */
  int grad_dtype;    /* dmuon_dtype of G   (default DMUON_BF16) */
  int mom_dtype;     /* dmuon_dtype of B   (default DMUON_F32; only F32 supported) */
  float eps;         /* added to ||X||_F    (default 1e-7) */
  int nesterov;      /* 1: U = G + mu*B'; 0: U = B'  (default 1) */
  int variant;       /* dmuon_variant      (default AUTO) */
  float ns_a, ns_b, ns_c; /* quintic coefficients (default 3.4445, -4.7750, 2.0315) */
} dmuon_options;

/* Fill `opts` with the defaults listed above. */
void dmuon_options_init(dmuon_options* opts);

/*
 * dmuon_step -- one Muon step over `count` matrices, bf16 params and grads,
 * fp32 momenta.
 *   params[i]  device, rows_i x cols_i row-major, bf16; updated in place.
 *   grads[i]   device, same shape, bf16; read only.
 *   momenta[i] device, same shape, fp32; updated in place (B').
 *   shapes     host, 2*count int64: shapes[2i] = rows_i, shapes[2i+1] = cols_i.
 *   count      >= 0; 0 returns DMUON_OK without work.
 *   lr, wd, mu finite floats; ns_steps in [0, 16].
 * Matrices are grouped by (rows, cols); each group is planned once per
 * process (variant and tiles chosen by timing candidates on that group's
 * data; this first call synchronises `stream` and writes nothing to the
 * caller's buffers while timing) and groups run in descending measured cost.
 */
int dmuon_step(void* const* params, const void* const* grads, void* const* momenta,
               const int64_t* shapes, int count, float lr, float wd, float mu,
               int ns_steps, void* stream);

/* dmuon_step with explicit dtypes and options.  opts == NULL means defaults.
 * Supported: param/grad both BF16 (tensor-core path, bf16 operands, fp32
 * accumulate; an iterate of at most 5 rows in fp32 on the CUDA cores) or
 * both F32 (fp32 SIMT path); momenta F32. */
int dmuon_step_ex(void* const* params, const void* const* grads, void* const* momenta,
                  const int64_t* shapes, int count, float lr, float wd, float mu,
                  int ns_steps, const dmuon_options* opts, void* stream);

/*
 * dmuon_step_host_io -- dmuon_step_ex for gradients that live in HOST memory
 * (e.g. reduced or offloaded on the CPU), with the updated parameters copied
 * back to host memory.  The call splits every shape group into chunks of
 * about 16 MB of gradients (DMUON_IO_CHUNK_MB) and pipelines them over two
 * internal copy streams: later chunks' gradients travel host->device
 * (through four staging slots in the scratch) while a chunk is computed and
 * earlier chunks' parameters travel device->host.  Once every plan is
 * cached, consecutive chunks alternate between `stream` and an internal
 * compute stream, a quarter of the first and of the last chunk run as
 * pieces of their own (a short pipeline fill and drain), and when one shape
 * group is compute-bound (square matrices) and another copy-bound (wide
 * ones), the chunks of the groups run
 * interleaved, each group's spread evenly over the call, so that both kinds
 * overlap.  Matrices of at most 256 KB whose host buffers are pinned
 * and 16-byte aligned are copied by a kernel that reads and writes the
 * mapped host memory, one launch per chunk; other matrices take one
 * copy-engine transfer each (DMUON_IO_COPY=dma|kernel forces one kind;
 * out-kernel takes the kernel for every copy-out).
 *   params[i]          device, updated in place (as dmuon_step).
 *   grads_host[i]      host, rows_i x cols_i row-major; pinned (page-locked)
 *                      memory for the copies to run asynchronously.
 *   momenta[i]         device fp32, updated in place.
 *   params_host_out    NULL (no copy-out) or host pointers that receive the
 *                      updated parameters (pinned for asynchronous copies).
 * Asynchronous on `stream`: the host buffers must stay valid, and
 * params_host_out is complete, only once `stream` has reached the end of the
 * call's work (e.g. after cudaStreamSynchronize).  Side streams for small
 * groups are not used in this mode.
 */
int dmuon_step_host_io(void* const* params, const void* const* grads_host, void* const* momenta,
                       void* const* params_host_out, const int64_t* shapes, int count, float lr,
                       float wd, float mu, int ns_steps, const dmuon_options* opts, void* stream);

/*
 * dmuon_compute_update -- everything but the parameter write: updates the
 * momenta like dmuon_step and writes the orthogonalised update O (before the
 * 0.2*sqrt(max) scale) to out[i], device fp32, rows_i x cols_i row-major.
 * For parity tests and for callers that apply O themselves.
 */
int dmuon_compute_update(const void* const* grads, void* const* momenta,
                         const int64_t* shapes, int count, float mu, int ns_steps,
                         const dmuon_options* opts, float* const* out, void* stream);

/*
 * dmuon_compute_update_noalloc -- dmuon_compute_update for ONE matrix that
 * allocates nothing.  No counterpart on the pages: it exists for callers that
 * cannot allocate device memory inside their step, e.g. a framework whose
 * caching allocator owns all of device memory and forbids outside cudaMalloc,
 * or a loop that cannot take the device-wide synchronisation that
 * cudaMalloc/cudaFree imply.  (dmuon_set_workspace is the other route.)
 *   grad      device, rows x cols row-major (dtype opts->grad_dtype); read only.
 *   momentum  device, rows x cols fp32; updated in place (B').
 *   out       device, rows x cols fp32: the update O, as dmuon_compute_update.
 * Scratch is a fixed 64 MiB array in the library's device image, held by
 * every GPU that loads the library until the process exits.  A matrix whose
 * scratch exceeds it (about 4M bf16 elements for a square matrix, more for
 * wide ones) is rejected with DMUON_ERR_INVALID before any launch.  The
 * first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  The address is kept for the life of the process, so
 * cudaDeviceReset while the library is loaded is not supported.
 * Plan: opts->variant == DMUON_VARIANT_BATCHED runs a resident kernel when
 * the shape fits one (see DMUON_VARIANT_BATCHED); otherwise the call uses the
 * plan the autotuner cached for this shape (count 1) when there is one, else
 * the direct form; it never autotunes.
 * All calls share the one array and it keeps the last call's contents (each
 * call writes every word it reads before reading it, except the error word
 * below): calls whose GPU work overlaps, e.g. on two streams without
 * ordering between them, race.
 * A bounded device-side wait that gives up (DMUON_ERR_DEVICE_TIMEOUT) leaves
 * its code in an error word of the array; the call that launched it has
 * already returned.  Each call first reads that word (4 bytes, on the
 * per-thread default stream, so it does not wait for `stream`), except while
 * `stream` is being captured; if it holds a code, the call clears it and
 * returns DMUON_ERR_DEVICE_TIMEOUT without launching anything.  A timeout is
 * therefore reported by a later call of this entry point.
 * Calls no cudaMalloc, cudaFree or other allocating routine.
 */
int dmuon_compute_update_noalloc(const void* grad, void* momentum, int64_t rows, int64_t cols, float mu,
                                 int ns_steps, const dmuon_options* opts, float* out, void* stream);

/*
 * dmuon_gemm_bf16 -- the tensor-core GEMM core on its own (tests, tuning):
 *   D[l] = alpha * A[l] * op(B[l]) + beta * C[l]            l = 0..batch-1
 * A: device bf16, M x K row-major (K contiguous), leading dim lda, batch
 *    stride sa (elements).  B: device bf16; b_kmajor = 1: stored N x K
 *    (op(B) = B^T), b_kmajor = 0: stored K x N (op(B) = B).  C, D: device
 *    bf16 M x N (C may be NULL => beta ignored).  All leading dims and batch
 *    strides must be multiples of 8 elements and pointers 16-byte aligned.
 *    tile: 128 or 256 = one CTA per 128 x tile output tile, 512 = a CTA pair
 *    (tcgen05 cta_group::2) per 256 x 256 tile, 0 = 256.
 *    sym = 1 (needs M == N) declares the result symmetric: only the tiles
 *    that meet the upper triangle are computed and each element (r, c >= r)
 *    is also written to (c, r).
 */
int dmuon_gemm_bf16(const void* A, int64_t lda, int64_t sa, const void* B, int64_t ldb,
                    int64_t sb, int b_kmajor, const void* C, int64_t ldc, int64_t sc,
                    void* D, int64_t ldd, int64_t sd, int M, int N, int K, int batch,
                    float alpha, float beta, int tile, int sym, void* stream);

/* Autotune cache: save / load (text, one line per shape key, keyed also by
 * GPU name, SM count and library version) and clear. */
int dmuon_cache_save(const char* path);
int dmuon_cache_load(const char* path);
void dmuon_cache_clear(void);

/* Number of cached shape keys, and the plan of key `i` as text
 * ("rows cols dtype steps variant tile chunk cost_ms", dtype being the
 * iterate's: "f32" for fp32 parameters and for iterates of at most 5 rows)
 * into buf (NUL-terminated). */
int dmuon_cache_size(void);
int dmuon_cache_entry(int i, char* buf, size_t len);

/*
 * dmuon_set_workspace -- use a caller-owned device buffer of `bytes` bytes
 * (256-byte aligned) as scratch instead of the library's own allocation.
 * NULL / 0 returns to library-managed scratch.  A call whose plan needs more
 * than `bytes` fails with DMUON_ERR_OOM before any launch.
 */
int dmuon_set_workspace(void* dev_ptr, size_t bytes);

/* Scratch bytes the library would need for dmuon_step / dmuon_step_ex /
 * dmuon_compute_update on this set of shapes (planning only, no allocation,
 * no launch).  dmuon_step_host_io needs more (staging slots and a second
 * compute region); with a caller workspace too small for the second region
 * it runs its chunks on one stream. */
int dmuon_workspace_size(const int64_t* shapes, int count, int param_dtype, size_t* bytes);

/*
 * Kernel timing for benchmarks.  While enabled, the library records CUDA
 * events on the stream it launches on: the Newton-Schulz products of one
 * chunk of a shape group are bracketed as one chain (one pair of events
 * around all of them, none between two of its kernels, so short launches are
 * not stretched by the timing itself); every other launch gets its own pair.
 * dmuon_timing_get synchronises those events and returns, for kernel class
 * `kind` (0 = tensor-core GEMM, 1 = momentum, 2 = SIMT GEMM, 3 = other,
 * 4 = the tensor-core GEMM chains of the CTA-pair kernel alone, a subset of
 * 0), the number of launches, their summed device time in ms, the
 * algorithmic FLOPs (GEMM: 2*M*N*K*batch over the computed tiles) and
 * algorithmic bytes (elementwise kernels).
 */
void dmuon_timing_enable(int enable);
void dmuon_timing_reset(void);
int dmuon_timing_get(int kind, int64_t* launches, double* ms, double* flops, double* bytes);

/*
 * dmuon_adamw_step -- one AdamW step for the parameters that are not
 * matrices.  "DeepSpeed 現已支援 Muon Optimizer" (setupai.cc), section
 * 技術深入: Muon trains the matrix parameters (2-D weights, and convolution
 * filters once flattened) while AdamW trains the rest, such as embeddings,
 * biases and the final classification layer.  The pages give no AdamW
 * formula; this is the published algorithm with decoupled weight decay and
 * bias correction, per element, in fp32:
 *   m = beta1 m + (1 - beta1) g,   v = beta2 v + (1 - beta2) g^2
 *   p = (1 - lr wd) p - lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps)
 * with one rounding of p to its dtype.  All tensors run in one launch.
 *   params[i]      device, numels[i] elements, dtype `dtype` (DMUON_BF16 or
 *                  DMUON_F32), updated in place.
 *   grads[i]       device, same dtype and size, read only.
 *   exp_avg[i], exp_avg_sq[i]
 *                  device fp32 moment buffers (start at zero), in place.
 *   numels[i]      element count (>= 0; 0 skips the tensor).  Any layout:
 *                  the four buffers of a tensor are walked as flat arrays.
 *   step           1 for the first step, then 2, 3, ... (bias correction).
 * The pointer arrays are host memory, read during the call.  Asynchronous
 * on `stream`.  Errors (before any launch, nothing modified):
 * DMUON_ERR_INVALID for a null pointer, numel < 0, step < 1, a non-finite
 * hyperparameter, beta outside [0, 1) or eps < 0; DMUON_ERR_DTYPE for
 * another dtype; DMUON_ERR_OOM if the device tables cannot be allocated.
 * 16-byte aligned buffers take a 4-element vector path; others are handled
 * element by element.
 */
int dmuon_adamw_step(void* const* params, const void* const* grads, float* const* exp_avg,
                     float* const* exp_avg_sq, const int64_t* numels, int count, float lr,
                     float beta1, float beta2, float eps, float wd, int64_t step, int dtype,
                     void* stream);

/*
 * dmuon_selftest_wait -- checks the device-side failure path: launches a
 * one-block kernel whose mbarrier wait nothing completes, with a limit of
 * limit_ms (1..2000).  The kernel gives up, records the timeout in the
 * host-visible error word and returns; the call synchronises `stream` and
 * returns DMUON_ERR_DEVICE_TIMEOUT when that path works (DMUON_OK would mean
 * the wait did not time out).  The context stays usable afterwards.
 */
int dmuon_selftest_wait(int limit_ms, void* stream);

/*
 * dmuon_debug_groups -- the shape groups a step forms from `shapes` (count x 2
 * int64, rows and cols per matrix): host logic only (no device work, no GPU
 * needed), for tests of the grouping (DMuon release article, section 2:
 * matrices are grouped by shape to feed the GPU).  Matrices whose iterate is m x n
 * (m = min, n = max of rows and cols) form one group, in order of first
 * appearance.  For group g, out[6g .. 6g+5] = (m, n, matrices, matrices
 * stored n x m, chunk, iterate in fp32 ? 1 : 0) for up to `cap` groups;
 * `chunk` is the matrices per chain of launches (scratch within the
 * workspace budget; with grads_host != 0, as for dmuon_step_host_io, also
 * about DMUON_IO_CHUNK_MB of gradients).  If `members` is not NULL it
 * receives the `count` matrix indices group by group, those stored m x n
 * first.  Returns the number of groups; DMUON_ERR_INVALID for a bad shape or
 * argument, DMUON_ERR_DTYPE for a bad param_dtype.
 */
int dmuon_debug_groups(const int64_t* shapes, int count, int param_dtype, int grads_host, int64_t* out, int cap,
                       int* members);

/*
 * dmuon_debug_io_order -- the order in which a step issues its chunks, for a
 * description of its shape groups: host logic only (no device work, no GPU
 * needed), for tests of the scheduler (DMuon release article, section 3:
 * work is ordered by each shape group's measured cost).  Group g (listed in issue order, i.e.
 * by descending measured cost) has counts[g] matrices in chunks of
 * chunks[g], a measured chunk cost cost_ms[g] (ms), bytes[g] bytes per matrix
 * over the host link (the larger direction) and sm_copy[g] != 0 when its
 * host copies run through the copy kernel.  cached != 0 describes a
 * dmuon_step_host_io call with every plan cached (chunks merged across
 * groups when one is compute-bound and another copy-bound at a nominal
 * 50 GB/s, the first and last chunks' quarters split off); cached = 0 any
 * other call (group by group).  Writes up to `cap` pieces as (group, first
 * matrix, matrices) int triples into `out` and returns the number of pieces;
 * DMUON_ERR_INVALID on bad arguments.  The host arrays are the caller's.
 */
int dmuon_debug_io_order(const int* counts, const int* chunks, const double* cost_ms, const double* bytes,
                         const int* sm_copy, int ngroups, int cached, int* out, int cap);

/* Number of kernels the library launched since load (all kinds). */
int64_t dmuon_launch_count(void);

/* Thread-local message of the last error ("" if none). */
const char* dmuon_last_error(void);

/* DMUON_VERSION of the loaded library. */
int dmuon_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DMUON_H */
