// internal.h -- launchers shared by the library's host code (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace dmuon {

// Batched GEMM on the tensor cores:  D[l] = epi(A[l] * op(B[l]))
//   A  bf16, M x K, K contiguous (row stride lda, batch stride sa, elements)
//   B  bf16, b_kmajor ? N x K (K contiguous) : K x N (N contiguous)
struct TcGemm {
  const void* A;
  long long lda, sa;
  const void* B;
  long long ldb, sb;
  bool b_kmajor;
  int M, N, K, batch;
  int tile;  // 128 / 256: one CTA, 128 x tile output tile; 512: CTA pair, 256 x 256
  bool sym;  // M == N and the result is symmetric: upper-triangle tiles only, mirrored
  Epilogue epi;
  // CTA pair only (tile 512): symmetric matrices kept as their 256 x 256 blocks
  // on and above the diagonal.  1: A (M x K, M == K) is one; 2: B as stored
  // (K x N, K == N, MN-major) is one; 4: the symmetric result is stored that
  // way (no mirrored copy).  Ignored for other tiles.
  int upper = 0;
};

// Same contract in fp32 on the CUDA cores (fp32 path; any leading dims).
struct SimtGemm {
  const float* A;
  long long lda, sa;
  const float* B;
  long long ldb, sb;
  bool b_kmajor;
  int M, N, K, batch;
  Epilogue epi;
};

// Kernel classes for timing (dmuon_timing_get).
// KIND_TC_GEMM_PAIR is a view for dmuon_timing_get: the KIND_TC_GEMM
// launches of the CTA-pair kernel alone.
enum KernelKind { KIND_TC_GEMM = 0, KIND_EW = 1, KIND_SIMT_GEMM = 2, KIND_OTHER = 3, KIND_TC_GEMM_PAIR = 4 };

cudaError_t launch_tc_gemm(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms);
// 3-D bf16 tensor map {inner, outer, batch} with a 128-byte swizzle and
// zero fill outside the extents (row stride ld, batch stride bstride, in
// elements; box box_inner x box_outer x 1).
bool tensor_map_bf16(CUtensorMap* m, const void* base, long long inner, long long outer, int batch, long long ld,
                     long long bstride, int box_inner, int box_outer);
// Output tiles a launch of this shape processes (symmetric skipping included).
long long tc_gemm_tiles(int M, int N, int batch, int tile, bool sym);
cudaError_t launch_simt_gemm(const SimtGemm& g, cudaStream_t s);

// Momentum + Nesterov + per-matrix sum of squares (partials), writing the
// wide-orientation iterate X (bf16 or fp32) for `cnt` same-shape matrices.
struct MomentumArgs {
  const void* const* G;  // device table of cnt pointers
  void* const* B;        // device table of cnt pointers (fp32, updated in place)
  void* X;               // [cnt][m][ldx] wide orientation
  long long ldx;
  int x_f32, g_f32;
  int rows, cols;        // stored shape
  int transposed;        // rows > cols
  int cnt;
  float mu;
  int nesterov;
  float* partials;       // [cnt][nblk]
  int nblk;              // partial slots per matrix
  int aligned;           // every G/B base 16-byte aligned (vector path allowed)
};
cudaError_t launch_momentum(const MomentumArgs& a, cudaStream_t s);
// Number of partial slots launch_momentum uses for this shape.
int momentum_partials(int rows, int cols);

// s[l] = 1 / (sqrt(sum partials[l][:]) + eps),  s2[l] = s[l]^2.
cudaError_t launch_norm_finalize(const float* partials, int nblk, int cnt, float eps, float* s, float* s2,
                                 cudaStream_t st);

// O = s[l] * X (zero Newton-Schulz steps) through the epilogue (apply / out).
cudaError_t launch_scale_epilogue(const void* X, long long ldx, int x_f32, int m, int n, int cnt,
                                  const float* s, const Epilogue& epi, cudaStream_t st);

// Resident Newton-Schulz for small matrices (m <= 128, n <= 512), direct form,
// one CTA per block of up to 8 stacked matrices; ends with `fin`.
bool ns_small_supported(int m, int n);
int ns_small_group(int m);
cudaError_t launch_ns_small(const void* X0, long long ldx, const float* s, const float* s2, int cnt, int m, int n,
                            int steps, float a, float b, float c, const Epilogue& fin, cudaStream_t st, int* err);

// fp32 Newton-Schulz, direct form, every step of `cnt` same-shape matrices in
// one cooperative launch (one CTA per SM, grid barrier between products);
// ends with `fin`.  X0/Xp/Xq: [cnt][m][ldx], A/P: [cnt][m][ldm] scratch; sync:
// three words of scratch.
struct NsF32 {
  const float* X0;
  float* Xp;
  float* Xq;
  float* A;
  float* P;
  long long ldx, ldm, sx, sq;  // row strides and per-matrix strides (elements)
  const float* s;
  const float* s2;
  int cnt, m, n, steps;
  float a, b, c;
  Epilogue fin;
  unsigned* sync;
};
bool ns_f32_supported(int m, int n);
cudaError_t launch_ns_f32(const NsF32& g, cudaStream_t st, int* err, int num_sms);

// Resident Newton-Schulz for medium bf16 matrices (128 < m <= 256, or m <= 128
// with 512 < n; n <= 1024), Gram form: one CTA pair per matrix, the m x m
// chain (A, P, Q) in shared memory, X0 ([cnt][m][ldx]) read twice, never
// written.  Ends with `fin`.
bool ns_mid_supported(int m, int n);
cudaError_t launch_ns_mid(const void* X0, long long ldx, const float* s, const float* s2, int cnt, int m, int n,
                          int steps, float a, float b, float c, const Epilogue& fin, cudaStream_t st, int* err,
                          int num_sms);
double ns_mid_flops(int m, int n, int steps, int cnt);

// AdamW over `count` tensors in one launch (see kernels_ew.cu).  Tables are
// device arrays; chunk_start[t] is the first chunk of tensor t (prefix sums of
// adamw_chunks(numel)), numel[t] its element count (> 0).
struct AdamwArgs {
  void* const* P;           // params, bf16 or fp32 (p_f32), updated in place
  const void* const* G;     // grads, same dtype as P
  float* const* M;          // first moments, fp32, in place
  float* const* V;          // second moments, fp32, in place
  const long long* chunk_start;
  const long long* numel;
  int count;
  int p_f32;
  int aligned;              // every P/G/M/V base 16-byte aligned: 4-element vectors
  float lr, beta1, beta2, eps;
  float omb1, omb2;         // 1 - beta1, 1 - beta2
  float decay;              // 1 - lr * wd
  float bc1, bc2;           // 1 - beta1^t, 1 - beta2^t
};
long long adamw_chunks(long long numel);
cudaError_t launch_adamw(const AdamwArgs& a, long long total_chunks, cudaStream_t st);

// dst[l] <- src[l] for cnt buffers of `bytes` (a multiple of 16, every
// pointer 16-byte aligned; host pointers must be mapped pinned memory).
cudaError_t launch_copy_tables(const void* const* src, void* const* dst, long long bytes, int cnt, int num_sms,
                               cudaStream_t st);

// dst[0..3] <- p0..p3 (device table written by a one-thread kernel).
cudaError_t launch_store_ptrs(void** dst, void* p0, void* p1, void* p2, void* p3, cudaStream_t st);

// One-block kernel whose only mbarrier wait can never complete; it gives up
// after limit_ns and records kErrTimeout in *err.
cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t st);

// Relative Frobenius distance helper for the autotuner's accuracy gate:
// acc[0] += sum (x - y)^2, acc[1] += sum y^2 over cnt matrices m x n (ld).
cudaError_t launch_diff_norms(const void* X, const void* Y, long long ld, int m, int n, int cnt, int is_f32,
                              double* acc, cudaStream_t st);

}  // namespace dmuon
