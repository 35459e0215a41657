// gemm_simt.cu -- batched fp32 GEMM on the CUDA cores for the fp32 Muon path.
//
// The bf16 tensor-core path holds the update to about 1e-2 relative error;
// fp32 weights are held to 1e-4, which bf16 (or tf32) operands cannot reach.
// This kernel keeps the whole Newton-Schulz iteration in fp32 FFMA with the
// same epilogue contract as the tensor-core GEMM.  64x64 output tile per
// block, 16-deep k slices staged in shared memory, 4x4 outputs per thread.
#include "internal.h"

namespace dmuon {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A, long long lda, long long sa,
                                                        const float* __restrict__ B, long long ldb, long long sb,
                                                        int b_kmajor, int M, int N, int K, const Epilogue epi) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN + 4];
  const int l = blockIdx.z;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const float* Ab = A + static_cast<long long>(l) * sa;
  const float* Bb = B + static_cast<long long>(l) * sb;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    // A tile: 64 rows x 16 k (k contiguous in memory)
    for (int i = tid; i < TM * TK; i += 256) {
      const int r = i / TK, k = i % TK;
      const int gr = m0 + r, gk = k0 + k;
      As[k][r] = (gr < M && gk < K) ? Ab[static_cast<long long>(gr) * lda + gk] : 0.f;
    }
    // B tile: 16 k x 64 cols
    for (int i = tid; i < TN * TK; i += 256) {
      int c, k;
      if (b_kmajor) {
        c = i / TK;
        k = i % TK;
      } else {
        k = i / TN;
        c = i % TN;
      }
      const int gc = n0 + c, gk = k0 + k;
      float v = 0.f;
      if (gc < N && gk < K)
        v = b_kmajor ? Bb[static_cast<long long>(gc) * ldb + gk] : Bb[static_cast<long long>(gk) * ldb + gc];
      Bs[k][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const int col = n0 + tx * 4;
  if (col >= N) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) epilogue_row<4>(epi, l, m0 + ty * 4 + i, col, acc[i], M, N);
}

}  // namespace

cudaError_t launch_simt_gemm(const SimtGemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0) return cudaSuccess;
  if (g.batch > 65535) return cudaErrorInvalidValue;
  dim3 grid((g.N + TN - 1) / TN, (g.M + TM - 1) / TM, g.batch);
  simt_gemm_kernel<<<grid, 256, 0, s>>>(g.A, g.lda, g.sa, g.B, g.ldb, g.sb, g.b_kmajor ? 1 : 0, g.M, g.N, g.K,
                                        g.epi);
  return cudaGetLastError();
}

}  // namespace dmuon
