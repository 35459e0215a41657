// gemm_simt.cu -- batched fp32 GEMM on the CUDA cores for the fp32 Muon path.
//
// The bf16 tensor-core path holds the update to about 1e-2 relative error;
// fp32 weights are held to 1e-4, which bf16 (or tf32) operands cannot reach.
// This kernel keeps the whole Newton-Schulz iteration in fp32 FFMA with the
// same epilogue contract as the tensor-core GEMM.  32x32 output tile per
// block of 256 threads (2x2 outputs each), 32-deep k slices staged in shared
// memory: the fp32 workloads are single matrices of a few hundred rows, so
// small tiles are what spreads a product over the SMs; when even those leave
// SMs idle, K is split over a cluster of 2-8 CTAs (simt_gemm_splitk_kernel).
// Each slice's loads go to registers one slice ahead, so they are in flight
// while the previous slice is multiplied.
// Consecutive products are launched with programmatic dependent launch: each
// kernel lets the next one launch as soon as all its own CTAs are running,
// and waits for the previous one's results before reading anything, so a
// launch's start-up overlaps the previous product's tail.
#include "internal.h"

namespace dmuon {

namespace {

constexpr int TM = 32, TN = 32, TK = 32;

// Loads the A tile (32 rows x 32 k, k contiguous: coalesced along k) and the
// B tile (32 k x 32 columns) of the slice starting at k0 into registers,
// zero outside the matrix and at or beyond k_end.
__device__ __forceinline__ void fetch_tiles(const float* Ab, long long lda, const float* Bb, long long ldb, int b_kmajor,
                                            int M, int N, int k_end, int m0, int n0, int k0, int tid,
                                            float (&ra)[TM * TK / 256], float (&rb)[TN * TK / 256]) {
#pragma unroll
  for (int u = 0; u < TM * TK / 256; ++u) {
    const int i = tid + 256 * u;
    const int r = i / TK, k = i % TK;
    const int gr = m0 + r, gk = k0 + k;
    ra[u] = (gr < M && gk < k_end) ? Ab[static_cast<long long>(gr) * lda + gk] : 0.f;
  }
#pragma unroll
  for (int u = 0; u < TN * TK / 256; ++u) {
    const int i = tid + 256 * u;
    const int c = b_kmajor ? i / TK : i % TN, k = b_kmajor ? i % TK : i / TN;
    const int gc = n0 + c, gk = k0 + k;
    rb[u] = (gc < N && gk < k_end)
                ? (b_kmajor ? Bb[static_cast<long long>(gc) * ldb + gk] : Bb[static_cast<long long>(gk) * ldb + gc])
                : 0.f;
  }
}

__device__ __forceinline__ void store_tiles(float (&As)[TK][TM + 1], float (&Bs)[TK][TN + 1], int b_kmajor, int tid,
                                            const float (&ra)[TM * TK / 256], const float (&rb)[TN * TK / 256]) {
#pragma unroll
  for (int u = 0; u < TM * TK / 256; ++u) {
    const int i = tid + 256 * u;
    As[i % TK][i / TK] = ra[u];
  }
#pragma unroll
  for (int u = 0; u < TN * TK / 256; ++u) {
    const int i = tid + 256 * u;
    const int c = b_kmajor ? i / TK : i % TN, k = b_kmajor ? i % TK : i / TN;
    Bs[k][c] = rb[u];
  }
}

// acc += this thread's 2 x 2 outputs over one staged slice.
__device__ __forceinline__ void mult_slice(const float (&As)[TK][TM + 1], const float (&Bs)[TK][TN + 1], int tx, int ty,
                                           float (&acc)[2][2]) {
#pragma unroll 8
  for (int k = 0; k < TK; ++k) {
    const float a0 = As[k][ty * 2], a1 = As[k][ty * 2 + 1];
    const float b0 = Bs[k][tx * 2], b1 = Bs[k][tx * 2 + 1];
    acc[0][0] = fmaf(a0, b0, acc[0][0]);
    acc[0][1] = fmaf(a0, b1, acc[0][1]);
    acc[1][0] = fmaf(a1, b0, acc[1][0]);
    acc[1][1] = fmaf(a1, b1, acc[1][1]);
  }
}

__global__ void __launch_bounds__(256) simt_gemm_kernel(const float* __restrict__ A, long long lda, long long sa,
                                                        const float* __restrict__ B, long long ldb, long long sb,
                                                        int b_kmajor, int M, int N, int K, const Epilogue epi) {
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  grid_dep_wait();    // the previous product's results are complete and visible
  grid_dep_launch();  // the next product may start launching
  const int l = blockIdx.z;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 2 x 2 outputs each
  const float* Ab = A + static_cast<long long>(l) * sa;
  const float* Bb = B + static_cast<long long>(l) * sb;
  float acc[2][2] = {};
  float ra[TM * TK / 256], rb[TN * TK / 256];
  fetch_tiles(Ab, lda, Bb, ldb, b_kmajor, M, N, K, m0, n0, 0, tid, ra, rb);
  for (int k0 = 0; k0 < K; k0 += TK) {
    store_tiles(As, Bs, b_kmajor, tid, ra, rb);
    __syncthreads();
    // the next slice's loads are in flight while this one is multiplied
    if (k0 + TK < K) fetch_tiles(Ab, lda, Bb, ldb, b_kmajor, M, N, K, m0, n0, k0 + TK, tid, ra, rb);
    mult_slice(As, Bs, tx, ty, acc);
    __syncthreads();
  }
  const int col = n0 + tx * 2;
  if (col >= N) return;
#pragma unroll
  for (int i = 0; i < 2; ++i) epilogue_row<2>(epi, l, m0 + ty * 2 + i, col, acc[i], M, N);
}

// Split-K over a thread-block cluster.  The fp32 products are small (a few
// hundred rows), so 32 x 32 output tiles give fewer blocks than SMs; here a
// cluster of S CTAs shares one output tile, CTA r accumulating the r-th
// slice of K with the loop above.  The partial tiles are summed through
// distributed shared memory in a fixed CTA order (so the result does not
// depend on timing), and CTA r applies the epilogue to rows r*32/S ..
// (r+1)*32/S - 1 of the tile.
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__global__ void __launch_bounds__(256) simt_gemm_splitk_kernel(const float* __restrict__ A, long long lda, long long sa,
                                                               const float* __restrict__ B, long long ldb, long long sb,
                                                               int b_kmajor, int M, int N, int K, int S, int ks,
                                                               const Epilogue epi) {
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN + 1];
  __shared__ float part[TM][TN];
  grid_dep_wait();
  grid_dep_launch();
  const int l = blockIdx.z;
  const int r = static_cast<int>(cluster_rank());  // K slice of this CTA
  const int m0 = blockIdx.y * TM, n0 = (blockIdx.x / S) * TN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const float* Ab = A + static_cast<long long>(l) * sa;
  const float* Bb = B + static_cast<long long>(l) * sb;
  const int k_lo = r * ks, k_hi = min(K, k_lo + ks);
  float acc[2][2] = {};
  float ra[TM * TK / 256], rb[TN * TK / 256];
  if (k_lo < k_hi) fetch_tiles(Ab, lda, Bb, ldb, b_kmajor, M, N, k_hi, m0, n0, k_lo, tid, ra, rb);
  for (int k0 = k_lo; k0 < k_hi; k0 += TK) {
    store_tiles(As, Bs, b_kmajor, tid, ra, rb);
    __syncthreads();
    if (k0 + TK < k_hi) fetch_tiles(Ab, lda, Bb, ldb, b_kmajor, M, N, k_hi, m0, n0, k0 + TK, tid, ra, rb);
    mult_slice(As, Bs, tx, ty, acc);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) part[ty * 2 + i][tx * 2 + j] = acc[i][j];
  cluster_sync();  // every slice's partial tile is in its CTA's shared memory
  const int rows = TM / S;  // rows of the tile this CTA finishes
  const uint32_t base = smem_u32(&part[0][0]);
  for (int e = tid; e < rows * TN; e += 256) {
    const int rr = r * rows + e / TN, c = e % TN;
    const uint32_t off = static_cast<uint32_t>((rr * TN + c) * sizeof(float));
    float pq[8];  // every slice's partial in flight at once, then summed in slice order
#pragma unroll
    for (int q = 0; q < 8; ++q) pq[q] = q < S ? ld_dsmem_f32(mapa_shared(base + off, static_cast<uint32_t>(q))) : 0.f;
    float v[1] = {0.f};
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < S) v[0] += pq[q];
    if (n0 + c < N) epilogue_row<1>(epi, l, m0 + rr, n0 + c, v, M, N);
  }
  cluster_sync();  // no CTA leaves while another still reads its partial tile
}

}  // namespace

cudaError_t launch_simt_gemm(const SimtGemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0) return cudaSuccess;
  if (g.batch > 65535) return cudaErrorInvalidValue;
  const int tiles_n = (g.N + TN - 1) / TN, tiles_m = (g.M + TM - 1) / TM;
  const long long tiles = static_cast<long long>(tiles_n) * tiles_m * g.batch;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  // split K over a cluster until the grid covers two CTAs per SM (each CTA
  // holds 12.5 KB of shared memory and 64 registers per thread, so four
  // fit), keeping at least one TK-deep slice per CTA
  int S = 1;
  while (S < 8 && tiles * S < 2 * sms && g.K >= 2 * S * TK) S *= 2;
  if (S > 1) {
    const int ks = ((g.K + S * TK - 1) / (S * TK)) * TK;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(tiles_n * S), static_cast<unsigned>(tiles_m), static_cast<unsigned>(g.batch));
    cfg.blockDim = dim3(256);
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, simt_gemm_splitk_kernel, g.A, g.lda, g.sa, g.B, g.ldb, g.sb, g.b_kmajor ? 1 : 0,
                              g.M, g.N, g.K, S, ks, g.epi);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles_n), static_cast<unsigned>(tiles_m), static_cast<unsigned>(g.batch));
  cfg.blockDim = dim3(256);
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, simt_gemm_kernel, g.A, g.lda, g.sa, g.B, g.ldb, g.sb, g.b_kmajor ? 1 : 0, g.M, g.N,
                            g.K, g.epi);
}

}  // namespace dmuon
