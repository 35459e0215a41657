// kernels_ew.cu -- the HBM-bound elementwise stages of the Muon step.
//
// launch_momentum: one pass over G and B per matrix:
//     B' = mu*B + G  (written back, fp32),  U = G + mu*B' (or B'),
//     X  = U (or U^T for tall matrices) written as the bf16/fp32 iterate,
//     per-block partial sums of U^2 for the Frobenius norm.
//   12 bytes per element for bf16 G / fp32 B / bf16 X: read G (2), read and
//   write B (8), write X (2).  128-bit loads/stores on the aligned path; tall
//   matrices go through a 64x64 shared-memory transpose so both the reads and
//   the writes stay coalesced.
// launch_norm_finalize: s = 1/(||U||_F + eps) from the partials, in a fixed
//   order (deterministic).
// launch_scale_epilogue: O = s*X for zero Newton-Schulz steps.
// launch_diff_norms: ||X - Y||^2 and ||Y||^2 for the autotuner's gate.
#include "internal.h"

namespace dmuon {

namespace {

constexpr int EW_THREADS = 256;
constexpr int VEC = 8;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[w] = v;
  __syncthreads();
  float r = 0.f;
  if (threadIdx.x < 32) {
    r = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
  }
  return r;  // valid in thread 0
}

__device__ __forceinline__ void load8(const void* p, long long i, int is_f32, float (&g)[8]) {
  if (is_f32) {
    const float4* q = reinterpret_cast<const float4*>(static_cast<const float*>(p) + i);
    float4 a = __ldcs(q), b = __ldcs(q + 1);
    g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w; g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
  } else {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p) + i));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      float2 f = __bfloat1622float2(h[t]);
      g[2 * t] = f.x;
      g[2 * t + 1] = f.y;
    }
  }
}

// Streaming (evict-first) store of 8 fp32 values: the momentum buffer is not
// read again in this step.
__device__ __forceinline__ void store8_stream_f32(float* p, long long i, const float (&x)[8]) {
  float4* q = reinterpret_cast<float4*>(p + i);
  __stcs(q, make_float4(x[0], x[1], x[2], x[3]));
  __stcs(q + 1, make_float4(x[4], x[5], x[6], x[7]));
}

__device__ __forceinline__ void store8(void* p, long long i, int is_f32, const float (&x)[8]) {
  if (is_f32) {
    float4* q = reinterpret_cast<float4*>(static_cast<float*>(p) + i);
    q[0] = make_float4(x[0], x[1], x[2], x[3]);
    q[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(x[2 * t], x[2 * t + 1]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p) + i) = u;
  }
}

// Wide (rows <= cols) matrices: X has the stored layout (row stride ldx).
__global__ void __launch_bounds__(EW_THREADS) momentum_wide_kernel(const MomentumArgs a, int vec_ok) {
  __shared__ float red[EW_THREADS / 32];
  const int l = blockIdx.y;
  const void* G = a.G[l];
  float* B = static_cast<float*>(a.B[l]);
  const long long xoff = static_cast<long long>(l) * a.rows * a.ldx;
  const long long numel = static_cast<long long>(a.rows) * a.cols;
  const float mu = a.mu;
  float ss = 0.f;
  if (vec_ok) {
    // cols % 8 == 0 and every base 16-byte aligned: ldx == cols.  Two
    // vectors per thread per pass keep twice the bytes in flight.
    const long long nvec = numel / VEC;
    const long long stride = static_cast<long long>(gridDim.x) * EW_THREADS;
    long long v = static_cast<long long>(blockIdx.x) * EW_THREADS + threadIdx.x;
    for (; v + stride < nvec; v += 2 * stride) {
      const long long i0 = v * VEC, i1 = (v + stride) * VEC;
      float g0[8], b0[8], g1[8], b1[8], u[8];
      load8(G, i0, a.g_f32, g0);
      load8(B, i0, 1, b0);
      load8(G, i1, a.g_f32, g1);
      load8(B, i1, 1, b1);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        b0[t] = fmaf(mu, b0[t], g0[t]);
        u[t] = a.nesterov ? fmaf(mu, b0[t], g0[t]) : b0[t];
        ss = fmaf(u[t], u[t], ss);
      }
      store8_stream_f32(B, i0, b0);
      store8(a.X, xoff + i0, a.x_f32, u);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        b1[t] = fmaf(mu, b1[t], g1[t]);
        u[t] = a.nesterov ? fmaf(mu, b1[t], g1[t]) : b1[t];
        ss = fmaf(u[t], u[t], ss);
      }
      store8_stream_f32(B, i1, b1);
      store8(a.X, xoff + i1, a.x_f32, u);
    }
    if (v < nvec) {
      const long long i = v * VEC;
      float g[8], b[8], u[8];
      load8(G, i, a.g_f32, g);
      load8(B, i, 1, b);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        b[t] = fmaf(mu, b[t], g[t]);
        u[t] = a.nesterov ? fmaf(mu, b[t], g[t]) : b[t];
        ss = fmaf(u[t], u[t], ss);
      }
      store8_stream_f32(B, i, b);
      store8(a.X, xoff + i, a.x_f32, u);
    }
  } else {
    for (long long i = static_cast<long long>(blockIdx.x) * EW_THREADS + threadIdx.x; i < numel;
         i += static_cast<long long>(gridDim.x) * EW_THREADS) {
      const long long r = i / a.cols, c = i % a.cols;
      const float g = load_elem(G, i, a.g_f32);
      const float b = fmaf(mu, B[i], g);
      const float u = a.nesterov ? fmaf(mu, b, g) : b;
      B[i] = b;
      ss = fmaf(u, u, ss);
      store_elem(a.X, xoff + r * a.ldx + c, u, a.x_f32);
    }
  }
  const float tot = block_sum(ss, red);
  if (threadIdx.x == 0) a.partials[static_cast<long long>(l) * a.nblk + blockIdx.x] = tot;
}

// Tall (rows > cols) matrices: X = U^T (cols x rows), through a 64x64 tile.
constexpr int TT = 64;
__global__ void __launch_bounds__(EW_THREADS) momentum_tall_kernel(const MomentumArgs a) {
  __shared__ float tile[TT][TT + 1];
  __shared__ float red[EW_THREADS / 32];
  const int l = blockIdx.y;
  const void* G = a.G[l];
  float* B = static_cast<float*>(a.B[l]);
  const long long xoff = static_cast<long long>(l) * a.cols * a.ldx;  // X is cols x rows, row stride ldx
  const int tr = (a.rows + TT - 1) / TT, tc = (a.cols + TT - 1) / TT;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const float mu = a.mu;
  float ss = 0.f;
  for (int t = blockIdx.x; t < tr * tc; t += gridDim.x) {
    const int r0 = (t / tc) * TT, c0 = (t % tc) * TT;
    // read rows r0..r0+63 of the stored matrix, two columns per thread
#pragma unroll
    for (int k = 0; k < TT / 8; ++k) {
      const int rr = ty + 8 * k;
      const int r = r0 + rr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cc = 2 * tx + h;
        const int c = c0 + cc;
        float u = 0.f;
        if (r < a.rows && c < a.cols) {
          const long long i = static_cast<long long>(r) * a.cols + c;
          const float g = load_elem(G, i, a.g_f32);
          const float b = fmaf(mu, B[i], g);
          u = a.nesterov ? fmaf(mu, b, g) : b;
          B[i] = b;
          ss = fmaf(u, u, ss);
        }
        tile[rr][cc] = u;
      }
    }
    __syncthreads();
    // write X rows c0..c0+63 (= stored columns), columns r0..r0+63
#pragma unroll
    for (int k = 0; k < TT / 8; ++k) {
      const int cc = ty + 8 * k;
      const int xr = c0 + cc;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int rr = 2 * tx + h;
        const int xc = r0 + rr;
        if (xr < a.cols && xc < a.rows) store_elem(a.X, xoff + static_cast<long long>(xr) * a.ldx + xc, tile[rr][cc], a.x_f32);
      }
    }
    __syncthreads();
  }
  const float tot = block_sum(ss, red);
  if (threadIdx.x == 0) a.partials[static_cast<long long>(l) * a.nblk + blockIdx.x] = tot;
}

// Tall matrices, vector path (cols % 4 == 0, 16-byte aligned G and B):
// 64 x 128 tiles.  Each warp reads 8 rows of the tile, a lane four
// consecutive columns (one 16-byte load of B, one 8- or 16-byte load of G);
// U goes to shared memory transposed, and each warp then writes 16 rows of
// X (stored columns), eight elements per lane.  The shared tile is [128][64]
// floats with the row index XOR-swizzled by an even key of the column, so
// the transposed writes meet at most two lanes per bank.
constexpr int TVR = 64, TVC = 128;
__device__ __forceinline__ int tv_idx(int c, int r) { return c * TVR + (r ^ (((c >> 2) & 15) << 1)); }

__global__ void __launch_bounds__(EW_THREADS) momentum_tall_vec_kernel(const MomentumArgs a) {
  __shared__ __align__(16) float tile[TVC * TVR];
  __shared__ float red[EW_THREADS / 32];
  const int l = blockIdx.y;
  const void* G = a.G[l];
  float* B = static_cast<float*>(a.B[l]);
  const long long xoff = static_cast<long long>(l) * a.cols * a.ldx;  // X is cols x rows, row stride ldx
  const int tr = (a.rows + TVR - 1) / TVR, tc = (a.cols + TVC - 1) / TVC;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;  // 32 x 8
  const float mu = a.mu;
  float ss = 0.f;
  for (int t = blockIdx.x; t < tr * tc; t += gridDim.x) {
    const int r0 = (t / tc) * TVR, c0 = (t % tc) * TVC;
    const int c = c0 + 4 * lane;  // this lane's four stored columns
#pragma unroll 4
    for (int k = 0; k < TVR / 8; ++k) {
      const int rr = w + 8 * k;
      const int r = r0 + rr;
      float u[4] = {0.f, 0.f, 0.f, 0.f};
      if (r < a.rows && c < a.cols) {  // cols % 4 == 0: the four columns are in range together
        const long long i = static_cast<long long>(r) * a.cols + c;
        float g[4];
        if (a.g_f32) {
          const float4 gv = __ldcs(reinterpret_cast<const float4*>(static_cast<const float*>(G) + i));
          g[0] = gv.x; g[1] = gv.y; g[2] = gv.z; g[3] = gv.w;
        } else {
          const uint2 gv = __ldcs(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(G) + i));
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&gv);
          const float2 g01 = __bfloat1622float2(h[0]), g23 = __bfloat1622float2(h[1]);
          g[0] = g01.x; g[1] = g01.y; g[2] = g23.x; g[3] = g23.y;
        }
        const float4 bv = __ldcs(reinterpret_cast<const float4*>(B + i));
        float b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b[j] = fmaf(mu, b[j], g[j]);
          u[j] = a.nesterov ? fmaf(mu, b[j], g[j]) : b[j];
          ss = fmaf(u[j], u[j], ss);
        }
        __stcs(reinterpret_cast<float4*>(B + i), make_float4(b[0], b[1], b[2], b[3]));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) tile[tv_idx(4 * lane + j, rr)] = u[j];
    }
    __syncthreads();
    // X rows c0..c0+127 (stored columns), columns r0..r0+63: a lane writes
    // eight consecutive elements (16 bytes in bf16), eight lanes per X row,
    // so one warp instruction covers four rows of 128 bytes.  The four rows
    // of an instruction are 4 apart, so their swizzle keys differ and the
    // shared-memory reads meet no more than two lanes per bank.
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int cc = 16 * w + 4 * (lane >> 3) + k, seg = lane & 7;
      const int xr = c0 + cc, xc = r0 + 8 * seg;
      if (xr >= a.cols || xc >= a.rows) continue;
      float v[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float2 t = *reinterpret_cast<const float2*>(&tile[tv_idx(cc, 8 * seg + 2 * p)]);
        v[2 * p] = t.x;
        v[2 * p + 1] = t.y;
      }
      const long long o = xoff + static_cast<long long>(xr) * a.ldx + xc;
      if (xc + 8 <= a.rows) {
        if (a.x_f32) {
          float4* q = reinterpret_cast<float4*>(static_cast<float*>(a.X) + o);
          q[0] = make_float4(v[0], v[1], v[2], v[3]);
          q[1] = make_float4(v[4], v[5], v[6], v[7]);
        } else {
          uint4 u;
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
          for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(v[2 * t], v[2 * t + 1]);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.X) + o) = u;
        }
      } else {
        for (int t = 0; t < 8 && xc + t < a.rows; ++t) store_elem(a.X, o + t, v[t], a.x_f32);
      }
    }
    __syncthreads();
  }
  const float tot = block_sum(ss, red);
  if (threadIdx.x == 0) a.partials[static_cast<long long>(l) * a.nblk + blockIdx.x] = tot;
}

__global__ void norm_finalize_kernel(const float* __restrict__ partials, int nblk, float eps, float* s, float* s2) {
  const int l = blockIdx.x;
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < nblk; i += blockDim.x) acc += static_cast<double>(partials[static_cast<long long>(l) * nblk + i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += red[w];
    const double inv = 1.0 / (sqrt(t) + static_cast<double>(eps));
    s[l] = static_cast<float>(inv);
    s2[l] = static_cast<float>(inv * inv);
  }
}

__global__ void __launch_bounds__(256) scale_epilogue_kernel(const void* X, long long ldx, int x_f32, int m, int n,
                                                             const float* s, const Epilogue epi) {
  const int l = blockIdx.z;
  const int row = blockIdx.y * 8 + (threadIdx.x >> 5);
  const int col = blockIdx.x * 32 + (threadIdx.x & 31);
  if (row >= m) return;
  float v[1];
  v[0] = (col < n) ? s[l] * load_elem(X, static_cast<long long>(l) * m * ldx + static_cast<long long>(row) * ldx + col, x_f32) : 0.f;
  if (col < n) epilogue_row<1>(epi, l, row, col, v, m, n);
}

__global__ void diff_norms_kernel(const void* X, const void* Y, long long ld, int m, int n, int is_f32,
                                  double* acc) {
  const int l = blockIdx.y;
  double d = 0.0, y2 = 0.0;
  const long long numel = static_cast<long long>(m) * n;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < numel;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = i / n, c = i % n;
    const long long o = static_cast<long long>(l) * m * ld + r * ld + c;
    const double x = load_elem(X, o, is_f32), y = load_elem(Y, o, is_f32);
    d += (x - y) * (x - y);
    y2 += y * y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    d += __shfl_xor_sync(0xffffffffu, d, o);
    y2 += __shfl_xor_sync(0xffffffffu, y2, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&acc[0], d);
    atomicAdd(&acc[1], y2);
  }
}

// Waits on an mbarrier that nothing arrives on, with a short limit: the
// bounded-wait machinery of the GEMM kernels, exercised on its own.
__global__ void wait_selftest_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_limit(&bar, 0, &abort, limit_ns) && err)
    *reinterpret_cast<volatile int*>(err) = kErrTimeout;
}

// Writes four pointers, passed by value, into a device table: a pointer
// table built on the device from kernel arguments, with no host buffer that
// must outlive the call.
__global__ void store_ptrs_kernel(void** dst, void* p0, void* p1, void* p2, void* p3) {
  dst[0] = p0;
  dst[1] = p1;
  dst[2] = p2;
  dst[3] = p3;
}

// Copies cnt buffers of `bytes` each, dst[l] <- src[l], through the SMs.
// Either side may be pinned host memory mapped into the device's address
// space: the host I/O pipeline gathers gradients from, and scatters
// parameters to, host memory this way with one launch per chunk instead of
// one copy-engine transfer per matrix.  All pointers 16-byte aligned and
// bytes % 16 == 0 (checked by the host).  Four 16-byte loads in flight per
// thread cover the PCIe round trip; 128-thread blocks without shared memory
// fit beside a persistent GEMM CTA on the same SM.
constexpr int COPY_THREADS = 128;
constexpr int COPY_UNROLL = 4;

__global__ void __launch_bounds__(COPY_THREADS) copy_tables_kernel(const uint4* const* __restrict__ src,
                                                                   uint4* const* __restrict__ dst, long long nvec) {
  const uint4* s = src[blockIdx.y];
  uint4* d = dst[blockIdx.y];
  const long long stride = static_cast<long long>(gridDim.x) * COPY_THREADS * COPY_UNROLL;
  for (long long base = static_cast<long long>(blockIdx.x) * COPY_THREADS * COPY_UNROLL + threadIdx.x; base < nvec;
       base += stride) {
    uint4 v[COPY_UNROLL];
#pragma unroll
    for (int u = 0; u < COPY_UNROLL; ++u) {
      const long long i = base + static_cast<long long>(u) * COPY_THREADS;
      if (i < nvec) v[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < COPY_UNROLL; ++u) {
      const long long i = base + static_cast<long long>(u) * COPY_THREADS;
      if (i < nvec) d[i] = v[u];
    }
  }
}

// AdamW over many tensors in one launch (the non-matrix parameters that
// train beside Muon: biases, norms, embeddings, the output layer).  Block b
// handles chunk b of the concatenated tensors: it finds its tensor by binary
// search in the chunk offsets, then each thread updates 4 consecutive
// elements per pass in fp32 -- m = b1 m + (1-b1) g, v = b2 v + (1-b2) g^2,
// p = (1 - lr wd) p - lr (m / bc1) / (sqrt(v / bc2) + eps) with bc = 1 - b^t
// -- and writes p back with one rounding to its dtype.  22 bytes per bf16
// element (p rw 4, g 2, m rw 8, v rw 8), 32 per fp32 element: HBM-bound.
constexpr int ADAM_THREADS = 256;
constexpr int ADAM_CHUNK = ADAM_THREADS * 4 * 4;  // 4 passes of 4 elements per thread

// Every rounding is explicit (no contraction left to the compiler), so the
// vector and element-by-element paths give the same bits.
__device__ __forceinline__ void adam_elem(float& p, float g, float& m, float& v, const AdamwArgs& a) {
  m = __fmaf_rn(a.beta1, m, __fmul_rn(a.omb1, g));
  v = __fmaf_rn(a.beta2, v, __fmul_rn(__fmul_rn(a.omb2, g), g));
  const float denom = __fadd_rn(__fsqrt_rn(__fdiv_rn(v, a.bc2)), a.eps);
  p = __fmaf_rn(p, a.decay, -__fmul_rn(a.lr, __fdiv_rn(__fdiv_rn(m, a.bc1), denom)));
}

__global__ void __launch_bounds__(ADAM_THREADS) adamw_kernel(const AdamwArgs a) {
  const long long chunk = blockIdx.x;
  int lo = 0, hi = a.count - 1;  // last tensor whose first chunk <= chunk
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.chunk_start[mid] <= chunk) lo = mid;
    else hi = mid - 1;
  }
  const int t = lo;
  const long long n = a.numel[t];
  const long long base = (chunk - a.chunk_start[t]) * ADAM_CHUNK;
  float* M = a.M[t];
  float* V = a.V[t];
  const bool vec = a.aligned != 0;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const long long e = base + (static_cast<long long>(pass) * ADAM_THREADS + threadIdx.x) * 4;
    if (e >= n) break;
    if (vec && e + 4 <= n) {
      float4 m4 = *reinterpret_cast<const float4*>(M + e);
      float4 v4 = *reinterpret_cast<const float4*>(V + e);
      float pv[4], gv[4];
      if (a.p_f32) {
        const float4 p4 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.P[t]) + e);
        const float4 g4 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.G[t]) + e);
        pv[0] = p4.x; pv[1] = p4.y; pv[2] = p4.z; pv[3] = p4.w;
        gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
      } else {
        const uint2 pu = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.P[t]) + e);
        const uint2 gu = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(a.G[t]) + e);
        const __nv_bfloat162* ph = reinterpret_cast<const __nv_bfloat162*>(&pu);
        const __nv_bfloat162* gh = reinterpret_cast<const __nv_bfloat162*>(&gu);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float2 pf = __bfloat1622float2(ph[q]), gf = __bfloat1622float2(gh[q]);
          pv[2 * q] = pf.x; pv[2 * q + 1] = pf.y;
          gv[2 * q] = gf.x; gv[2 * q + 1] = gf.y;
        }
      }
      adam_elem(pv[0], gv[0], m4.x, v4.x, a);
      adam_elem(pv[1], gv[1], m4.y, v4.y, a);
      adam_elem(pv[2], gv[2], m4.z, v4.z, a);
      adam_elem(pv[3], gv[3], m4.w, v4.w, a);
      *reinterpret_cast<float4*>(M + e) = m4;
      *reinterpret_cast<float4*>(V + e) = v4;
      if (a.p_f32) {
        *reinterpret_cast<float4*>(static_cast<float*>(a.P[t]) + e) = make_float4(pv[0], pv[1], pv[2], pv[3]);
      } else {
        uint2 pu;
        __nv_bfloat162* ph = reinterpret_cast<__nv_bfloat162*>(&pu);
        ph[0] = __floats2bfloat162_rn(pv[0], pv[1]);
        ph[1] = __floats2bfloat162_rn(pv[2], pv[3]);
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.P[t]) + e) = pu;
      }
    } else {
      for (int k = 0; k < 4 && e + k < n; ++k) {
        const long long i = e + k;
        float pv, gv;
        if (a.p_f32) {
          pv = static_cast<const float*>(a.P[t])[i];
          gv = static_cast<const float*>(a.G[t])[i];
        } else {
          pv = __bfloat162float(static_cast<const __nv_bfloat16*>(a.P[t])[i]);
          gv = __bfloat162float(static_cast<const __nv_bfloat16*>(a.G[t])[i]);
        }
        float m = M[i], v = V[i];
        adam_elem(pv, gv, m, v, a);
        M[i] = m;
        V[i] = v;
        if (a.p_f32) static_cast<float*>(a.P[t])[i] = pv;
        else static_cast<__nv_bfloat16*>(a.P[t])[i] = __float2bfloat16_rn(pv);
      }
    }
  }
}

}  // namespace

long long adamw_chunks(long long numel) { return (numel + ADAM_CHUNK - 1) / ADAM_CHUNK; }

cudaError_t launch_adamw(const AdamwArgs& a, long long total_chunks, cudaStream_t st) {
  if (a.count <= 0 || total_chunks <= 0) return cudaSuccess;
  if (total_chunks > 0x7fffffffLL) return cudaErrorInvalidValue;
  adamw_kernel<<<static_cast<unsigned>(total_chunks), ADAM_THREADS, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_copy_tables(const void* const* src, void* const* dst, long long bytes, int cnt, int num_sms,
                               cudaStream_t st) {
  if (cnt <= 0 || bytes <= 0) return cudaSuccess;
  if (cnt > 65535 || bytes % 16 != 0) return cudaErrorInvalidValue;
  const long long nvec = bytes / 16;
  const long long per_block = static_cast<long long>(COPY_THREADS) * COPY_UNROLL;
  long long bx = (static_cast<long long>(num_sms) * 2 + cnt - 1) / cnt;  // about two blocks per SM in all
  const long long need = (nvec + per_block - 1) / per_block;
  if (bx > need) bx = need;
  if (bx < 1) bx = 1;
  dim3 grid(static_cast<unsigned>(bx), cnt);
  copy_tables_kernel<<<grid, COPY_THREADS, 0, st>>>(reinterpret_cast<const uint4* const*>(src),
                                                    reinterpret_cast<uint4* const*>(dst), nvec);
  return cudaGetLastError();
}

cudaError_t launch_store_ptrs(void** dst, void* p0, void* p1, void* p2, void* p3, cudaStream_t st) {
  store_ptrs_kernel<<<1, 1, 0, st>>>(dst, p0, p1, p2, p3);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int* err, unsigned long long limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

int momentum_partials(int rows, int cols) {
  const long long numel = static_cast<long long>(rows) * cols;
  // Many short blocks: each thread makes one pass of two 8-element vectors
  // (wide) or the block takes one 64 x 64 tile (tall).  Against one resident
  // wave of long grid-stride blocks this took the kernel from 0.81 to 0.89
  // of the measured HBM bandwidth on 64 x 1024^2 (the hardware scheduler
  // balances short blocks over the SMs and memory partitions).
  long long nb;
  if (rows > cols)
    nb = static_cast<long long>((rows + TT - 1) / TT) * ((cols + TT - 1) / TT);
  else
    nb = (numel + EW_THREADS * VEC * 2 - 1) / (EW_THREADS * VEC * 2);
  if (nb < 1) nb = 1;
  if (nb > 4096) nb = 4096;
  return static_cast<int>(nb);
}

cudaError_t launch_momentum(const MomentumArgs& a, cudaStream_t s) {
  if (a.cnt <= 0) return cudaSuccess;
  if (a.cnt > 65535) return cudaErrorInvalidValue;
  dim3 grid(a.nblk, a.cnt);
  if (a.transposed) {
    // the vector path reads four columns with one load: cols % 4 == 0 and
    // 16-byte aligned G/B bases (a.aligned); its eight-element X stores
    // need 16-byte aligned rows (ldx % 8 == 0, X base 16-byte aligned)
    if (a.cols % 4 == 0 && a.aligned && (a.ldx & 7) == 0 && (reinterpret_cast<uintptr_t>(a.X) & 15) == 0)
      momentum_tall_vec_kernel<<<grid, EW_THREADS, 0, s>>>(a);
    else
      momentum_tall_kernel<<<grid, EW_THREADS, 0, s>>>(a);
  } else {
    // The vector path needs cols % 8 == 0 (then ldx == cols) and 16-byte
    // aligned G/B bases (checked by the host: a.aligned).
    const int vec_ok = (a.cols % VEC == 0) && (a.ldx == a.cols) && a.aligned ? 1 : 0;
    momentum_wide_kernel<<<grid, EW_THREADS, 0, s>>>(a, vec_ok);
  }
  return cudaGetLastError();
}

cudaError_t launch_norm_finalize(const float* partials, int nblk, int cnt, float eps, float* s, float* s2,
                                 cudaStream_t st) {
  if (cnt <= 0) return cudaSuccess;
  norm_finalize_kernel<<<cnt, 256, 0, st>>>(partials, nblk, eps, s, s2);
  return cudaGetLastError();
}

cudaError_t launch_scale_epilogue(const void* X, long long ldx, int x_f32, int m, int n, int cnt, const float* s,
                                  const Epilogue& epi, cudaStream_t st) {
  if (cnt <= 0) return cudaSuccess;
  if (cnt > 65535 || (m + 7) / 8 > 65535) return cudaErrorInvalidValue;
  dim3 grid((n + 31) / 32, (m + 7) / 8, cnt);
  scale_epilogue_kernel<<<grid, 256, 0, st>>>(X, ldx, x_f32, m, n, s, epi);
  return cudaGetLastError();
}

cudaError_t launch_diff_norms(const void* X, const void* Y, long long ld, int m, int n, int cnt, int is_f32,
                              double* acc, cudaStream_t st) {
  if (cnt <= 0) return cudaSuccess;
  dim3 grid(64, cnt);
  diff_norms_kernel<<<grid, 256, 0, st>>>(X, Y, ld, m, n, is_f32, acc);
  return cudaGetLastError();
}

}  // namespace dmuon
