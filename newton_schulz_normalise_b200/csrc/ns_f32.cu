// ns_f32.cu -- the fp32 Newton-Schulz iteration in one cooperative launch.
//
// The fp32 path must hold the update to 1e-4 of the fp64 result, which bf16
// or tf32 tensor-core operands cannot, so it runs on the CUDA cores (FFMA).
// Its matrices are small (the fp32 workload is one 256 x 512 weight): as
// separate launches, each of the 3K products of the direct form pays a
// launch and a drain that cost more than its arithmetic.  Here one
// cooperative launch, one CTA per SM, runs every product of every step:
//   A  = X X^T              (s^2 on the first step)   symmetric: upper tiles, mirrored
//   P  = c A A + b A + a I                             symmetric: upper tiles, mirrored
//   X' = P X                (s on the first step; the last step ends in the
//                            caller's epilogue: parameter write or fp32 O)
// with a grid-wide barrier between products.  X, A and P stay in the
// scratch, where the 126 MB L2 holds them between products.  Each CTA takes
// 16 x 16 output tiles in turn; a tile's operand rows are staged in shared
// memory whole (up to 1024 deep at a time) so their loads are in flight
// together, and each thread sums its output over k with four independent
// accumulators added in a fixed order (the result does not depend on timing).
// The barrier's waits are bounded (2 s): on expiry the kernel records
// kErrTimeout in the error word and every CTA leaves.
#include <algorithm>
#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int FT = 16;           // output tile rows / columns
constexpr int FKC = 1024;        // k depth staged per chunk
constexpr int F_THREADS = 256;   // one output per thread
constexpr int F_LD = FKC + 4;    // padded row of a staged slab (floats): 16-byte aligned rows, rows 4 banks apart

struct F32Args {
  const float* X0;      // [cnt][m][ldx] unnormalised iterate (wide orientation)
  float* Xb[2];         // ping-pong iterates, same layout
  float* A;             // [cnt][m][ldm]
  float* P;             // [cnt][m][ldm]
  long long ldx, ldm, sx, sq;
  const float* s;       // 1 / (||U|| + eps) per matrix
  const float* s2;
  int cnt, m, n, steps;
  float a, b, c;
  Epilogue fin;         // the last step's epilogue (alpha 1: the scale is applied here)
  unsigned* sync;       // [0] arrivals, [1] generation, [2] abort (zeroed before the launch)
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier of the cooperative launch; false once any CTA aborted
// (its own wait timed out, or another CTA's did).
__device__ bool grid_barrier(unsigned* sync, int* err) {
  __shared__ int ok_s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned g0 = ld_acquire(&sync[1]);
    __threadfence();  // this CTA's results before its arrival
    if (atomicAdd(&sync[0], 1u) == gridDim.x - 1) {
      atomicExch(&sync[0], 0u);
      __threadfence();
      st_release(&sync[1], g0 + 1);
    } else {
      const unsigned long long t0 = global_ns();
      while (ld_acquire(&sync[1]) == g0) {
        if (ld_acquire(&sync[2])) {
          ok = 0;
          break;
        }
        if (global_ns() - t0 > kWaitLimitNs) {
          atomicExch(&sync[2], 1u);
          if (err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
    ok_s = ok && !ld_acquire(&sync[2]);
  }
  __syncthreads();
  return ok_s != 0;
}

// Tile t of a symmetric T x T tile grid (upper triangle, row by row) ->
// (tm, tn) with tn >= tm.
__device__ __forceinline__ void sym_tile(int u, int T, int& tm, int& tn) {
  tm = 0;
  while (u >= T - tm) {
    u -= T - tm;
    ++tm;
  }
  tn = tm + u;
}

// Loads the float4 at element k (of kc valid) of a row, zero past the end.
__device__ __forceinline__ float4 ld_row4(const float* src, int k, int kc) {
  if (k + 4 <= kc) return *reinterpret_cast<const float4*>(src);
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (k < kc) v.x = src[0];
  if (k + 1 < kc) v.y = src[1];
  if (k + 2 < kc) v.z = src[2];
  return v;
}

constexpr int LB = 8;  // float4 loads per thread in flight before they are stored

// Stages a 16-row x kc slab whose rows are contiguous along k (rows beyond
// `rows` read as zero) into dst[r * F_LD + k], LB loads in flight per thread.
__device__ __forceinline__ void stage_rows(float* dst, const float* __restrict__ src, long long ld, int r0, int rows,
                                           int k0, int kc) {
  const int kq = (kc + 3) / 4;  // float4 per row
  const int total = FT * kq;
  for (int base = threadIdx.x; base < total; base += F_THREADS * LB) {
    float4 v[LB];
#pragma unroll
    for (int j = 0; j < LB; ++j) {
      const int i = base + j * F_THREADS;
      v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < total) {
        const int r = i / kq, k = (i % kq) * 4;
        if (r0 + r < rows) v[j] = ld_row4(src + static_cast<long long>(r0 + r) * ld + k0 + k, k, kc);
      }
    }
#pragma unroll
    for (int j = 0; j < LB; ++j) {
      const int i = base + j * F_THREADS;
      if (i < total) {
        const int r = i / kq, k = (i % kq) * 4;
        *reinterpret_cast<float4*>(dst + r * F_LD + k) = v[j];
      }
    }
  }
}

// Stages kc rows of 16 columns (k-major storage: row k, columns c0..c0+15)
// transposed into dst[c * F_LD + k]; columns beyond `cols` and rows from kc
// up to the next multiple of 4 (the compute loop's padding) are zero.
__device__ __forceinline__ void stage_cols(float* dst, const float* __restrict__ src, long long ld, int c0, int cols,
                                           int k0, int kc) {
  const int total = ((kc + 3) & ~3) * (FT / 4);
  for (int base = threadIdx.x; base < total; base += F_THREADS * LB) {
    float4 v[LB];
#pragma unroll
    for (int j = 0; j < LB; ++j) {
      const int i = base + j * F_THREADS;
      v[j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < total) {
        const int k = i / (FT / 4), cc = (i % (FT / 4)) * 4;
        if (k < kc) v[j] = ld_row4(src + static_cast<long long>(k0 + k) * ld + c0 + cc, c0 + cc, cols);
      }
    }
#pragma unroll
    for (int j = 0; j < LB; ++j) {
      const int i = base + j * F_THREADS;
      if (i < total) {
        const int k = i / (FT / 4), cc = (i % (FT / 4)) * 4;
        dst[(cc + 0) * F_LD + k] = v[j].x;
        dst[(cc + 1) * F_LD + k] = v[j].y;
        dst[(cc + 2) * F_LD + k] = v[j].z;
        dst[(cc + 3) * F_LD + k] = v[j].w;
      }
    }
  }
}

// One 16 x 16 output tile: out(ty, tx) = sum_k Aop[r0 + ty][k] * B(k, c0 + tx),
// B(k, c) = Bop[c][k] (b_kmajor) or Bop[k][c].  Rows of Aop / Bop beyond their
// extents read as zero.  Returns this thread's sum.
__device__ float tile_dot(const float* __restrict__ Aop, long long lda, int arows, const float* __restrict__ Bop,
                          long long ldb, int bcols, bool b_kmajor, int K, int r0, int c0, float* As, float* Bs) {
  const int tid = threadIdx.x;
  const int ty = tid / FT, tx = tid % FT;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
  for (int k0 = 0; k0 < K; k0 += FKC) {
    const int kc = min(FKC, K - k0);
    const int kc4 = (kc + 3) & ~3;
    __syncthreads();  // the previous chunk's (or tile's) reads of As / Bs are done
    stage_rows(As, Aop, lda, r0, arows, k0, kc);
    if (b_kmajor)
      stage_rows(Bs, Bop, ldb, c0, bcols, k0, kc);
    else
      stage_cols(Bs, Bop, ldb, c0, bcols, k0, kc);
    __syncthreads();
    const float* a = As + ty * F_LD;
    const float* b = Bs + tx * F_LD;
#pragma unroll 4
    for (int k = 0; k < kc4; k += 4) {
      const float4 av = *reinterpret_cast<const float4*>(a + k);
      const float4 bv = *reinterpret_cast<const float4*>(b + k);
      acc0 = fmaf(av.x, bv.x, acc0);
      acc1 = fmaf(av.y, bv.y, acc1);
      acc2 = fmaf(av.z, bv.z, acc2);
      acc3 = fmaf(av.w, bv.w, acc3);
    }
  }
  return (acc0 + acc1) + (acc2 + acc3);
}

__global__ void __launch_bounds__(F_THREADS, 1) ns_f32_kernel(const F32Args p, int* err) {
  extern __shared__ float fsm[];
  float* As = fsm;
  float* Bs = fsm + FT * F_LD;
  const int tid = threadIdx.x;
  const int ty = tid / FT, tx = tid % FT;
  const int T = (p.m + FT - 1) / FT;         // m x m tile grid
  const int Tn = (p.n + FT - 1) / FT;        // columns of X in tiles
  const int sym_tiles = T * (T + 1) / 2;
  const float* cur = p.X0;
  for (int k = 0; k < p.steps; ++k) {
    const bool first = (k == 0), last = (k == p.steps - 1);
    // ---- A = X X^T   (upper tiles; blocks above the diagonal mirrored)
    for (int t = blockIdx.x; t < sym_tiles * p.cnt; t += gridDim.x) {
      const int l = t / sym_tiles;
      int tm, tn;
      sym_tile(t % sym_tiles, T, tm, tn);
      const float* X = cur + l * p.sx;
      float v = tile_dot(X, p.ldx, p.m, X, p.ldx, p.m, true, p.n, tm * FT, tn * FT, As, Bs);
      if (first) v *= p.s2[l];
      const int r = tm * FT + ty, c = tn * FT + tx;
      if (r < p.m && c < p.m) {
        float* A = p.A + l * p.sq;
        A[static_cast<long long>(r) * p.ldm + c] = v;
        if (tn > tm) A[static_cast<long long>(c) * p.ldm + r] = v;
      }
    }
    if (!grid_barrier(p.sync, err)) return;
    // ---- P = c A A + b A + a I   (right operand A as stored)
    for (int t = blockIdx.x; t < sym_tiles * p.cnt; t += gridDim.x) {
      const int l = t / sym_tiles;
      int tm, tn;
      sym_tile(t % sym_tiles, T, tm, tn);
      const float* A = p.A + l * p.sq;
      float v = tile_dot(A, p.ldm, p.m, A, p.ldm, p.m, false, p.m, tm * FT, tn * FT, As, Bs);
      const int r = tm * FT + ty, c = tn * FT + tx;
      if (r < p.m && c < p.m) {
        v = p.c * v + p.b * A[static_cast<long long>(r) * p.ldm + c] + (r == c ? p.a : 0.f);
        float* P = p.P + l * p.sq;
        P[static_cast<long long>(r) * p.ldm + c] = v;
        if (tn > tm) P[static_cast<long long>(c) * p.ldm + r] = v;
      }
    }
    if (!grid_barrier(p.sync, err)) return;
    // ---- X' = P X
    float* nxt = p.Xb[k & 1];
    for (int t = blockIdx.x; t < T * Tn * p.cnt; t += gridDim.x) {
      const int l = t / (T * Tn);
      const int u = t % (T * Tn);
      const int tm = u / Tn, tn = u % Tn;
      const float* P = p.P + l * p.sq;
      const float* X = cur + l * p.sx;
      float v = tile_dot(P, p.ldm, p.m, X, p.ldx, p.n, false, p.m, tm * FT, tn * FT, As, Bs);
      if (first) v *= p.s[l];
      const int r = tm * FT + ty, c = tn * FT + tx;
      if (r < p.m && c < p.n) {
        if (last) {
          float o[1] = {v};
          epilogue_row<1>(p.fin, l, r, c, o, p.m, p.n);
        } else {
          nxt[l * p.sx + static_cast<long long>(r) * p.ldx + c] = v;
        }
      }
    }
    if (last) break;
    if (!grid_barrier(p.sync, err)) return;
    cur = nxt;
  }
}

}  // namespace

bool ns_f32_supported(int m, int n) { return m >= 1 && m <= 1024 && n >= 1; }

cudaError_t launch_ns_f32(const NsF32& g, cudaStream_t st, int* err, int num_sms) {
  if (g.cnt <= 0 || g.steps <= 0) return cudaSuccess;
  if (!ns_f32_supported(g.m, g.n) || (g.ldx & 7) || (g.ldm & 7) || (g.sx & 7) || (g.sq & 7))
    return cudaErrorInvalidValue;
  constexpr int smem = 2 * FT * F_LD * static_cast<int>(sizeof(float));  // 131,584 bytes
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] { attr = cudaFuncSetAttribute(ns_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
  if (attr != cudaSuccess) return attr;
  F32Args p;
  p.X0 = g.X0;
  p.Xb[0] = g.Xp;
  p.Xb[1] = g.Xq;
  p.A = g.A;
  p.P = g.P;
  p.ldx = g.ldx;
  p.ldm = g.ldm;
  p.sx = g.sx;
  p.sq = g.sq;
  p.s = g.s;
  p.s2 = g.s2;
  p.cnt = g.cnt;
  p.m = g.m;
  p.n = g.n;
  p.steps = g.steps;
  p.a = g.a;
  p.b = g.b;
  p.c = g.c;
  p.fin = g.fin;
  p.fin.alpha = 1.f;
  p.fin.alpha_vec = nullptr;
  p.fin.beta = 0.f;
  p.fin.beta_vec = nullptr;
  p.fin.C = nullptr;
  p.sync = g.sync;
  const long long T = (g.m + FT - 1) / FT, Tn = (g.n + FT - 1) / FT;
  const long long most = std::max(T * (T + 1) / 2, T * Tn) * g.cnt;  // tiles of the largest product
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ns_f32_kernel, F_THREADS, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int grid = static_cast<int>(std::min<long long>(most, num_sms));  // every CTA resident: one per SM
  e = cudaMemsetAsync(g.sync, 0, 3 * sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  void* args[] = {&p, &err};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(ns_f32_kernel), dim3(grid), dim3(F_THREADS), args,
                                     smem, st);
}

}  // namespace dmuon
