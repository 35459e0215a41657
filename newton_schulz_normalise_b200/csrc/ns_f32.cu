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
// 32 x 32 output tiles in turn (a 256 x 512 matrix needs one round per
// product); a tile's operand rows are staged in shared memory whole (up to
// 512 deep at a time) so their loads are in flight together, and each thread
// sums its 2 x 2 outputs over k with independent accumulators added in a
// fixed order (the result does not depend on timing).
// The barrier's waits are bounded (2 s): on expiry the kernel records
// kErrTimeout in the error word and every CTA leaves.
#include <algorithm>
#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int FT = 32;           // output tile rows / columns
constexpr int FH = FT / 2;       // a thread's outputs: rows ty, ty + 16; columns tx, tx + 16
constexpr int FKC = 512;         // k depth staged per chunk
constexpr int F_THREADS = 512;   // two halves of 16 x 16 threads, 2 x 2 outputs each, splitting k
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

__device__ __forceinline__ unsigned ld_relaxed(const unsigned* p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier of the cooperative launch; false once any CTA aborted
// (its own wait timed out, or another CTA's did).  Thread 0 of each CTA
// reads the generation, publishes the CTA's writes and arrives; the last
// arrival resets the count and releases the next generation; the others spin
// on relaxed loads (checking the abort flag and the time limit every 64
// polls) and acquire once the generation moves.
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
      for (unsigned it = 1; ld_relaxed(&sync[1]) == g0; ++it) {
        if ((it & 63) == 0) {
          if (ld_relaxed(&sync[2])) {
            ok = 0;
            break;
          }
          if (global_ns() - t0 > kWaitLimitNs) {
            atomicExch(&sync[2], 1u);
            if (err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
            ok = 0;
            break;
          }
        }
      }
      (void)ld_acquire(&sync[1]);  // orders the other CTAs' results before this CTA's next reads
    }
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

// Stages a 32-row x kc slab whose rows are contiguous along k (rows beyond
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

// Stages kc rows of 32 columns (k-major storage: row k, columns c0..c0+31)
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

// One 32 x 32 output tile: o[i][j] = sum_k Aop[r0 + ty + 16 i][k] * B(k, c0 + tx + 16 j),
// B(k, c) = Bop[c][k] (b_kmajor) or Bop[k][c].  Rows of Aop / Bop beyond their
// extents read as zero.  Rows ty and ty + 16 of a slab sit 16 rows apart, so
// the 16 columns of a quarter warp's 16-byte shared loads hit distinct banks.
// The two halves of the block take the two halves of each staged chunk's k
// range; the upper half's sums are added to the lower half's through shared
// memory (valid in the lower half, threads 0..255), in a fixed order.
__device__ void tile_dot(const float* __restrict__ Aop, long long lda, int arows, const float* __restrict__ Bop,
                         long long ldb, int bcols, bool b_kmajor, int K, int r0, int c0, float* As, float* Bs,
                         float (&o)[2][2]) {
  const int tid = threadIdx.x;
  const int half = tid >> 8, t8 = tid & 255;
  const int ty = t8 / FH, tx = t8 % FH;
  float acc[2][2][2] = {};  // [i][j][even / odd k quad]
  for (int k0 = 0; k0 < K; k0 += FKC) {
    const int kc = min(FKC, K - k0);
    const int kc4 = (kc + 3) & ~3;
    const int kh = ((kc4 / 4 + 1) / 2) * 4;  // the lower half's k range, a multiple of 4
    __syncthreads();  // the previous chunk's (or tile's) reads of As / Bs are done
    stage_rows(As, Aop, lda, r0, arows, k0, kc);
    if (b_kmajor)
      stage_rows(Bs, Bop, ldb, c0, bcols, k0, kc);
    else
      stage_cols(Bs, Bop, ldb, c0, bcols, k0, kc);
    __syncthreads();
    const float* a0 = As + ty * F_LD;
    const float* a1 = As + (ty + FH) * F_LD;
    const float* b0 = Bs + tx * F_LD;
    const float* b1 = Bs + (tx + FH) * F_LD;
    const int kb = half ? kh : 0, ke = half ? kc4 : kh;
#pragma unroll 2
    for (int k = kb; k < ke; k += 4) {
      const int h = (k >> 2) & 1;
      const float4 x0 = *reinterpret_cast<const float4*>(a0 + k);
      const float4 x1 = *reinterpret_cast<const float4*>(a1 + k);
      const float4 y0 = *reinterpret_cast<const float4*>(b0 + k);
      const float4 y1 = *reinterpret_cast<const float4*>(b1 + k);
      acc[0][0][h] = fmaf(x0.x, y0.x, fmaf(x0.y, y0.y, fmaf(x0.z, y0.z, fmaf(x0.w, y0.w, acc[0][0][h]))));
      acc[0][1][h] = fmaf(x0.x, y1.x, fmaf(x0.y, y1.y, fmaf(x0.z, y1.z, fmaf(x0.w, y1.w, acc[0][1][h]))));
      acc[1][0][h] = fmaf(x1.x, y0.x, fmaf(x1.y, y0.y, fmaf(x1.z, y0.z, fmaf(x1.w, y0.w, acc[1][0][h]))));
      acc[1][1][h] = fmaf(x1.x, y1.x, fmaf(x1.y, y1.y, fmaf(x1.z, y1.z, fmaf(x1.w, y1.w, acc[1][1][h]))));
    }
  }
  __syncthreads();  // every thread is done reading As / Bs: the upper half's sums go to Bs
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float v = acc[i][j][0] + acc[i][j][1];
      if (half) Bs[(i * 2 + j) * 256 + t8] = v;
      o[i][j] = v;
    }
  __syncthreads();
  if (!half) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) o[i][j] += Bs[(i * 2 + j) * 256 + t8];
  }
}

__global__ void __launch_bounds__(F_THREADS, 1) ns_f32_kernel(const F32Args p, int* err) {
  extern __shared__ float fsm[];
  float* As = fsm;
  float* Bs = fsm + FT * F_LD;
  const int tid = threadIdx.x;
  const bool writer = tid < 256;             // the lower half holds the finished sums
  const int ty = (tid & 255) / FH, tx = (tid & 255) % FH;
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
      float o[2][2];
      tile_dot(X, p.ldx, p.m, X, p.ldx, p.m, true, p.n, tm * FT, tn * FT, As, Bs, o);
      const float sc = first ? p.s2[l] : 1.f;
      float* A = p.A + l * p.sq;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int r = tm * FT + ty + FH * i, c = tn * FT + tx + FH * j;
          if (writer && r < p.m && c < p.m) {
            A[static_cast<long long>(r) * p.ldm + c] = sc * o[i][j];
            if (tn > tm) A[static_cast<long long>(c) * p.ldm + r] = sc * o[i][j];
          }
        }
    }
    if (!grid_barrier(p.sync, err)) return;
    // ---- P = c A A + b A + a I   (right operand A as stored)
    for (int t = blockIdx.x; t < sym_tiles * p.cnt; t += gridDim.x) {
      const int l = t / sym_tiles;
      int tm, tn;
      sym_tile(t % sym_tiles, T, tm, tn);
      const float* A = p.A + l * p.sq;
      float o[2][2];
      tile_dot(A, p.ldm, p.m, A, p.ldm, p.m, false, p.m, tm * FT, tn * FT, As, Bs, o);
      float* P = p.P + l * p.sq;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int r = tm * FT + ty + FH * i, c = tn * FT + tx + FH * j;
          if (writer && r < p.m && c < p.m) {
            const float v = p.c * o[i][j] + p.b * A[static_cast<long long>(r) * p.ldm + c] + (r == c ? p.a : 0.f);
            P[static_cast<long long>(r) * p.ldm + c] = v;
            if (tn > tm) P[static_cast<long long>(c) * p.ldm + r] = v;
          }
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
      float o[2][2];
      tile_dot(P, p.ldm, p.m, X, p.ldx, p.n, false, p.m, tm * FT, tn * FT, As, Bs, o);
      const float sc = first ? p.s[l] : 1.f;
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int r = tm * FT + ty + FH * i, c = tn * FT + tx + FH * j;
          if (writer && r < p.m && c < p.n) {
            if (last) {
              float v[1] = {sc * o[i][j]};
              epilogue_row<1>(p.fin, l, r, c, v, p.m, p.n);
            } else {
              nxt[l * p.sx + static_cast<long long>(r) * p.ldx + c] = sc * o[i][j];
            }
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
  constexpr int smem = 2 * FT * F_LD * static_cast<int>(sizeof(float));  // 132,096 bytes
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
