// ns_small.cu -- resident Newton-Schulz for small matrices (m <= 128, n <= 512).
//
// "Some matrices fill a GPU alone, some must be grouped to feed it" (DMuon
// release article, section 2): for small shapes this kernel runs all K
// quintic steps of a group inside one CTA per block of matrices, with the
// iterate, A and P resident in shared memory and the accumulators in TMEM,
// so nothing goes back to HBM between steps.
//
// Up to 8 matrices (m <= 128 / g rows each, g a power of two) are stacked
// into one 128-row block, so every tcgen05.mma runs at its full M = 128:
//   S = X X^T       (128 x 128, K = n)   cross-matrix blocks are zeroed, so
//   A = s^2 S       (first step) is block-diagonal,
//   P = c A A + b A + a I                 block-diagonal as well, and
//   X' = P X        (128 x n, K = 128)   acts on each matrix separately.
// X, A and P live in the 128-byte-swizzled K-major layout that the MMA reads
// directly; the same bytes serve as the MN-major right operand (a K-major
// matrix with rows = k is the MN-major layout of its row-major self).  P
// overwrites A in place (each thread reads its row of A before writing the
// same row of P), and the three products of a step run one after another,
// so each accumulates from TMEM column 0: a CTA needs max(128, n) columns.
// For n <= 256 that is 97 KB of shared memory and 256 TMEM columns, so two
// CTAs share an SM and each hides the other's latency.
// Eight warps drain the accumulators: the two warps of a TMEM lane quarter
// own the same 32 rows and take alternate 32-column chunks, so each pass
// between two products takes half as long as with one warp per quarter.
// One thread issues the MMAs; every wait is bounded (2 s).
#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int SM_ROWS = 128;
constexpr int ATOM = SM_ROWS * 128;  // one 64-column K-major atom: 128 rows x 128 B = 16 KB

// Byte offset of element (r, c) in a 128-row, SW128 K-major tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (c >> 6) * ATOM + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

// Writes 32 consecutive columns col..col+31 of row r (fp32) as bf16.
__device__ __forceinline__ void put_row32(uint8_t* tile, int r, int col, const float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(o[q * 8 + 2 * t], o[q * 8 + 2 * t + 1]);
    *reinterpret_cast<uint4*>(tile + sw128_off(r, col + q * 8)) = u;
  }
}

__device__ __forceinline__ void get_row32(const uint8_t* tile, int r, int col, float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = *reinterpret_cast<const uint4*>(tile + sw128_off(r, col + q * 8));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = __bfloat1622float2(h[t]);
      o[q * 8 + 2 * t] = f.x;
      o[q * 8 + 2 * t + 1] = f.y;
    }
  }
}

__device__ __forceinline__ bool finite_scale(float s) { return s > 0.f && s <= 3.0e38f; }  // false for NaN and Inf

struct SmallArgs {
  const __nv_bfloat16* X0;  // [cnt][m][ldx] unnormalised iterate (wide orientation)
  long long ldx;
  const float* s;           // 1 / (||U|| + eps) per matrix
  const float* s2;
  int cnt, m, n, g, mr;     // g matrices of mr rows per CTA
  int steps;
  float a, b, c;
  Epilogue fin;             // final write: apply / out / store, per matrix
};

// Issues the K/16 MMAs of one product and commits them to `bar`.
__device__ __forceinline__ void issue(uint32_t d_tmem, uint32_t a_base, uint32_t b_base, bool b_mn, int K, int N,
                                      uint64_t* bar) {
  const uint32_t idesc = idesc_bf16_f32(SM_ROWS, N, b_mn);
  for (int kk = 0; kk < K / 16; ++kk) {
    const uint64_t ad = smem_desc_sw128(a_base + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
    const uint64_t bd = b_mn ? smem_desc_sw128(b_base + kk * 16 * 128, ATOM, 1024)
                             : smem_desc_sw128(b_base + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
    umma_bf16(d_tmem, ad, bd, idesc, kk != 0 ? 1u : 0u);
  }
  umma_commit(bar);
}

__host__ __device__ constexpr int small_tmem_cols(int n) { return n <= 128 ? 128 : (n <= 256 ? 256 : 512); }

constexpr int SM_THREADS = 256;  // 8 warps: two per TMEM lane quarter

// Drains columns [0, limit) of this warp's TMEM lanes in the 32-column chunks
// half*32, half*32 + 64, ... (the other warp of the lane quarter takes the
// rest); fn(c0, v) gets each chunk as fp32.  With PAIR two loads are in
// flight per wait (for passes whose fn needs few registers).
template <bool PAIR, typename F>
__device__ __forceinline__ void drain(uint32_t trow, int half, int limit, F&& fn) {
#pragma unroll 1
  for (int c0 = half * 32; c0 < limit; c0 += PAIR ? 128 : 64) {
    uint32_t r0[32], r1[32];
    const bool two = PAIR && c0 + 64 < limit;  // warp-uniform
    tmem_ld_32cols_async(trow + c0, r0);
    if (two) tmem_ld_32cols_async(trow + c0 + 64, r1);
    tmem_wait_ld();
    float v[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r0[t]);
    fn(c0, v);
    if (two) {
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(r1[t]);
      fn(c0 + 64, v);
    }
  }
}

__global__ void __launch_bounds__(SM_THREADS, 2) ns_small_kernel(const SmallArgs p, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int xatoms = (p.n + 63) / 64;
  uint8_t* Xs = smem;                      // 128 x n, xatoms atoms
  uint8_t* As = Xs + xatoms * ATOM;        // 128 x 128: A, then P in place
  uint8_t* Ps = As;
  uint64_t* bar = reinterpret_cast<uint64_t*>(As + 2 * ATOM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* live = const_cast<int*>(abort) + 1;  // [8]

  const int tid = threadIdx.x, warp = tid >> 5;
  const int r = tid & (SM_ROWS - 1);    // TMEM lane = tile row of this thread
  const int half = tid >> 7;            // which of the lane quarter's two warps: 32-column chunks half, half+2, ...
  const int j = r / p.mr, i = r % p.mr;  // matrix of the block, row inside it
  const int l = blockIdx.x * p.g + j;    // matrix index in the group
  const bool valid_row = (l < p.cnt) && (i < p.m);

  if (tid == 0) {
    mbar_init(bar, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, small_tmem_cols(p.n));
    tmem_relinquish();
  }
  // Which of this block's matrices have a positive finite scale s.  A matrix
  // whose s is not (a NaN or Inf in its gradient) is loaded as zeros: the
  // stacked products multiply across matrices (0 * NaN = NaN), so its values
  // must not reach the shared tile; its output is NaN instead.
  if (tid < p.g) {
    const int ll = blockIdx.x * p.g + tid;
    live[tid] = ll < p.cnt && finite_scale(p.s[ll]);
  }
  // The fused update reads every weight of the block at the end: start
  // bringing them into L2 now, behind the Newton-Schulz steps.
  if (p.fin.mode == EPI_APPLY) {
    const int esz = p.fin.w_f32 ? 4 : 2;
    const long long srows = p.fin.transposed ? p.n : p.m, scols = p.fin.transposed ? p.m : p.n;
    const long long bytes = ((srows - 1) * p.fin.ldw + scols) * esz;
    for (int jj = 0; jj < p.g && blockIdx.x * p.g + jj < p.cnt; ++jj) {
      const uint8_t* w = static_cast<const uint8_t*>(p.fin.W[blockIdx.x * p.g + jj]);
      for (long long off = static_cast<long long>(tid) * 128; off < bytes; off += SM_THREADS * 128) prefetch_l2(w + off);
      if (tid == 0) prefetch_l2(w + bytes - 1);
    }
  }
  __syncthreads();
  // X0 -> shared (zero rows outside the matrices), as 16-byte asynchronous
  // copies so that all of a thread's loads are in flight at once.
  const int chunks = xatoms * 8;  // 16-byte chunks per row (n padded to 64)
  for (int idx = tid; idx < SM_ROWS * chunks; idx += SM_THREADS) {
    const int rr = idx / chunks, q = idx % chunks;
    const int jj = rr / p.mr, ii = rr % p.mr, ll = blockIdx.x * p.g + jj;
    uint8_t* dst = Xs + sw128_off(rr, q * 8);
    if (live[jj] && ii < p.m && q * 8 < p.n) {
      const __nv_bfloat16* src = p.X0 + static_cast<long long>(ll) * p.m * p.ldx + static_cast<long long>(ii) * p.ldx + q * 8;
      if (q * 8 + 8 <= p.n) {
        cp_async16(smem_u32(dst), src, 16);
      } else {
        uint4 u = make_uint4(0, 0, 0, 0);
        __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(&u);
        for (int t = 0; t < 8 && q * 8 + t < p.n; ++t) h[t] = src[t];
        *reinterpret_cast<uint4*>(dst) = u;
      }
    } else {
      cp_async16(smem_u32(dst), p.X0, 0);  // zero fill
    }
  }
  cp_async_wait_all();
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t xs = smem_u32(Xs), as = smem_u32(As), ps = smem_u32(Ps);
  // A poisoned matrix runs with zero scales, so its rows of X, A and P stay
  // zero (its stacked neighbours see only zeros); its output is NaN.
  const bool poisoned = valid_row && !finite_scale(p.s[l]);
  const float sl = valid_row && !poisoned ? p.s[l] : 0.f;
  const float s2l = valid_row && !poisoned ? p.s2[l] : 0.f;
  const int npad = xatoms * 64;
  uint32_t phase = 0;
  bool ok = true;

  for (int k = 0; k < p.steps && ok; ++k) {
    const bool first = (k == 0), last = (k == p.steps - 1);
    // ---- S = X X^T
    if (tid == 0) issue(tmem, xs, xs, false, npad, SM_ROWS, bar);
    ok = mbar_wait(bar, phase, abort);
    phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    drain<true>(trow, half, SM_ROWS, [&](int c0, float (&v)[32]) {
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const bool same = ((c0 + t) / p.mr) == j;
        v[t] = same ? (first ? s2l * v[t] : v[t]) : 0.f;  // block-diagonal A
      }
      put_row32(As, r, c0, v);
    });
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- P = c A A + b A + a I
    if (tid == 0) issue(tmem, as, as, true, SM_ROWS, SM_ROWS, bar);
    ok = mbar_wait(bar, phase, abort);
    phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    drain<false>(trow, half, SM_ROWS, [&](int c0, float (&v)[32]) {
      float av[32];
      get_row32(As, r, c0, av);  // this row of A, then the same row of P over it
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = p.c * v[t] + p.b * av[t] + ((c0 + t) == r ? p.a : 0.f);
      put_row32(Ps, r, c0, v);
    });
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // ---- X' = P X  (N up to 512 in two halves of at most 256 columns)
    if (tid == 0) {
      const int n0 = npad < 256 ? npad : 256;
      const uint32_t idesc0 = idesc_bf16_f32(SM_ROWS, n0, true);
      for (int kk = 0; kk < SM_ROWS / 16; ++kk) {
        const uint64_t ad = smem_desc_sw128(ps + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
        umma_bf16(tmem, ad, smem_desc_sw128(xs + kk * 16 * 128, ATOM, 1024), idesc0, kk != 0 ? 1u : 0u);
      }
      if (npad > 256) {
        const uint32_t idesc1 = idesc_bf16_f32(SM_ROWS, npad - 256, true);
        for (int kk = 0; kk < SM_ROWS / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(ps + (kk >> 2) * ATOM + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem + 256, ad, smem_desc_sw128(xs + 4 * ATOM + kk * 16 * 128, ATOM, 1024), idesc1,
                    kk != 0 ? 1u : 0u);
        }
      }
      umma_commit(bar);
    }
    ok = mbar_wait(bar, phase, abort);
    phase ^= 1;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    const float alpha = first ? sl : 1.f;
    if (!last) {
      drain<false>(trow, half, npad, [&](int c0, float (&v)[32]) {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] *= alpha;
        put_row32(Xs, r, c0, v);
      });
    } else {
      drain<false>(trow, half, npad, [&](int c0, float (&v)[32]) {
        if (!valid_row || c0 >= p.n) return;
        // fin: alpha 1 (the step's scale is applied here), per-matrix pointers
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = poisoned ? __int_as_float(0x7fc00000) : v[t] * alpha;
        epilogue_row<32>(p.fin, l, i, c0, v, p.m, p.n);
      });
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (p.steps == 0 && valid_row) {  // O = s X0
#pragma unroll 1
    for (int c0 = half * 32; c0 < p.n; c0 += 64) {
      float v[32];
      get_row32(Xs, r, c0, v);
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = poisoned ? __int_as_float(0x7fc00000) : v[t] * sl;
      epilogue_row<32>(p.fin, l, i, c0, v, p.m, p.n);
    }
  }
  __syncthreads();
  if (*abort && tid == 0 && err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, small_tmem_cols(p.n));
  }
}

}  // namespace

bool ns_small_supported(int m, int n) { return m >= 1 && m <= 128 && n >= 1 && n <= 512; }

int ns_small_group(int m) {
  int g = 1;
  while (g < 8 && m * 2 * g <= 128) g *= 2;
  return g;
}

cudaError_t launch_ns_small(const void* X0, long long ldx, const float* s, const float* s2, int cnt, int m, int n,
                            int steps, float a, float b, float c, const Epilogue& fin, cudaStream_t st, int* err) {
  if (cnt <= 0) return cudaSuccess;
  if (!ns_small_supported(m, n) || (ldx & 7) || (reinterpret_cast<uintptr_t>(X0) & 15)) return cudaErrorInvalidValue;
  SmallArgs p;
  p.X0 = static_cast<const __nv_bfloat16*>(X0);
  p.ldx = ldx;
  p.s = s;
  p.s2 = s2;
  p.cnt = cnt;
  p.m = m;
  p.n = n;
  p.g = ns_small_group(m);
  p.mr = SM_ROWS / p.g;
  p.steps = steps;
  p.a = a;
  p.b = b;
  p.c = c;
  p.fin = fin;
  p.fin.alpha = 1.f;
  p.fin.alpha_vec = nullptr;
  p.fin.beta = 0.f;
  p.fin.C = nullptr;
  const int xatoms = (n + 63) / 64;                     // X: up to 8 atoms (n <= 512)
  const int smem = (xatoms + 2) * ATOM + 1024 + 64;      // + A / P (2 atoms), alignment, barrier
  constexpr int kMaxSmem = (8 + 2) * ATOM + 1024 + 64;   // 164,928 bytes
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem);
  });
  if (attr != cudaSuccess) return attr;
  const int grid = (cnt + p.g - 1) / p.g;
  ns_small_kernel<<<grid, SM_THREADS, smem, st>>>(p, err);
  return cudaGetLastError();
}

}  // namespace dmuon
