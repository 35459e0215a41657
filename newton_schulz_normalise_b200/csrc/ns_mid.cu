// ns_mid.cu -- resident Newton-Schulz for medium bf16 matrices (m <= 256, n <= 1024).
//
// Small matrices must be grouped to feed the GPU (DMuon release article,
// section 2).  A 256 x 1024 matrix is too large for one CTA to keep on chip
// (its bf16 iterate alone is 512 KB), but A = X X^T and the polynomial P are
// 256 x 256: here one cluster of two CTAs (a tcgen05 cta_group::2 pair,
// M = 256) runs all K steps of the direct form for one matrix at a time,
// keeping A and P in shared memory and streaming X over k from the scratch:
//   S  = X X^T      K = n: each CTA loads its 128 rows of X per 64-deep k
//                   block, and that one box is both its half of the MMA's A
//                   operand and its half of B (B's N range = its rows).
//   A  = s^2 S      (first step) drained from TMEM into each CTA's shared
//                   memory as its 128 rows, K-major; then each CTA gathers
//                   A[0..255][its 128 columns] (its own rows from itself,
//                   the peer's through distributed shared memory) into the
//                   MN-major layout of the right operand: A as stored.
//   P  = c A A + b A + a I   written over A in place (row by row).
//   X' = P X        (s on the first step) in chunks of 256 columns, X as the
//                   MN-major right operand (64 x 64 boxes, each CTA its half
//                   of the chunk's columns), two TMEM accumulators so a
//                   chunk's drain overlaps the next chunk's MMAs.  A chunk of
//                   X' depends only on the same chunk of X, whose loads are
//                   complete before its MMAs, so X' overwrites X in place
//                   (the working buffer Xw; X0 itself is only read).  The
//                   last step ends in the caller's epilogue instead.
// Warps 0-7 drain TMEM (two per lane quarter, alternate 32-column chunks),
// warp 8 lane 0 issues TMA loads, warp 9 owns TMEM and, in the leader CTA,
// lane 0 issues the MMAs.  Every thread passes the same cluster barriers in
// the same order whatever happens, and every mbarrier wait is bounded (2 s):
// a stalled pipeline records kErrTimeout and the kernel runs to its end
// without waiting further.
#include <algorithm>
#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int HR = 128;                     // rows per CTA (TMEM lanes)
constexpr int MATOM = HR * 128;             // 16 KB: 128 rows x 64 bf16, 128-byte swizzled, K-major
constexpr int MSTAGES = 4;
constexpr int MSTAGE = 16384;               // S: 128 rows x 64 k; X': 64 k x 2 boxes of 64 n
constexpr int AOP_BYTES = 4 * MATOM;        // own 128 rows of A (then P), K = 256
constexpr int BLAY_BLOCK = 256 * 128;       // 256 k-rows x 64 n (128 B), MN-major
constexpr int BLAY_BYTES = 2 * BLAY_BLOCK;  // this CTA's 128 columns
constexpr int MID_THREADS = 320;            // warps 0-7 drain, 8 producer, 9 TMEM / MMA
constexpr int MID_SMEM = MSTAGES * MSTAGE + AOP_BYTES + BLAY_BYTES + 1024 + 256;

struct MidArgs {
  int cnt, m, n, steps;
  float a, b, c;
  const float* s;   // 1 / (||U|| + eps) per matrix
  const float* s2;
  __nv_bfloat16* Xw;
  long long ldx, sx;
  Epilogue fin;     // last step: alpha 1 (the first step's scale is applied here)
};

// Byte offset of element (r, c) of a 128-row, 128-byte-swizzled K-major tile
// made of 64-column atoms.
__device__ __forceinline__ uint32_t kmaj_off(int r, int c) {
  return (c >> 6) * MATOM + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}

__device__ __forceinline__ void put32(uint8_t* tile, int r, int col, const float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(o[q * 8 + 2 * t], o[q * 8 + 2 * t + 1]);
    *reinterpret_cast<uint4*>(tile + kmaj_off(r, col + q * 8)) = u;
  }
}

__device__ __forceinline__ void get32(const uint8_t* tile, int r, int col, float (&o)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 u = *reinterpret_cast<const uint4*>(tile + kmaj_off(r, col + q * 8));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float2 f = __bfloat1622float2(h[t]);
      o[q * 8 + 2 * t] = f.x;
      o[q * 8 + 2 * t + 1] = f.y;
    }
  }
}

__device__ __forceinline__ uint4 ld_dsmem_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Orders this thread's generic-proxy global writes before later async-proxy
// (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void phase_sync() {
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(MID_THREADS, 1)
    ns_mid_kernel(const __grid_constant__ CUtensorMap mK0, const __grid_constant__ CUtensorMap mN0,
                  const __grid_constant__ CUtensorMap mKw, const __grid_constant__ CUtensorMap mNw, const MidArgs p,
                  int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Aop = smem + MSTAGES * MSTAGE;
  uint8_t* Blay = Aop + AOP_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(Blay + BLAY_BYTES);
  uint64_t* empty = full + MSTAGES;
  uint64_t* accb = empty + MSTAGES;  // S and P products done (multicast commit)
  uint64_t* tfull = accb + 1;        // X' chunk accumulator a ready
  uint64_t* tempty = tfull + 2;      // leader's: accumulator a drained by both CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (tid == 0) {
    for (int i = 0; i < MSTAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(accb, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 8);  // every drain warp of both CTAs
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&mK0);
    tma_prefetch_desc(&mN0);
    tma_prefetch_desc(&mKw);
    tma_prefetch_desc(&mNw);
  }
  if (warp == 9) {
    tmem_alloc2(tmem_slot, 512);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nS = (p.n + 63) / 64;    // k blocks of S = X X^T
  const int nC = (p.n + 255) / 256;  // column chunks of X' = P X
  const int nX = nC * 4;             // X' loads per step (K = 256 in 4 blocks)
  const int pre = nX < MSTAGES ? nX : MSTAGES;
  const bool drain = warp < 8;
  const int q = warp & 3, half = warp >> 2;
  const int rloc = q * 32 + lane;                       // this thread's accumulator row in the CTA
  const int grow = static_cast<int>(rank) * HR + rloc;  // its row in the matrix
  const uint32_t tlane = tmem + (static_cast<uint32_t>(q * 32) << 16);
  const uint32_t fbar0 = mapa_shared(smem_u32(&full[0]), 0);
  const uint32_t aop_s = smem_u32(Aop), blay_s = smem_u32(Blay);
  const uint32_t peer_aop = mapa_shared(aop_s, rank ^ 1u);
  constexpr uint32_t IDESC_K = idesc_bf16_f32(256, 256, false);
  constexpr uint32_t IDESC_MN = idesc_bf16_f32(256, 256, true);

  // pipeline state (each role keeps its own)
  int pst = 0, mst = 0;           // producer / MMA ring position
  uint32_t pph = 0, mph = 0;
  uint32_t accph = 0;             // drains: parity of accb
  uint32_t use_mma[2] = {0, 0};   // MMA: uses of each X' accumulator
  uint32_t use_drn[2] = {0, 0};   // drains: uses of each X' accumulator

  for (int l = pair; l < p.cnt; l += npairs) {
    for (int k = 0; k < p.steps; ++k) {
      const bool first = (k == 0), last = (k == p.steps - 1);
      const CUtensorMap* mK = first ? &mK0 : &mKw;
      const CUtensorMap* mN = first ? &mN0 : &mNw;
      // ------------------------------------------------ S = X X^T
      if (warp == 8 && lane == 0) {
        for (int i = 0; i < nS + pre && !*abort; ++i) {  // S blocks, then the first X' blocks
          if (!mbar_wait(&empty[pst], pph ^ 1, abort)) break;
          uint8_t* st = smem + pst * MSTAGE;
          const uint32_t fb = fbar0 + static_cast<uint32_t>(pst * 8);
          if (rank == 0) mbar_arrive_expect_tx(&full[pst], 2 * MSTAGE);
          if (i < nS) {
            tma_load_3d_pair(st, mK, fb, i * 64, static_cast<int>(rank) * HR, l);
          } else {
            const int j = (i - nS) / 4, kb = (i - nS) % 4;
            const int n0 = j * 256 + static_cast<int>(rank) * 128;
            tma_load_3d_pair(st, mN, fb, n0, kb * 64, l);
            tma_load_3d_pair(st + 8192, mN, fb, n0 + 64, kb * 64, l);
          }
          if (++pst == MSTAGES) {
            pst = 0;
            pph ^= 1;
          }
        }
      }
      if (warp == 9 && lane == 0 && rank == 0) {
        bool ok = true;
        for (int kb = 0; kb < nS && ok; ++kb) {
          ok = mbar_wait(&full[mst], mph, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + mst * MSTAGE);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t d = smem_desc_sw128(sa + kk * 32, 16, 1024);
            umma_bf16_pair(tmem, d, d, IDESC_K, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(&empty[mst], 0x3);
          if (++mst == MSTAGES) {
            mst = 0;
            mph ^= 1;
          }
        }
        if (ok) umma_commit_pair(accb, 0x3);
      }
      __syncwarp();
      if (drain) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accb, accph, abort));
        if (ok) {
          tc_fence_after();
          const float sc = first ? p.s2[l] : 1.f;
#pragma unroll 1
          for (int c0 = half * 32; c0 < 256; c0 += 64) {
            float v[32];
            tmem_ld_32cols(tlane + c0, v);
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] *= sc;
            put32(Aop, rloc, c0, v);
          }
        }
      }
      accph ^= 1;
      fence_proxy_async();
      phase_sync();  // both CTAs' rows of A are in shared memory
      // ------------------------------------------------ gather A[:, own columns] (MN-major)
      if (drain) {
        for (int u = tid; u < 2 * 256 * 8; u += 256) {
          const int j = u >> 11, kr = (u >> 3) & 255, c8 = u & 7;
          const uint32_t src = static_cast<uint32_t>((2 * static_cast<int>(rank) + j) * MATOM + (kr & 127) * 128 +
                                                     ((c8 ^ (kr & 7)) << 4));
          const bool mine = (kr >> 7) == static_cast<int>(rank);
          const uint4 v = mine ? *reinterpret_cast<const uint4*>(Aop + src) : ld_dsmem_v4(peer_aop + src);
          *reinterpret_cast<uint4*>(Blay + j * BLAY_BLOCK + kr * 128 + ((c8 ^ (kr & 7)) << 4)) = v;
        }
      }
      fence_proxy_async();
      phase_sync();  // both operand layouts complete; the peer no longer reads this CTA's A
      // ------------------------------------------------ P = c A A + b A + a I
      if (warp == 9 && lane == 0 && rank == 0 && !*abort) {
#pragma unroll 1
        for (int kk = 0; kk < 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(aop_s + (kk >> 2) * MATOM + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(blay_s + kk * 16 * 128, BLAY_BLOCK, 1024);
          umma_bf16_pair(tmem, ad, bd, IDESC_MN, kk != 0 ? 1u : 0u);
        }
        umma_commit_pair(accb, 0x3);
      }
      __syncwarp();
      if (drain) {
        const bool ok = __all_sync(0xffffffffu, mbar_wait(accb, accph, abort));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int c0 = half * 32; c0 < 256; c0 += 64) {
            float v[32], av[32];
            tmem_ld_32cols(tlane + c0, v);
            get32(Aop, rloc, c0, av);
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] = p.c * v[t] + p.b * av[t] + (c0 + t == grow ? p.a : 0.f);
            put32(Aop, rloc, c0, v);
          }
        }
      }
      accph ^= 1;
      fence_proxy_async();
      phase_sync();  // P complete in both CTAs
      // ------------------------------------------------ X' = P X, chunk by chunk
      if (warp == 8 && lane == 0) {
        for (int i = pre; i < nX && !*abort; ++i) {
          if (!mbar_wait(&empty[pst], pph ^ 1, abort)) break;
          uint8_t* st = smem + pst * MSTAGE;
          const uint32_t fb = fbar0 + static_cast<uint32_t>(pst * 8);
          if (rank == 0) mbar_arrive_expect_tx(&full[pst], 2 * MSTAGE);
          const int j = i / 4, kb = i % 4;
          const int n0 = j * 256 + static_cast<int>(rank) * 128;
          tma_load_3d_pair(st, mN, fb, n0, kb * 64, l);
          tma_load_3d_pair(st + 8192, mN, fb, n0 + 64, kb * 64, l);
          if (++pst == MSTAGES) {
            pst = 0;
            pph ^= 1;
          }
        }
      }
      if (warp == 9 && lane == 0 && rank == 0) {
        bool ok = !*abort;
        for (int j = 0; j < nC && ok; ++j) {
          const int a = j & 1;
          if (use_mma[a] > 0) ok = mbar_wait(&tempty[a], (use_mma[a] - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t dt = tmem + static_cast<uint32_t>(a * 256);
          for (int kb = 0; kb < 4 && ok; ++kb) {
            ok = mbar_wait(&full[mst], mph, abort);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sb = smem_u32(smem + mst * MSTAGE);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc_sw128(aop_s + kb * MATOM + kk * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(sb + kk * 16 * 128, 8192, 1024);
              umma_bf16_pair(dt, ad, bd, IDESC_MN, (kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit_pair(&empty[mst], 0x3);
            if (++mst == MSTAGES) {
              mst = 0;
              mph ^= 1;
            }
          }
          if (ok) umma_commit_pair(&tfull[a], 0x3);
          ++use_mma[a];
        }
      }
      __syncwarp();
      if (drain) {
        const float sc = first ? p.s[l] : 1.f;
        __nv_bfloat16* Xl = p.Xw + static_cast<long long>(l) * p.sx;
        for (int j = 0; j < nC; ++j) {
          const int a = j & 1;
          const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[a], use_drn[a] & 1, abort));
          ++use_drn[a];
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = half * 32; c0 < 256; c0 += 64) {
            const int col = j * 256 + c0;
            float v[32];
            tmem_ld_32cols(tlane + static_cast<uint32_t>(a * 256 + c0), v);
            if (grow >= p.m || col >= p.n) continue;
#pragma unroll
            for (int t = 0; t < 32; ++t) v[t] *= sc;
            if (last) {
              epilogue_row<32>(p.fin, l, grow, col, v, p.m, p.n);
            } else if (col + 32 <= p.n) {
              uint4* dst = reinterpret_cast<uint4*>(Xl + static_cast<long long>(grow) * p.ldx + col);
#pragma unroll
              for (int qq = 0; qq < 4; ++qq) {
                uint4 u;
                __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
                for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(v[qq * 8 + 2 * t], v[qq * 8 + 2 * t + 1]);
                dst[qq] = u;
              }
            } else {
              for (int t = 0; t < 32 && col + t < p.n; ++t)
                Xl[static_cast<long long>(grow) * p.ldx + col + t] = __float2bfloat16_rn(v[t]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[a]), 0));
        }
      }
      fence_proxy_async_global();
      phase_sync();  // the step's iterate is written and visible to the next step's loads
    }
  }
  if (warp == 8 && lane == 0) {  // the last commits on every stage have arrived before the CTA exits
    for (int i = 0; i < MSTAGES && !*abort; ++i) {
      if (!mbar_wait(&empty[pst], pph ^ 1, abort)) break;
      if (++pst == MSTAGES) {
        pst = 0;
        pph ^= 1;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (*abort && tid == 0 && err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc2(tmem, 512);
  }
}

}  // namespace

bool ns_mid_supported(int m, int n) { return m >= 1 && m <= 256 && n <= 1024 && !ns_small_supported(m, n); }

double ns_mid_flops(int m, int n, int steps, int cnt) {
  (void)m;
  const double nS = (n + 63) / 64 * 64.0, nC = (n + 255) / 256 * 256.0;
  return 2.0 * steps * cnt * (256.0 * 256.0 * nS + 256.0 * 256.0 * 256.0 + 256.0 * nC * 256.0);
}

cudaError_t launch_ns_mid(const void* X0, void* Xw, long long ldx, const float* s, const float* s2, int cnt, int m,
                          int n, int steps, float a, float b, float c, const Epilogue& fin, cudaStream_t st, int* err,
                          int num_sms) {
  if (cnt <= 0 || steps <= 0) return cudaSuccess;
  if (!ns_mid_supported(m, n) || (ldx & 7) || (reinterpret_cast<uintptr_t>(X0) & 15) ||
      (reinterpret_cast<uintptr_t>(Xw) & 15))
    return cudaErrorInvalidValue;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [num_sms] {
    attr = cudaFuncSetAttribute(ns_mid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, MID_SMEM);
    if (attr != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(MID_THREADS);
    cfg.dynamicSmemBytes = MID_SMEM;
    cudaLaunchAttribute at;
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = 2;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, ns_mid_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();
      max_clusters = num_sms / 2;
    }
    if (max_clusters <= 0) max_clusters = num_sms / 2;
  });
  if (attr != cudaSuccess) return attr;
  const long long sx = static_cast<long long>(m) * ldx;
  CUtensorMap mK0, mN0, mKw, mNw;
  if (!tensor_map_bf16(&mK0, X0, n, m, cnt, ldx, sx, 64, 128) || !tensor_map_bf16(&mN0, X0, n, m, cnt, ldx, sx, 64, 64) ||
      !tensor_map_bf16(&mKw, Xw, n, m, cnt, ldx, sx, 64, 128) || !tensor_map_bf16(&mNw, Xw, n, m, cnt, ldx, sx, 64, 64))
    return cudaErrorInvalidValue;
  MidArgs p;
  p.cnt = cnt;
  p.m = m;
  p.n = n;
  p.steps = steps;
  p.a = a;
  p.b = b;
  p.c = c;
  p.s = s;
  p.s2 = s2;
  p.Xw = static_cast<__nv_bfloat16*>(Xw);
  p.ldx = ldx;
  p.sx = sx;
  p.fin = fin;
  p.fin.alpha = 1.f;
  p.fin.alpha_vec = nullptr;
  p.fin.beta = 0.f;
  p.fin.beta_vec = nullptr;
  p.fin.C = nullptr;
  const int pairs = static_cast<int>(std::min<long long>(cnt, max_clusters));
  ns_mid_kernel<<<2 * pairs, MID_THREADS, MID_SMEM, st>>>(mK0, mN0, mKw, mNw, p, err);
  return cudaGetLastError();
}

}  // namespace dmuon
