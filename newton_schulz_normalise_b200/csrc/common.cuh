// common.cuh -- device helpers shared by the Muon-step kernels (sm_100a).
//
// PTX wrappers for mbarriers, TMA bulk-tensor loads and the 5th-generation
// tensor cores (tcgen05 / TMEM), every wait bounded in time, and the GEMM
// epilogue that both the tensor-core and the SIMT GEMMs use.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dmuon {

// ---------------------------------------------------------------- errors
// Device-side error code written to the word a launch is given (a mapped
// host word the library checks at its next call, or a slot of the static
// scratch).  Codes match the DMUON_ERR_* values in dmuon.h.
constexpr int kErrTimeout = -5;

// A wait on an mbarrier gives up after this long (ns).  No correct wait in
// these kernels lasts more than a few microseconds.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of `parity` to complete.  Returns false (and raises
// *abort) when the wait exceeds `limit_ns` or another role already aborted,
// so a stalled pipeline ends the kernel instead of hanging it.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait_limit(bar, parity, abort, kWaitLimitNs);
}

// ---------------------------------------------------------------- dependent launch
// With programmatic dependent launch a kernel may start before the previous
// kernel on the stream has finished: everything before grid_dep_wait() must
// not touch memory that kernel writes or reads.  grid_dep_launch() lets the
// next kernel start its own prologue.  Both are no-ops without the launch
// attribute.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}
// 3-D tiled load (x innermost, in elements) into CTA shared memory; completion
// is signalled on `bar` as transaction bytes.  x must be a multiple of 8 for
// 16-bit elements (every caller passes multiples of 64).
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 3-D tiled store from CTA shared memory (bulk async group of this thread).
// Elements of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, const void* src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(m),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D(tmem) (+)= A(smem desc) * B(smem desc), bf16 x bf16 -> fp32.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Issues the load of 32 consecutive fp32 columns of this warp's 32 TMEM lanes
// into r (thread t gets lane base lane + t); r is valid after tmem_wait_ld().
__device__ __forceinline__ void tmem_ld_32cols_async(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 16-byte global -> shared copy that does not block the thread (cp.async);
// with src_bytes 0 it writes zeros and reads nothing.  Complete after
// cp_async_wait_all().
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's committed cp.async groups are pending.
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Asks for the 128-byte line holding p to be brought into L2 (a hint; p must
// lie inside an allocation).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes: thread t gets
// lane (base lane + t), columns col..col+31.
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// A cluster of two CTAs on neighbouring SMs shares one 256-row MMA: the
// leader (rank 0) issues it, each CTA supplies half of A and half of B from
// its own shared memory and holds half of the accumulator in its own TMEM.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared-memory address of the same object in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
  return out;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the mbarrier at `bar`'s offset in every CTA of `mask` once the
// pair's MMAs issued so far are done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}
// 3-D tiled load into this CTA's shared memory whose completion is counted
// on an mbarrier that may live in the peer CTA (cluster address).  No
// multicast: each CTA fetches its own half.
__device__ __forceinline__ void tma_load_3d_pair(void* dst, const CUtensorMap* m, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(m), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled bf16 tile.
//   K-major operand (rows of 64 elements = 128 B along K): lbo unused (16),
//     sbo = 1024 (distance between 8-row groups).
//   MN-major operand (rows of 64 elements = 128 B along M/N, one row per k):
//     lbo = distance between 64-element M/N blocks, sbo = 1024 (8 k-rows).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, bf16 A and B, fp32 D, A K-major or
// MN-major, B K-major or MN-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool b_mn_major, bool a_mn_major = false) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------- epilogue
enum EpiMode : int {
  EPI_STORE = 0,  // D = alpha*acc + beta*C + diag*I, stored as D's dtype
  EPI_APPLY = 1,  // O = alpha*acc + beta*C; W <- decay*W - lr_scale*O (W in original orientation)
  EPI_OUT = 2,    // O = alpha*acc + beta*C written as fp32 in original orientation
};

// Per-launch epilogue description.  Matrix index l of the batch selects the
// per-matrix factors and pointers.
struct Epilogue {
  int mode;
  float alpha, beta, diag;       // scalar factors
  const float* alpha_vec;        // optional per-matrix factor on alpha
  const float* beta_vec;         // optional per-matrix factor on beta
  const void* C;                 // optional addend, dtype c_f32 ? float : bf16
  long long ldc, sc;
  int c_f32;
  void* D;                       // EPI_STORE output
  long long ldd, sd;
  int d_f32;
  void* const* W;                // EPI_APPLY: per-matrix parameter pointers
  float* const* Out;             // EPI_OUT: per-matrix fp32 outputs
  int w_f32;                     // parameter dtype
  int transposed;                // the iterate is the transpose of the stored matrix
  long long ldw;                 // row length of the stored (original) matrix
  float decay, lr_scale;         // W <- decay*W - lr_scale*O
  int sym;                       // EPI_STORE of a symmetric M x M result: only the blocks on
                                 // and above the block diagonal run; blocks above it are
                                 // also stored mirrored (see the tensor-core kernels)
                                 // unless the launch keeps the result upper-only
};

__device__ __forceinline__ float load_elem(const void* p, long long i, int is_f32) {
  return is_f32 ? static_cast<const float*>(p)[i]
                : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}
__device__ __forceinline__ void store_elem(void* p, long long i, float v, int is_f32) {
  if (is_f32)
    static_cast<float*>(p)[i] = v;
  else
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

// Applies the epilogue to `cnt` (<= 32) consecutive columns col..col+cnt-1 of
// row `row` of matrix `l`; v[] holds the fp32 accumulators.  M, N bound the
// valid region.  Vector paths need 16-byte aligned rows (checked).  With
// `mirror` (EPI_STORE of a symmetric result) every element is also stored at
// its transposed position.
template <int CNT>
__device__ __forceinline__ void epilogue_row(const Epilogue& e, int l, int row, int col, const float (&v)[CNT],
                                             int M, int N, bool mirror = false) {
  if (row >= M) return;
  float alpha = e.alpha, beta = e.beta;
  if (e.alpha_vec) alpha *= e.alpha_vec[l];
  if (e.beta_vec) beta *= e.beta_vec[l];
  const bool full = (col + CNT <= N);
  float o[CNT];
  // ---- addend C
  if (e.C != nullptr && beta != 0.f) {
    const long long cbase = static_cast<long long>(l) * e.sc + static_cast<long long>(row) * e.ldc + col;
    if (!e.c_f32 && full && (CNT % 8 == 0) && ((cbase & 7) == 0)) {
      const uint4* cp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(e.C) + cbase);
#pragma unroll
      for (int q = 0; q < CNT / 8; ++q) {
        uint4 u = cp[q];
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float2 f = __bfloat1622float2(h[t]);
          o[q * 8 + 2 * t] = alpha * v[q * 8 + 2 * t] + beta * f.x;
          o[q * 8 + 2 * t + 1] = alpha * v[q * 8 + 2 * t + 1] + beta * f.y;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < CNT; ++j)
        o[j] = (col + j < N) ? alpha * v[j] + beta * load_elem(e.C, cbase + j, e.c_f32) : 0.f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < CNT; ++j) o[j] = alpha * v[j];
  }
  if (e.diag != 0.f && row >= col && row < col + CNT) {
#pragma unroll
    for (int j = 0; j < CNT; ++j)
      if (col + j == row) o[j] += e.diag;
  }
  // ---- output
  if (e.mode == EPI_STORE) {
    const long long dbase = static_cast<long long>(l) * e.sd + static_cast<long long>(row) * e.ldd + col;
    if (mirror) {
      // (c, row): lanes hold consecutive rows, so each c is one contiguous
      // segment across the warp
      const long long mbase = static_cast<long long>(l) * e.sd + row;
#pragma unroll
      for (int j = 0; j < CNT; ++j)
        if (col + j < N) store_elem(e.D, mbase + static_cast<long long>(col + j) * e.ldd, o[j], e.d_f32);
    }
    if (!e.d_f32 && full && (CNT % 8 == 0) && ((dbase & 7) == 0)) {
      uint4* dp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(e.D) + dbase);
#pragma unroll
      for (int q = 0; q < CNT / 8; ++q) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(o[q * 8 + 2 * t], o[q * 8 + 2 * t + 1]);
        dp[q] = u;
      }
    } else {
#pragma unroll
      for (int j = 0; j < CNT; ++j)
        if (col + j < N) store_elem(e.D, dbase + j, o[j], e.d_f32);
    }
  } else if (e.mode == EPI_APPLY) {
    void* W = e.W[l];
    if (!e.transposed) {
      const long long wbase = static_cast<long long>(row) * e.ldw + col;
      // every load is issued before the first store, so the row's loads are
      // in flight together (a store may alias a later load for the compiler)
      if (!e.w_f32 && full && (CNT % 8 == 0) && ((wbase & 7) == 0) &&
          ((reinterpret_cast<uintptr_t>(W) & 15) == 0)) {
        uint4* wp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(W) + wbase);
        uint4 u[CNT / 8 > 0 ? CNT / 8 : 1];
#pragma unroll
        for (int q = 0; q < CNT / 8; ++q) u[q] = wp[q];
#pragma unroll
        for (int q = 0; q < CNT / 8; ++q) {
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u[q]);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            float2 w = __bfloat1622float2(h[t]);
            h[t] = __floats2bfloat162_rn(e.decay * w.x - e.lr_scale * o[q * 8 + 2 * t],
                                         e.decay * w.y - e.lr_scale * o[q * 8 + 2 * t + 1]);
          }
          wp[q] = u[q];
        }
      } else {
        constexpr int G = CNT < 16 ? CNT : 16;  // loads in flight per group (register budget)
#pragma unroll
        for (int j0 = 0; j0 < CNT; j0 += G) {
          float w[G];
#pragma unroll
          for (int j = 0; j < G; ++j) w[j] = (col + j0 + j < N) ? load_elem(W, wbase + j0 + j, e.w_f32) : 0.f;
#pragma unroll
          for (int j = 0; j < G; ++j)
            if (col + j0 + j < N) store_elem(W, wbase + j0 + j, e.decay * w[j] - e.lr_scale * o[j0 + j], e.w_f32);
        }
      }
    } else {
      // iterate element (row, col+j) is stored element (col+j, row): lanes of
      // a warp hold consecutive rows, so each j is a coalesced row segment.
      constexpr int G = CNT < 16 ? CNT : 16;
#pragma unroll
      for (int j0 = 0; j0 < CNT; j0 += G) {
        float w[G];
#pragma unroll
        for (int j = 0; j < G; ++j)
          w[j] = (col + j0 + j < N) ? load_elem(W, static_cast<long long>(col + j0 + j) * e.ldw + row, e.w_f32) : 0.f;
#pragma unroll
        for (int j = 0; j < G; ++j)
          if (col + j0 + j < N)
            store_elem(W, static_cast<long long>(col + j0 + j) * e.ldw + row, e.decay * w[j] - e.lr_scale * o[j0 + j],
                       e.w_f32);
      }
    }
  } else {  // EPI_OUT
    float* out = e.Out[l];
    const long long obase = static_cast<long long>(row) * e.ldw + col;
    if (!e.transposed && full && (CNT % 4 == 0) && ((obase & 3) == 0) &&
        ((reinterpret_cast<uintptr_t>(out) & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < CNT / 4; ++q)
        reinterpret_cast<float4*>(out + obase)[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      return;
    }
#pragma unroll
    for (int j = 0; j < CNT; ++j)
      if (col + j < N) {
        const long long i = e.transposed ? static_cast<long long>(col + j) * e.ldw + row
                                         : static_cast<long long>(row) * e.ldw + col + j;
        out[i] = o[j];
      }
  }
}

}  // namespace dmuon
