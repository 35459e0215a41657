// gemm_tc.cu -- batched bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Every Newton-Schulz product of the Muon step is one launch of this kernel:
//   A = X X^T        (both operands K-major rows of X)
//   B = c A A + b A  (A symmetric, so A serves as its own K-major transpose)
//   X' = B X + a X   (X is the MN-major B operand)
// plus the Gram-space products, which have the same two operand forms.
//
// Design (one persistent CTA per SM, 256 threads, warp-specialised):
//   warp 0 lane 0   TMA producer: 128x64 A tile + BNx64 B tile per stage,
//                   128-byte swizzle, into a STAGES-deep ring guarded by
//                   full/empty mbarriers.
//   warp 1 lane 0   MMA issuer: 4 x tcgen05.mma (128 x BN x 16) per stage into
//                   one of two TMEM accumulators (2 x BN fp32 columns), then
//                   tcgen05.commit frees the stage / publishes the tile.
//   warp 2          allocates and frees TMEM.
//   warps 4..7      epilogue: tcgen05.ld 32 columns at a time (warp w reads
//                   TMEM lanes 32*(w-4)..+31 = tile rows), applies
//                   alpha*acc + beta*C (+ diag) or the fused parameter update,
//                   stores to global, and hands the accumulator back.
// The epilogue of tile i overlaps the main loop of tile i+1.  Every mbarrier
// wait is bounded (2 s); on expiry the kernel records kErrTimeout in the
// host-visible error word, every role leaves its loop and TMEM is freed.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

template <int BN, bool B_MN>
__global__ void __launch_bounds__(256, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const Epilogue epi, int M, int N, int K, int batch, int* err) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int tiles_m = (M + BM - 1) / BM;
  const int tiles_n = (N + BN - 1) / BN;
  const int num_kb = (K + BK - 1) / BK;
  const long long tiles_per_mat = static_cast<long long>(tiles_m) * tiles_n;
  const long long total = tiles_per_mat * batch;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (long long t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      const int l = static_cast<int>(t / tiles_per_mat);
      const int rem = static_cast<int>(t % tiles_per_mat);
      const int tm = rem / tiles_n, tn = rem % tiles_n;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
        uint8_t* sa = smem + stage * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
        tma_load_3d(sa, &tmA, &full[stage], kb * BK, tm * BM, l);
        if (B_MN) {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_3d(sb + j * (BK * 128), &tmB, &full[stage], tn * BN + j * 64, kb * BK, l);
        } else {
          tma_load_3d(sb, &tmB, &full[stage], kb * BK, tn * BN, l);
        }
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ MMA issuer
    constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, B_MN);
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (long long t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * BN;
      bool ok = true;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * C::STAGE_BYTES);
        const uint32_t sb = sa + C::A_BYTES;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bdesc =
              B_MN ? smem_desc_sw128(sb + kk * 16 * 128, BK * 128, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
          umma_bf16(d_tmem, adesc, bdesc, IDESC, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue
    const int ew = warp - 4;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      const int l = static_cast<int>(t / tiles_per_mat);
      const int rem = static_cast<int>(t % tiles_per_mat);
      const int tm = rem / tiles_n, tn = rem % tiles_n;
      // every lane observes the barrier; the vote reconverges the warp before
      // the warp-collective tcgen05.ld and makes an abort warp-uniform
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort));
      if (!ok) break;
      tc_fence_after();
      const int row = tm * BM + ew * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        const int col = tn * BN + c0;
        float v[32];
        tmem_ld_32cols(tbase + c0, v);  // warp-collective: all lanes participate
        if (col < N) epilogue_row<32>(epi, l, row, col, v, M, N);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  __syncthreads();
  if (*abort && threadIdx.x == 0 && err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

cudaError_t get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode ? cudaSuccess : cudaErrorNotSupported;
}

// 3-D bf16 tensor map {inner, outer, batch} with 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, long long inner, long long outer, int batch, long long ld,
              long long bstride, int box_inner, int box_outer) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                        static_cast<cuuint64_t>(batch)};
  long long bs = batch > 1 ? bstride : ld * outer;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(bs * 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, bool B_MN>
cudaError_t launch_impl(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms) {
  using C = TcCfg<BN>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(tc_gemm_kernel<BN, B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap ma, mb;
  if (!make_map(&ma, g.A, g.K, g.M, g.batch, g.lda, g.sa, BK, BM)) return cudaErrorInvalidValue;
  bool ok = B_MN ? make_map(&mb, g.B, g.N, g.K, g.batch, g.ldb, g.sb, 64, BK)
                 : make_map(&mb, g.B, g.K, g.N, g.batch, g.ldb, g.sb, BK, BN);
  if (!ok) return cudaErrorInvalidValue;
  const long long tiles =
      static_cast<long long>((g.M + BM - 1) / BM) * ((g.N + BN - 1) / BN) * static_cast<long long>(g.batch);
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  tc_gemm_kernel<BN, B_MN><<<grid, 256, C::SMEM_BYTES, s>>>(ma, mb, g.epi, g.M, g.N, g.K, g.batch, dev_err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0) return cudaSuccess;
  // TMA: 16-byte aligned bases, row and batch strides multiples of 16 bytes.
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(g.A) || !al16(g.B) || (g.lda & 7) || (g.ldb & 7) || (g.sa & 7) || (g.sb & 7))
    return cudaErrorMisalignedAddress;
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  const bool mn = !g.b_kmajor;
  if (g.bn == 128) return mn ? launch_impl<128, true>(g, s, dev_err, num_sms) : launch_impl<128, false>(g, s, dev_err, num_sms);
  return mn ? launch_impl<256, true>(g, s, dev_err, num_sms) : launch_impl<256, false>(g, s, dev_err, num_sms);
}

}  // namespace dmuon
