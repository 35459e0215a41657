// gemm_tc.cu -- batched bf16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Every Newton-Schulz product of the Muon step is one launch of this file's
// kernels:
//   A = X X^T             (both operands K-major rows of X; symmetric result)
//   P = c A A + b A + a I (right operand as stored, MN-major; symmetric
//                          result; the identity is the epilogue's diagonal add)
//   X' = P X              (X is the MN-major right operand)
// and the Gram-space products, which have the same operand forms.
//
// Two kernels, both persistent (one CTA per SM, 384 threads) and
// warp-specialised:
//   warp 0 lane 0   TMA producer into a ring of stages (128-byte swizzle)
//                   guarded by full/empty mbarriers.
//   warp 1 lane 0   MMA issuer: tcgen05.mma per 16-deep k slice into one of
//                   two TMEM accumulators; tcgen05.commit frees the stage and
//                   publishes a finished tile.
//   warp 2          allocates / frees TMEM.
//   warps 4..11     epilogue: tcgen05.ld 32 columns at a time (warp w reads
//                   TMEM lanes 32*(w%4)..+31 = tile rows; the two warps of a
//                   quarter take alternate column chunks), applies the fused
//                   epilogue and stores; then hands the accumulator back.
// tc_gemm_kernel:  one CTA computes a 128 x BN tile (BN = 128 or 256).
// tc_gemm2_kernel: a cluster of two CTAs computes a 256 x 256 tile with
//                  tcgen05.mma.cta_group::2: each CTA loads 128 rows of A and
//                  128 rows/columns of B (32 KB per 64-deep stage instead of
//                  48 KB for the same MMA work per SM), the leader issues the
//                  MMA, and each CTA drains its own 128 accumulator lanes.
// Symmetric results (sym): only blocks on or above the block diagonal run;
// blocks above it are stored twice (as computed and mirrored).  bf16
// results are staged per warp through shared memory and written with TMA
// stores.
// Every mbarrier wait is bounded (2 s); on expiry the kernel records
// kErrTimeout in the host-visible error word, every role leaves its loop and
// TMEM is freed.
#include <cudaTypedefs.h>

#include <mutex>

#include "internal.h"

namespace dmuon {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row

// Tile t of a launch -> (matrix l, tile row tm, tile column tn).
// Tiles are taken in bands of RB tile rows, column by column inside a band,
// so the ~74-148 tiles in flight at once cover a few rows and a few columns
// (their operand rows and columns stay in L2) instead of one or two whole
// tile rows, which re-read the right operand from DRAM once per tile row
// when it is wide.  With sym the result is symmetric and only blocks on or
// above the block diagonal run: row tm holds the tiles tn >= first(tm) =
// floor(tm*bm/bn), i.e. column tn holds the rows tm < ceil((tn+1)*bn/bm).
// Tiles strictly above it (tn > first(tm)) are also stored mirrored;
// diagonal blocks are computed in full and stored as they are, so every
// element is written once.  The order changes nothing in any tile's result.
constexpr int RB = 8;  // tile rows per band

__host__ __device__ __forceinline__ int sym_rows_below(int tn, int bm, int bn) {  // rows tm with first(tm) <= tn
  return ((tn + 1) * bn + bm - 1) / bm;
}

__device__ __forceinline__ void decode_tile(long long t, long long per_mat, int tiles_m, int tiles_n, int bm,
                                            int bn, bool sym, int& l, int& tm, int& tn, bool& mirror) {
  l = static_cast<int>(t / per_mat);
  long long u = t % per_mat;
  mirror = false;
  for (int r0 = 0; r0 < tiles_m; r0 += RB) {
    const int r1 = r0 + RB < tiles_m ? r0 + RB : tiles_m;
    if (!sym) {
      const long long band = static_cast<long long>(r1 - r0) * tiles_n;
      if (u < band) {
        tn = static_cast<int>(u / (r1 - r0));
        tm = r0 + static_cast<int>(u % (r1 - r0));
        return;
      }
      u -= band;
      continue;
    }
    for (int c = (r0 * bm) / bn; c < tiles_n; ++c) {
      int hi = sym_rows_below(c, bm, bn);
      hi = hi < r1 ? hi : r1;
      const int cnt = hi - r0;
      if (u < cnt) {
        tn = c;
        tm = r0 + static_cast<int>(u);
        mirror = tn > (tm * bm) / bn;
        return;
      }
      u -= cnt;
    }
  }
  tm = tiles_m - 1;  // not reached for t < per_mat * batch
  tn = tiles_n - 1;
}

// ---------------------------------------------------------------- staged epilogue
// EPI_STORE with a bf16 result goes through shared memory, one warp at a
// time (no barrier between the epilogue warps).  Eight epilogue warps: the
// two warps of a TMEM lane quarter own the same 32 rows of the CTA's
// 128-row block and take alternate 32-column chunks, so one warp's memory
// latency overlaps its sibling's work.  Per chunk, through a ring of two
// 32 x 32 buffers (64-byte swizzle, conflict free for one row per lane):
//   lane 0 TMA-loads the chunk's C addend into the ring buffer,
//   each lane reads its row of C, forms alpha*acc + beta*C (+ diag) and
//   writes the bf16 result back in place, lane 0 TMA-stores the 32 x 32 box;
//   for a mirrored tile the transposed box goes through a second pair of
//   buffers to the mirrored position.
// A buffer is refilled only after the store issued from it has read it
// (bulk_wait_read).  One bulk group per chunk keeps that accounting exact.
constexpr int EPI_WARPS = 8;                  // two per TMEM lane quarter, alternate chunks
constexpr int THREADS = 128 + 32 * EPI_WARPS;  // warps 0..3: producer, MMA, TMEM, idle
constexpr int CH = 32;                        // columns per chunk
constexpr int WBOX = 32 * CH * 2;             // one 32 x 32 bf16 box, 2 KB
constexpr int NRING = 2;                      // C / result ring per warp
constexpr int WARP_STG = (NRING + 2) * WBOX;  // + 2 mirror buffers
constexpr int STG_TOTAL = EPI_WARPS * WARP_STG;  // 64 KB
constexpr int NCBAR = EPI_WARPS * NRING;      // one mbarrier per ring buffer

struct StageState {
  uint32_t it = 0;      // chunks processed by this warp (ring position)
  uint32_t phases = 0;  // parity bit per ring buffer's mbarrier
};

template <int BN>
__device__ __forceinline__ void store_tile_staged(const Epilogue& e, const CUtensorMap* tmC, const CUtensorMap* tmD,
                                                  const CUtensorMap* tmDm, uint8_t* wstg, uint64_t* cbar,
                                                  uint32_t tbase, int l, int row0w, int col0, int M, int N,
                                                  bool mirror, int lane, int half, StageState& st,
                                                  volatile int* abort) {
  float alpha = e.alpha, beta = e.beta;
  if (e.alpha_vec) alpha *= e.alpha_vec[l];
  if (e.beta_vec) beta *= e.beta_vec[l];
  const bool has_c = e.C != nullptr && beta != 0.f;
  const int row = row0w + lane;
  constexpr int NCH = BN / CH;
  constexpr int STRIDE = EPI_WARPS / 4;  // warps sharing this lane quarter take every STRIDE-th chunk
#pragma unroll 1
  for (int i = half; i < NCH; i += STRIDE) {
    const int col = col0 + i * CH;
    const uint32_t b = st.it % NRING;
    uint8_t* buf = wstg + b * WBOX;
    uint8_t* mbuf = wstg + (NRING + (st.it & 1)) * WBOX;
    const bool live = col < N && row0w < M;  // a 32-row box wholly below the result is not stored
    if (lane == 0) {
      bulk_wait_read<1>();  // the stores issued from these buffers two chunks ago have read them
      if (has_c && live) {
        mbar_arrive_expect_tx(&cbar[b], WBOX);
        tma_load_3d(buf, tmC, &cbar[b], col, row0w, l);
      }
    }
    __syncwarp();
    float v[32];
    tmem_ld_32cols(tbase + i * CH, v);  // warp-collective
    if (live) {
      if (has_c) {
        mbar_wait(&cbar[b], (st.phases >> b) & 1, abort);
        st.phases ^= 1u << b;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4* slot = reinterpret_cast<uint4*>(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4));
        float o[8];
        if (has_c) {
          const uint4 cu = *slot;
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&cu);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float2 f = __bfloat1622float2(h[t]);
            o[2 * t] = alpha * v[q * 8 + 2 * t] + beta * f.x;
            o[2 * t + 1] = alpha * v[q * 8 + 2 * t + 1] + beta * f.y;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) o[t] = alpha * v[q * 8 + t];
        }
        if (e.diag != 0.f) {
#pragma unroll
          for (int t = 0; t < 8; ++t)
            if (col + q * 8 + t == row) o[t] += e.diag;
        }
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(o[2 * t], o[2 * t + 1]);
        *slot = u;
        if (mirror) {
          __nv_bfloat16* mb = reinterpret_cast<__nv_bfloat16*>(mbuf);
#pragma unroll
          for (int t = 0; t < 8; ++t) mb[(q * 8 + t) * 32 + lane] = __float2bfloat16_rn(o[t]);
        }
      }
    }
    fence_proxy_async();
    __syncwarp();
    if (lane == 0) {
      if (live) {
        tma_store_3d(tmD, buf, col, row0w, l);
        if (mirror) tma_store_3d(tmDm, mbuf, row0w, col, l);
      }
      bulk_commit();
    }
    ++st.it;
  }
}

// ---------------------------------------------------------------- transposed parameter write
// EPI_APPLY of a bf16 parameter stored as the transpose of the iterate (a
// tall weight): iterate element (row, col) updates W[col][row].  Per 32 x 32
// chunk the warp moves the W box (32 rows of W, 64 bytes each) through a
// 2 KB staging buffer with 16-byte coalesced loads and stores: 8 memory
// instructions per lane and chunk instead of one 2-byte load and store per
// element.  In the buffer, lane r (iterate row) updates column r of every box
// row: two lanes per 4-byte word, no bank conflict.
__device__ __forceinline__ void box_rw(uint8_t* box, __nv_bfloat16* W, long long ldw, int wr0, int wc0, int nrows,
                                       int ncols, bool vec, bool load, int lane) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int idx = q * 32 + lane;
    const int br = idx >> 2, seg = idx & 3;
    uint4* sp = reinterpret_cast<uint4*>(box + br * 64 + seg * 16);
    if (br >= nrows) continue;
    __nv_bfloat16* gp = W + static_cast<long long>(wr0 + br) * ldw + wc0 + seg * 8;
    if (vec && seg * 8 + 8 <= ncols) {
      if (load)
        *sp = *reinterpret_cast<const uint4*>(gp);
      else
        *reinterpret_cast<uint4*>(gp) = *sp;
    } else {
      __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(sp);
      for (int t = 0; t < 8; ++t)
        if (seg * 8 + t < ncols) {
          if (load)
            h[t] = gp[t];
          else
            gp[t] = h[t];
        }
    }
  }
}

// The fused parameter write of a tile whose weight is stored transposed:
// iterate element (row, col) is W[col][row].  Per 32-column chunk the warp
// moves the 32 x 32 box of W (W rows col.., columns row0w..) through shared
// memory: 16-byte coalesced loads, the update by one lane per W column,
// 16-byte coalesced stores.  The boxes of the warp's chunks alternate
// between two buffers, and each box is fetched with cp.async two chunks
// ahead, so its load is in flight while the previous chunk is updated.
template <int BN>
__device__ __forceinline__ void apply_tile_transposed(const Epilogue& e, uint8_t* wstg, uint32_t tbase, int l,
                                                      int row0w, int col0, int M, int N, int lane, int half) {
  float alpha = e.alpha, beta = e.beta;
  if (e.alpha_vec) alpha *= e.alpha_vec[l];
  if (e.beta_vec) beta *= e.beta_vec[l];
  __nv_bfloat16* W = static_cast<__nv_bfloat16*>(e.W[l]);
  const bool vec = ((reinterpret_cast<uintptr_t>(W) & 15) == 0) && ((e.ldw & 7) == 0);
  const int row = row0w + lane;
  constexpr int STRIDE = EPI_WARPS / 4;
  constexpr int NT = BN / CH / STRIDE;  // chunks of this warp: half, half + STRIDE, ...
  // W box of this warp's chunk t into buffer t & 1: asynchronous for whole
  // 16-byte segments, plain loads for a ragged edge
  auto fetch = [&](int t) {
    const int col = col0 + (half + STRIDE * t) * CH;
    if (col >= N || row0w >= M) return;
    const int nrows = N - col < 32 ? N - col : 32;
    const int ncols = M - row0w < 32 ? M - row0w : 32;
    uint8_t* box = wstg + (t & 1) * WBOX;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int idx = q * 32 + lane;
      const int br = idx >> 2, seg = idx & 3;
      if (br >= nrows) continue;
      const __nv_bfloat16* gp = W + static_cast<long long>(col + br) * e.ldw + row0w + seg * 8;
      uint8_t* sp = box + br * 64 + seg * 16;
      if (vec && seg * 8 + 8 <= ncols) {
        cp_async16(smem_u32(sp), gp, 16);
      } else {
        __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(sp);
        for (int k = 0; k < 8; ++k)
          if (seg * 8 + k < ncols) h[k] = gp[k];
      }
    }
  };
  fetch(0);
  cp_async_commit();
  if (NT > 1) fetch(1);
  cp_async_commit();
#pragma unroll 1
  for (int t = 0; t < NT; ++t) {
    const int i = half + STRIDE * t;
    const int col = col0 + i * CH;
    float v[32];
    tmem_ld_32cols(tbase + i * CH, v);  // warp-collective
    cp_async_wait_group<1>();           // this chunk's box (one newer group may be pending)
    __syncwarp();
    uint8_t* box = wstg + (t & 1) * WBOX;
    const bool live = col < N && row0w < M;
    const int nrows = N - col < 32 ? N - col : 32;     // W rows of the box
    const int ncols = M - row0w < 32 ? M - row0w : 32;  // W columns of the box
    if (live && row < M) {
      __nv_bfloat16* bx = reinterpret_cast<__nv_bfloat16*>(box);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (j >= nrows) break;
        float o = alpha * v[j];
        if (e.C != nullptr && beta != 0.f)
          o += beta * load_elem(e.C, static_cast<long long>(l) * e.sc + static_cast<long long>(row) * e.ldc + col + j,
                                e.c_f32);
        if (e.diag != 0.f && col + j == row) o += e.diag;
        const float w = __bfloat162float(bx[j * 32 + lane]);
        bx[j * 32 + lane] = __float2bfloat16_rn(e.decay * w - e.lr_scale * o);
      }
    }
    __syncwarp();
    if (live) box_rw(box, W, e.ldw, col, row0w, nrows, ncols, vec, false, lane);
    __syncwarp();  // the buffer is free: fetch the chunk after next into it
    if (t + 2 < NT) fetch(t + 2);
    cp_async_commit();
  }
  cp_async_wait_group<0>();
}

long long tiles_per_matrix(int M, int N, int bm, int bn, bool sym) {
  const int tm = (M + bm - 1) / bm, tn = (N + bn - 1) / bn;
  if (!sym) return static_cast<long long>(tm) * tn;
  long long s = 0;
  for (int i = 0; i < tm; ++i) s += tn - (i * bm) / bn;
  return s;
}

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN == 256 ? 3 : 5;
  static constexpr int TMEM_COLS = 2 * BN;  // two accumulators
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_TOTAL + 1024 /*align*/ + 256 /*barriers*/;
};

// ============================================================== one CTA per tile
template <int BN, bool B_MN>
__global__ void __launch_bounds__(THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                   const __grid_constant__ CUtensorMap tmDm, const Epilogue epi, int M, int N, int K, int batch,
                   int sym, long long per_mat, int staged, int* err) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES;  // 1024-aligned staging for the epilogue
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + STG_TOTAL);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* cbar = tempty + 2;  // NCBAR: C loads of the staged epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cbar + NCBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCBAR; ++i) mbar_init(&cbar[i], 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI_WARPS);  // one arrival per epilogue warp
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
  grid_dep_wait();  // the previous kernel's results are complete and visible from here on

  const int tiles_m = (M + BM - 1) / BM;
  const int tiles_n = (N + BN - 1) / BN;
  const int num_kb = (K + BK - 1) / BK;
  const long long total = per_mat * batch;
  const bool sy = sym != 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    for (long long t = blockIdx.x; t < total && !*abort; t += gridDim.x) {
      int l, tm, tn;
      bool mir;
      decode_tile(t, per_mat, tiles_m, tiles_n, BM, BN, sy, l, tm, tn, mir);
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
    // drain: the last commits on every stage have arrived before the CTA exits
    for (int i = 0; i < C::STAGES && !*abort; ++i) {
      if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
      if (++stage == C::STAGES) {
        stage = 0;
        phase ^= 1;
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
    const int ep = warp - 4;       // epilogue warp 0..EPI_WARPS-1
    const int ew = warp & 3;       // TMEM lane quarter this warp may read
    const int half = ep >> 2;      // which of the quarter's warps
    int acc = 0;
    uint32_t acc_phase = 0;
    StageState st;
    uint8_t* wstg = stg + ep * WARP_STG;
    const bool apply_t = !staged && epi.mode == EPI_APPLY && epi.transposed && !epi.w_f32;
    for (long long t = blockIdx.x; t < total; t += gridDim.x) {
      int l, tm, tn;
      bool mir;
      decode_tile(t, per_mat, tiles_m, tiles_n, BM, BN, sy, l, tm, tn, mir);
      // every lane observes the barrier; the vote reconverges the warp before
      // the warp-collective tcgen05.ld and makes an abort warp-uniform
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort));
      if (!ok) break;
      tc_fence_after();
      const int row = tm * BM + ew * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * BN;
      if (staged) {
        store_tile_staged<BN>(epi, &tmC, &tmD, &tmDm, wstg, cbar + ep * NRING, tbase, l, tm * BM + ew * 32, tn * BN,
                              M, N, mir, lane, half, st, abort);
      } else if (apply_t) {
        apply_tile_transposed<BN>(epi, wstg, tbase, l, tm * BM + ew * 32, tn * BN, M, N, lane, half);
      } else {
#pragma unroll 1
        for (int c0 = half * 32; c0 < BN; c0 += 32 * (EPI_WARPS / 4)) {
          const int col = tn * BN + c0;
          float v[32];
          tmem_ld_32cols(tbase + c0, v);  // warp-collective: all lanes participate
          if (col < N) epilogue_row<32>(epi, l, row, col, v, M, N, mir);
        }
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

  if (warp >= 4 && lane == 0) bulk_wait<0>();  // each warp's staged stores complete before the CTA exits
  grid_dep_launch();
  __syncthreads();
  if (*abort && threadIdx.x == 0 && err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ============================================================== CTA pair per 256 x 256 tile
constexpr int P_BM = 256;                       // tile rows (128 per CTA)
constexpr int P_BN = 256;                       // tile columns (128 per CTA's B half)
constexpr int P_A_BYTES = BM * BK * 2;          // 16 KB
constexpr int P_B_BYTES = (P_BN / 2) * BK * 2;  // 16 KB
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_STAGES = 5;
constexpr int P_TMEM_COLS = 2 * P_BN;  // two 256-column accumulators = all 512 columns
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + STG_TOTAL + 1024 + 256;

// Symmetric operands stored upper-only (flags).  A chain of products on
// pair tiles keeps each symmetric result as its 256 x 256 blocks on and above
// the block diagonal, without the mirrored copy.  A consumer reads a sub-tile
// that lies below the diagonal from the stored block across it, transposed:
//   A operand (rows of block tm, a 64-deep k block in block kb/4 < tm):
//     stored rows k, columns m -> two 64 x 64 boxes, the MN-major A layout;
//   B operand taken as stored, MN-major (k block in block kb/4 > tn):
//     stored rows n, columns k -> one 64 x 128 box, the K-major B layout.
// The MMA of that k block takes the matching descriptors and major-ness; the
// values are the ones the mirror would have held, so results are unchanged.
constexpr int SYM_A = 1;    // A operand is a symmetric matrix stored upper-only
constexpr int SYM_B = 2;    // B operand (as stored) is one
constexpr int SYM_OUT = 4;  // the symmetric result is stored upper-only (no mirror)

template <bool B_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tc_gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                    const __grid_constant__ CUtensorMap tmDm, const __grid_constant__ CUtensorMap tmAt,
                    const __grid_constant__ CUtensorMap tmBt, const Epilogue epi, int M, int N, int K, int batch,
                    int sym, long long per_mat, int staged, int flags, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stg = smem + P_STAGES * P_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + STG_TOTAL);
  uint64_t* empty = full + P_STAGES;
  uint64_t* tfull = empty + P_STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* cbar = tempty + 2;  // NCBAR: C loads of the staged epilogue
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cbar + NCBAR);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader (issues the MMA)

  if (threadIdx.x == 0) {
    for (int i = 0; i < NCBAR; ++i) mbar_init(&cbar[i], 1);
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);   // used in the leader only: its arrive_expect_tx
      mbar_init(&empty[s], 1);  // one multicast commit per phase, in both CTAs
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);   // multicast commit, both CTAs
      mbar_init(&tempty[a], 2 * EPI_WARPS);  // leader's: every epilogue warp of both CTAs
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (flags & SYM_A) tma_prefetch_desc(&tmAt);
    if ((flags & SYM_B) && B_MN) tma_prefetch_desc(&tmBt);
  }
  if (warp == 2) {
    tmem_alloc2(tmem_slot, P_TMEM_COLS);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // the previous kernel's results are complete and visible from here on

  const int tiles_m = (M + P_BM - 1) / P_BM;
  const int tiles_n = (N + P_BN - 1) / P_BN;
  const int num_kb = (K + BK - 1) / BK;
  const long long total = per_mat * batch;
  const bool sy = sym != 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    int stage = 0;
    uint32_t phase = 0;
    for (long long t = pair; t < total && !*abort; t += npairs) {
      int l, tm, tn;
      bool mir;
      decode_tile(t, per_mat, tiles_m, tiles_n, P_BM, P_BN, sy, l, tm, tn, mir);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
        uint8_t* sa = smem + stage * P_STAGE_BYTES;
        uint8_t* sb = sa + P_A_BYTES;
        const uint32_t fbar = mapa_shared(smem_u32(&full[stage]), 0);
        if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
        const int kblk = (kb * BK) / P_BM;  // the 256-block of this k range
        const int m0 = tm * P_BM + static_cast<int>(rank) * BM;
        if ((flags & SYM_A) && kblk < tm) {  // below the diagonal: the stored block across it, transposed
#pragma unroll
          for (int j = 0; j < BM / 64; ++j)
            tma_load_3d_pair(sa + j * (BK * 128), &tmAt, fbar, m0 + j * 64, kb * BK, l);
        } else {
          tma_load_3d_pair(sa, &tmA, fbar, kb * BK, m0, l);
        }
        const int n0 = tn * P_BN + static_cast<int>(rank) * (P_BN / 2);
        if (B_MN && (flags & SYM_B) && kblk > tn) {
          tma_load_3d_pair(sb, &tmBt, fbar, kb * BK, n0, l);
        } else if (B_MN) {
#pragma unroll
          for (int j = 0; j < P_BN / 2 / 64; ++j)
            tma_load_3d_pair(sb + j * (BK * 128), &tmB, fbar, n0 + j * 64, kb * BK, l);
        } else {
          tma_load_3d_pair(sb, &tmB, fbar, kb * BK, n0, l);
        }
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    for (int i = 0; i < P_STAGES && !*abort; ++i) {  // drain the last commits
      if (!mbar_wait(&empty[stage], phase ^ 1, abort)) break;
      if (++stage == P_STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------ MMA issuer (leader)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (long long t = pair; t < total && !*abort; t += npairs) {
      int l, tm = 0, tn = 0;
      bool mir;
      if (flags & (SYM_A | SYM_B)) decode_tile(t, per_mat, tiles_m, tiles_n, P_BM, P_BN, sy, l, tm, tn, mir);
      if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + acc * P_BN;
      bool ok = true;
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + stage * P_STAGE_BYTES);
        const uint32_t sb = sa + P_A_BYTES;
        const int kblk = (kb * BK) / P_BM;
        const bool a_mn = (flags & SYM_A) && kblk < tm;           // A loaded transposed (MN-major)
        const bool b_mn = B_MN && !((flags & SYM_B) && kblk > tn);  // B as stored (MN-major) or transposed
        const uint32_t idesc = idesc_bf16_f32(P_BM, P_BN, b_mn, a_mn);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t adesc =
              a_mn ? smem_desc_sw128(sa + kk * 16 * 128, BK * 128, 1024) : smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bdesc =
              b_mn ? smem_desc_sw128(sb + kk * 16 * 128, BK * 128, 1024) : smem_desc_sw128(sb + kk * 32, 16, 1024);
          umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit_pair(&empty[stage], 0x3);
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit_pair(&tfull[acc], 0x3);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    const int ep = warp - 4;
    const int ew = warp & 3;
    const int half = ep >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    StageState st;
    uint8_t* wstg = stg + ep * WARP_STG;
    const bool apply_t = !staged && epi.mode == EPI_APPLY && epi.transposed && !epi.w_f32;
    for (long long t = pair; t < total; t += npairs) {
      int l, tm, tn;
      bool mir;
      decode_tile(t, per_mat, tiles_m, tiles_n, P_BM, P_BN, sy, l, tm, tn, mir);
      if (flags & SYM_OUT) mir = false;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&tfull[acc], acc_phase, abort));
      if (!ok) break;
      tc_fence_after();
      const int row0 = tm * P_BM + static_cast<int>(rank) * BM;
      const int row = row0 + ew * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(ew * 32) << 16) + acc * P_BN;
      if (staged) {
        store_tile_staged<P_BN>(epi, &tmC, &tmD, &tmDm, wstg, cbar + ep * NRING, tbase, l, row0 + ew * 32,
                                tn * P_BN, M, N, mir, lane, half, st, abort);
      } else if (apply_t) {
        apply_tile_transposed<P_BN>(epi, wstg, tbase, l, row0 + ew * 32, tn * P_BN, M, N, lane, half);
      } else {
#pragma unroll 1
        for (int c0 = half * 32; c0 < P_BN; c0 += 32 * (EPI_WARPS / 4)) {
          const int col = tn * P_BN + c0;
          float v[32];
          tmem_ld_32cols(tbase + c0, v);
          if (col < N) epilogue_row<32>(epi, l, row, col, v, M, N, mir);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  if (warp >= 4 && lane == 0) bulk_wait<0>();  // each warp's staged stores complete before the CTA exits
  grid_dep_launch();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (*abort && threadIdx.x == 0 && err) *reinterpret_cast<volatile int*>(err) = kErrTimeout;
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, P_TMEM_COLS);
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

// 3-D bf16 tensor map {inner, outer, batch}.
bool make_map(CUtensorMap* m, const void* base, long long inner, long long outer, int batch, long long ld,
              long long bstride, int box_inner, int box_outer,
              CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                        static_cast<cuuint64_t>(batch)};
  long long bs = batch > 1 ? bstride : ld * outer;
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld * 2), static_cast<cuuint64_t>(bs * 2)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_outer), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Maps of the staged epilogue: 32 x 32 boxes of C (load) and of D (store),
// 64-byte swizzle to match the staging layout, and the mirrored 32 x 32 box
// of D without swizzle.  Returns false when the result cannot take the staged
// path (the epilogue then stores from registers).
bool make_stage_maps(const TcGemm& g, CUtensorMap* mc, CUtensorMap* md, CUtensorMap* mm) {
  const Epilogue& e = g.epi;
  if (e.mode != EPI_STORE || e.d_f32 || !e.D) return false;
  if ((reinterpret_cast<uintptr_t>(e.D) & 15) || (e.ldd & 7) || (g.batch > 1 && (e.sd & 7))) return false;
  if (e.C && (e.c_f32 || (reinterpret_cast<uintptr_t>(e.C) & 15) || (e.ldc & 7) || (g.batch > 1 && (e.sc & 7))))
    return false;
  if (!make_map(md, e.D, g.N, g.M, g.batch, e.ldd, e.sd, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return false;
  if (!make_map(mm, e.D, g.N, g.M, g.batch, e.ldd, e.sd, 32, 32, CU_TENSOR_MAP_SWIZZLE_NONE)) return false;
  if (e.C && !make_map(mc, e.C, g.N, g.M, g.batch, e.ldc, e.sc, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B)) return false;
  return true;
}

template <int BN, bool B_MN>
cudaError_t launch_one(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms) {
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
  CUtensorMap mc = ma, md = ma, mm = ma;
  const int staged = make_stage_maps(g, &mc, &md, &mm) ? 1 : 0;
  const long long per_mat = tiles_per_matrix(g.M, g.N, BM, BN, g.sym);
  const long long tiles = per_mat * g.batch;
  const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_gemm_kernel<BN, B_MN>, ma, mb, mc, md, mm, g.epi, g.M, g.N, g.K, g.batch,
                            g.sym ? 1 : 0, per_mat, staged, dev_err);
}

template <bool B_MN>
cudaError_t launch_pair(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms) {
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(attr_once, [num_sms] {
    attr_err = cudaFuncSetAttribute(tc_gemm2_kernel<B_MN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    P_SMEM_BYTES);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, tc_gemm2_kernel<B_MN>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      max_clusters = num_sms / 2;
    }
    if (max_clusters <= 0) max_clusters = num_sms / 2;
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap ma, mb;
  if (!make_map(&ma, g.A, g.K, g.M, g.batch, g.lda, g.sa, BK, BM)) return cudaErrorInvalidValue;
  bool ok = B_MN ? make_map(&mb, g.B, g.N, g.K, g.batch, g.ldb, g.sb, 64, BK)
                 : make_map(&mb, g.B, g.K, g.N, g.batch, g.ldb, g.sb, BK, P_BN / 2);
  if (!ok) return cudaErrorInvalidValue;
  CUtensorMap mc = ma, md = ma, mm = ma;
  const int staged = make_stage_maps(g, &mc, &md, &mm) ? 1 : 0;
  // transposed views of upper-only symmetric operands: A's stored rows k,
  // columns m in 64 x 64 boxes; B's stored rows n, columns k in 64 x 128 boxes
  int flags = g.upper & (SYM_A | SYM_B | SYM_OUT);
  if ((flags & SYM_A) && g.M != g.K) return cudaErrorInvalidValue;
  if ((flags & SYM_B) && (!B_MN || g.K != g.N)) return cudaErrorInvalidValue;
  if ((flags & SYM_OUT) && !(g.sym && staged)) flags &= ~SYM_OUT;  // the mirror is written unless staged
  CUtensorMap mat = ma, mbt = mb;
  if ((flags & SYM_A) && !make_map(&mat, g.A, g.K, g.M, g.batch, g.lda, g.sa, 64, 64)) return cudaErrorInvalidValue;
  if ((flags & SYM_B) && !make_map(&mbt, g.B, g.N, g.K, g.batch, g.ldb, g.sb, BK, P_BN / 2))
    return cudaErrorInvalidValue;
  const long long per_mat = tiles_per_matrix(g.M, g.N, P_BM, P_BN, g.sym);
  const long long tiles = per_mat * g.batch;
  const long long pairs = tiles < max_clusters ? tiles : max_clusters;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = P_SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tc_gemm2_kernel<B_MN>, ma, mb, mc, md, mm, mat, mbt, g.epi, g.M, g.N, g.K, g.batch,
                            g.sym ? 1 : 0, per_mat, staged, flags, dev_err);
}

}  // namespace

bool tensor_map_bf16(CUtensorMap* m, const void* base, long long inner, long long outer, int batch, long long ld,
                     long long bstride, int box_inner, int box_outer) {
  if (get_encode() != cudaSuccess) return false;
  return make_map(m, base, inner, outer, batch, ld, bstride, box_inner, box_outer);
}

long long tc_gemm_tiles(int M, int N, int batch, int tile, bool sym) {
  if (tile == 512) return tiles_per_matrix(M, N, P_BM, P_BN, sym) * batch;
  return tiles_per_matrix(M, N, BM, tile == 128 ? 128 : 256, sym) * batch;
}

cudaError_t launch_tc_gemm(const TcGemm& g, cudaStream_t s, int* dev_err, int num_sms) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0 || g.batch <= 0) return cudaSuccess;
  if (g.sym && g.M != g.N) return cudaErrorInvalidValue;
  // TMA: 16-byte aligned bases, row and batch strides multiples of 16 bytes.
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(g.A) || !al16(g.B) || (g.lda & 7) || (g.ldb & 7) || (g.sa & 7) || (g.sb & 7))
    return cudaErrorMisalignedAddress;
  cudaError_t e = get_encode();
  if (e != cudaSuccess) return e;
  TcGemm h = g;
  h.epi.sym = g.sym ? 1 : 0;
  const bool mn = !g.b_kmajor;
  if (g.tile == 512)
    return mn ? launch_pair<true>(h, s, dev_err, num_sms) : launch_pair<false>(h, s, dev_err, num_sms);
  if (g.tile == 128)
    return mn ? launch_one<128, true>(h, s, dev_err, num_sms) : launch_one<128, false>(h, s, dev_err, num_sms);
  return mn ? launch_one<256, true>(h, s, dev_err, num_sms) : launch_one<256, false>(h, s, dev_err, num_sms);
}

}  // namespace dmuon
