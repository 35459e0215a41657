// dmuon_api.cu -- host side of the Muon step: validation, shape groups,
// per-shape autotune cache, scratch layout and the Newton-Schulz drivers
// behind the C ABI of include/dmuon.h.
//
// Shape-adaptive execution (DMuon release article, wjxwpt.net, section 2
// "shape-adaptive execution stack"; DMuon announcement, m.zaocj.com,
// "自變量三招"): matrices are grouped by shape; the first time a shape key is
// met, every candidate (direct or Gram-space Newton-Schulz, tile width) runs
// on that group's own data into scratch, is timed with CUDA events, and must
// agree with the direct form within a gate before it can win; the winner and
// its measured cost are cached and reused for that key.  Section 3 of the
// same article measures each shape group's full computation once and uses
// the costs to order work; on one GPU the groups are issued in descending
// measured cost.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <climits>
#include <atomic>
#include <cmath>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "../../include/dmuon.h"
#include "internal.h"

namespace dmuon {
namespace {

// ------------------------------------------------------------------ errors
thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  if (getenv("DMUON_TRACE")) fprintf(stderr, "[dmuon] error %d: %s\n", code, buf);
  return code;
}

#define CUDA_TRY(expr)                                                                          \
  do {                                                                                          \
    cudaError_t e__ = (expr);                                                                   \
    if (e__ != cudaSuccess) return fail(DMUON_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e__)); \
  } while (0)

bool trace_on() {
  static int v = getenv("DMUON_TRACE") ? 1 : 0;
  return v != 0;
}

// ------------------------------------------------------------------ timing
// While timing is enabled, a launch outside a TimedChain is bracketed by its
// own pair of events.  A TimedChain (the Newton-Schulz products of one chunk,
// run_ns) is bracketed by ONE pair of events around all of its launches:
// nothing else is enqueued between them, so the window is the chain's device
// time, with no event between two of its kernels to delay the next launch or
// break programmatic dependent launch.  A record's kind is that of its first
// launch; `pair` marks chains of the CTA-pair GEMM.
struct TimedLaunch {
  int kind;
  bool pair;
  cudaEvent_t a, b;
  double flops, bytes;
  long long launches;
};
std::mutex g_tmu;
std::atomic<int> g_timing{0};
std::vector<TimedLaunch> g_timed;
std::vector<cudaEvent_t> g_event_pool;
std::atomic<long long> g_launches{0};
thread_local TimedLaunch* t_chain = nullptr;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Runs `launch` (which enqueues one kernel on `s`), bracketed by events when
// timing is enabled and no chain is open.
template <class F>
cudaError_t launch_k(int kind, double flops, double bytes, cudaStream_t s, F&& launch) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_timing.load(std::memory_order_relaxed)) return launch();
  if (t_chain) {
    if (t_chain->launches == 0) t_chain->kind = kind;
    t_chain->flops += flops;
    t_chain->bytes += bytes;
    ++t_chain->launches;
    return launch();
  }
  std::lock_guard<std::mutex> lk(g_tmu);
  TimedLaunch t{kind, false, take_event(), take_event(), flops, bytes, 1};
  cudaEventRecord(t.a, s);
  cudaError_t e = launch();
  cudaEventRecord(t.b, s);
  g_timed.push_back(t);
  return e;
}

// Scope of one timed chain of launches on stream `s` (no-op unless timing).
class TimedChain {
 public:
  TimedChain(cudaStream_t s, bool pair) : s_(s) {
    if (!g_timing.load(std::memory_order_relaxed) || t_chain) return;
    {
      std::lock_guard<std::mutex> lk(g_tmu);
      rec_ = TimedLaunch{KIND_OTHER, pair, take_event(), take_event(), 0.0, 0.0, 0};
    }
    cudaEventRecord(rec_.a, s_);
    t_chain = &rec_;
    on_ = true;
  }
  ~TimedChain() {
    if (!on_) return;
    t_chain = nullptr;
    cudaEventRecord(rec_.b, s_);
    std::lock_guard<std::mutex> lk(g_tmu);
    if (rec_.launches > 0) {
      g_timed.push_back(rec_);
    } else {
      g_event_pool.push_back(rec_.a);
      g_event_pool.push_back(rec_.b);
    }
  }
  TimedChain(const TimedChain&) = delete;
  TimedChain& operator=(const TimedChain&) = delete;

 private:
  cudaStream_t s_;
  TimedLaunch rec_{};
  bool on_ = false;
};

// ------------------------------------------------------------------ device context
struct DeviceCtx {
  int device = -1;
  int num_sms = 148;
  std::string name;
  std::mutex mu;
  void* ws = nullptr;  // scratch
  size_t ws_bytes = 0;
  bool ws_external = false;
  void* ext_ptr = nullptr;
  size_t ext_bytes = 0;
  // pinned staging for pointer tables (two slots, reused after their copy)
  void* pin[2] = {nullptr, nullptr};
  size_t pin_cap[2] = {0, 0};
  cudaEvent_t pin_ev[2] = {nullptr, nullptr};
  bool pin_used[2] = {false, false};
  int pin_next = 0;
  cudaEvent_t last_done = nullptr;
  bool has_last = false;
  int* err_host = nullptr;  // mapped pinned word the kernels write on timeout
  int* err_dev = nullptr;
  cudaEvent_t tune_a = nullptr, tune_b = nullptr;
  // side streams for shape groups too small to fill the GPU on their own
  static constexpr int kSide = 3;
  cudaStream_t side[kSide] = {};
  cudaEvent_t fork_ev = nullptr;
  cudaEvent_t side_done[kSide] = {};
  // AdamW pointer / size tables (device) and the event after the last AdamW launch
  void* adam_tab = nullptr;
  size_t adam_cap = 0;
  cudaEvent_t adam_done = nullptr;
  bool adam_used = false;
  // host I/O pipeline: copy-in and copy-out streams, kIoSlots staging slots
  static constexpr int kIoSlots = 4;
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t g_ready[kIoSlots] = {}, g_free[kIoSlots] = {}, w_done[kIoSlots] = {}, io_done = nullptr;
};

std::mutex g_ctx_mu;
std::map<int, std::unique_ptr<DeviceCtx>> g_ctx;
void* g_ext_ptr = nullptr;  // dmuon_set_workspace (applies to the current device)
size_t g_ext_bytes = 0;

int get_ctx(DeviceCtx** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_ctx_mu);
  auto it = g_ctx.find(dev);
  if (it == g_ctx.end()) {
    auto c = std::make_unique<DeviceCtx>();
    c->device = dev;
    cudaDeviceProp prop;
    CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
    c->num_sms = prop.multiProcessorCount;
    c->name = prop.name;
    if (prop.major != 10) return fail(DMUON_ERR_CUDA, "device %d (%s, sm_%d%d) is not an sm_100 GPU", dev, prop.name, prop.major, prop.minor);
    CUDA_TRY(cudaEventCreateWithFlags(&c->last_done, cudaEventDisableTiming));
    CUDA_TRY(cudaEventCreateWithFlags(&c->pin_ev[0], cudaEventDisableTiming));
    CUDA_TRY(cudaEventCreateWithFlags(&c->pin_ev[1], cudaEventDisableTiming));
    CUDA_TRY(cudaEventCreate(&c->tune_a));
    CUDA_TRY(cudaEventCreate(&c->tune_b));
    CUDA_TRY(cudaEventCreateWithFlags(&c->fork_ev, cudaEventDisableTiming));
    for (int i = 0; i < DeviceCtx::kSide; ++i) {
      CUDA_TRY(cudaStreamCreateWithFlags(&c->side[i], cudaStreamNonBlocking));
      CUDA_TRY(cudaEventCreateWithFlags(&c->side_done[i], cudaEventDisableTiming));
    }
    CUDA_TRY(cudaStreamCreateWithFlags(&c->cin, cudaStreamNonBlocking));
    CUDA_TRY(cudaStreamCreateWithFlags(&c->cout, cudaStreamNonBlocking));
    for (int i = 0; i < DeviceCtx::kIoSlots; ++i) {
      CUDA_TRY(cudaEventCreateWithFlags(&c->g_ready[i], cudaEventDisableTiming));
      CUDA_TRY(cudaEventCreateWithFlags(&c->g_free[i], cudaEventDisableTiming));
      CUDA_TRY(cudaEventCreateWithFlags(&c->w_done[i], cudaEventDisableTiming));
    }
    CUDA_TRY(cudaEventCreateWithFlags(&c->io_done, cudaEventDisableTiming));
    CUDA_TRY(cudaEventCreateWithFlags(&c->adam_done, cudaEventDisableTiming));
    CUDA_TRY(cudaHostAlloc(reinterpret_cast<void**>(&c->err_host), sizeof(int), cudaHostAllocMapped));
    *c->err_host = 0;
    CUDA_TRY(cudaHostGetDevicePointer(reinterpret_cast<void**>(&c->err_dev), c->err_host, 0));
    it = g_ctx.emplace(dev, std::move(c)).first;
  }
  *out = it->second.get();
  return DMUON_OK;
}

bool fault_alloc() {
  const char* f = getenv("DMUON_FAULT");
  return f && strstr(f, "alloc");
}

// DMUON_FAULT=wait: dmuon_compute_update_noalloc ends with a bounded wait
// that nothing completes (20 ms), so its error word records a timeout.
bool fault_wait() {
  const char* f = getenv("DMUON_FAULT");
  return f && strstr(f, "wait");
}

int ensure_ws(DeviceCtx& c, size_t bytes, cudaStream_t s) {
  if (g_ext_ptr) {
    if (bytes > g_ext_bytes)
      return fail(DMUON_ERR_OOM, "caller workspace too small: need %zu bytes, have %zu", bytes, g_ext_bytes);
    c.ws = g_ext_ptr;
    c.ws_bytes = g_ext_bytes;
    c.ws_external = true;
    return DMUON_OK;
  }
  if (c.ws_external) {  // returned to library-managed scratch
    c.ws = nullptr;
    c.ws_bytes = 0;
    c.ws_external = false;
  }
  if (bytes <= c.ws_bytes) return DMUON_OK;
  if (fault_alloc()) return fail(DMUON_ERR_OOM, "injected allocation failure (DMUON_FAULT=alloc)");
  CUDA_TRY(cudaStreamSynchronize(s));
  if (c.ws) {
    CUDA_TRY(cudaDeviceSynchronize());
    CUDA_TRY(cudaFree(c.ws));
    c.ws = nullptr;
    c.ws_bytes = 0;
  }
  size_t want = bytes + (bytes >> 4);  // 6% headroom for the next plan
  cudaError_t e = cudaMalloc(&c.ws, want);
  if (e != cudaSuccess) {
    cudaGetLastError();
    c.ws = nullptr;
    return fail(DMUON_ERR_OOM, "cudaMalloc(%zu) for scratch failed: %s", want, cudaGetErrorString(e));
  }
  c.ws_bytes = want;
  return DMUON_OK;
}

// ------------------------------------------------------------------ plans
struct Plan {
  int variant = DMUON_VARIANT_DIRECT;
  int tile = 256;        // 128 / 256: one CTA per 128 x tile output tile; 512: CTA pair, 256 x 256
  double cost_ms = 0.0;  // measured for one chunk of `chunk` matrices
};

struct Key {
  long long rows, cols;
  int f32, steps, cnt;
  bool operator<(const Key& o) const {
    return std::tie(rows, cols, f32, steps, cnt) < std::tie(o.rows, o.cols, o.f32, o.steps, o.cnt);
  }
};

std::mutex g_cache_mu;
std::map<Key, Plan> g_cache;

// Geometry of one matrix in its wide orientation.
struct Geo {
  int rows, cols;  // stored
  int m, n;        // iterate: m = min, n = max
  bool transposed;
  long long ldx, ldm;  // row strides (elements) of X (m x n) and of m x m buffers
  int esz;             // bytes per element of the iterate
  long long x_elems() const { return static_cast<long long>(m) * ldx; }
  long long q_elems() const { return static_cast<long long>(m) * ldm; }
};

Geo make_geo(long long rows, long long cols, bool f32) {
  Geo g;
  g.rows = static_cast<int>(rows);
  g.cols = static_cast<int>(cols);
  g.transposed = rows > cols;
  g.m = static_cast<int>(std::min(rows, cols));
  g.n = static_cast<int>(std::max(rows, cols));
  g.ldx = (g.n + 7) / 8 * 8;
  g.ldm = (g.m + 7) / 8 * 8;
  g.esz = f32 ? 4 : 2;
  return g;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// The dtype of the Newton-Schulz iterate: the parameters' dtype, except that
// bf16 weights whose iterate has at most kF32IterRows rows iterate in fp32.
// A Gaussian iterate with three to five rows has nearly equal normalised
// singular values, which the five quintic steps still send to clearly
// different values, so each bf16 rounding between the products turns the
// singular vectors and moves the update by several percent (a CPU emulation
// of the bf16 forms: up to 3.6% at 3 rows, 7.3% at 4 and 3.9% at 5; at most
// 1.9% from 6 rows up); products that small leave the tensor cores idle
// anyway.
constexpr long long kF32IterRows = 5;
bool iter_f32(bool param_f32, long long m) { return param_f32 || m <= kF32IterRows; }

// Scratch layout of one chunk of `cnt` matrices.
struct Layout {
  size_t X0, Xp, Xq, A, Bm, P, Q0, Q1, T, partials, s, s2, sync, total;
};

Layout make_layout(const Geo& g, int cnt, int nblk) {
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off += align256(bytes);
    return o;
  };
  const size_t xb = static_cast<size_t>(cnt) * g.x_elems() * g.esz;
  const size_t qb = static_cast<size_t>(cnt) * g.q_elems() * g.esz;
  L.X0 = take(xb);
  L.Xp = take(xb);
  L.Xq = take(xb);
  L.A = take(qb);
  L.Bm = take(qb);
  L.P = take(qb);
  L.Q0 = take(qb);
  L.Q1 = take(qb);
  L.T = L.Bm;  // T and the direct form's polynomial buffer are never live together
  L.partials = take(static_cast<size_t>(cnt) * nblk * sizeof(float));
  L.s = take(static_cast<size_t>(cnt) * sizeof(float));
  L.s2 = take(static_cast<size_t>(cnt) * sizeof(float));
  L.sync = take(16);  // grid-barrier words of the fp32 resident kernel
  L.total = off;
  return L;
}

size_t per_matrix_bytes(const Geo& g) { return 3 * g.x_elems() * g.esz + 5 * g.q_elems() * g.esz + 64; }

size_t budget_bytes() {
  const char* b = getenv("DMUON_WS_BUDGET_MB");
  size_t mb = b ? static_cast<size_t>(atoll(b)) : 8192;
  return mb << 20;
}

int chunk_size(const Geo& g, int count) {
  size_t per = per_matrix_bytes(g);
  size_t c = budget_bytes() / std::max<size_t>(per, 1);
  if (c < 1) c = 1;
  if (c > 65535) c = 65535;
  return static_cast<int>(std::min<size_t>(c, count));
}

// ------------------------------------------------------------------ NS driver
struct Hyper {
  float mu, lr, wd, eps, a, b, c;
  int steps, nesterov;
};

// A chunk of a shape group.  Its geometry g is the iterate's (m x n, m <= n):
// the first nwide matrices are stored m x n, the others n x m (the transposed
// weights of the same dimensions), and the Newton-Schulz products serve both.
struct Chunk {
  const Geo* g;
  int cnt;
  int nwide;
  uint8_t* base;  // scratch of this chunk
  Layout L;
  void* const* Gt;  // device pointer tables for this chunk
  void* const* Bt;
  void* const* Wt;
  float* const* Ot;
  int nblk;
  int aligned;
};

template <class T>
T* at(const Chunk& ch, size_t off) {
  return reinterpret_cast<T*>(ch.base + off);
}

// One GEMM of the NS recursion.  A: M x K rows (ld lda), B: K-major (N x K)
// or MN-major (K x N).  Dispatches to tensor cores (bf16) or SIMT (fp32).
// sym: the M x M result is symmetric; the tensor-core kernels compute only the
// tiles that meet the upper triangle and mirror them (FLOPs counted for the
// computed tiles only).
// upper (CTA-pair tiles only, see TcGemm): which symmetric operands and
// result are kept as their blocks on and above the diagonal.
int gemm(DeviceCtx& c, int cnt, bool f32, int tile, bool sym, const void* A, long long lda, long long sa,
         const void* B, long long ldb, long long sb, bool b_kmajor, int M, int N, int K, const Epilogue& e,
         cudaStream_t s, int upper = 0) {
  cudaError_t err;
  if (!f32) {
    const long long tiles = tc_gemm_tiles(M, N, cnt, tile, sym);
    const long long dense = tc_gemm_tiles(M, N, cnt, tile, false);
    const double flops = 2.0 * M * N * static_cast<double>(K) * cnt * static_cast<double>(tiles) / dense;
    TcGemm t{A, lda, sa, B, ldb, sb, b_kmajor, M, N, K, cnt, tile, sym, e, tile == 512 ? upper : 0};
    err = launch_k(KIND_TC_GEMM, flops, 0.0, s, [&] { return launch_tc_gemm(t, s, c.err_dev, c.num_sms); });
  } else {
    const double flops = 2.0 * M * N * static_cast<double>(K) * cnt;
    SimtGemm t{static_cast<const float*>(A), lda, sa, static_cast<const float*>(B), ldb, sb, b_kmajor, M, N, K, cnt, e};
    err = launch_k(KIND_SIMT_GEMM, flops, 0.0, s, [&] { return launch_simt_gemm(t, s); });
  }
  if (err != cudaSuccess) return fail(DMUON_ERR_CUDA, "gemm %dx%dx%d (batch %d) launch failed: %s", M, N, K, cnt, cudaGetErrorString(err));
  return DMUON_OK;
}

Epilogue store_epi(void* D, long long ldd, long long sd, bool f32, float alpha, const float* alpha_vec) {
  Epilogue e{};
  e.mode = EPI_STORE;
  e.alpha = alpha;
  e.alpha_vec = alpha_vec;
  e.D = D;
  e.ldd = ldd;
  e.sd = sd;
  e.d_f32 = f32;
  e.c_f32 = f32;
  return e;
}

// Runs K1 (momentum + norm partials) for each orientation part of a chunk
// (every launch covers ch.nblk partial slots per matrix), then the finalize.
int run_momentum(const Chunk& ch, bool f32, bool g_f32, const Hyper& h, cudaStream_t s) {
  const Geo& g = *ch.g;
  auto part = [&](int off, int cnt, bool tall) -> int {
    MomentumArgs a{};
    a.G = ch.Gt + off;
    a.B = ch.Bt + off;
    a.X = at<uint8_t>(ch, ch.L.X0) + static_cast<size_t>(off) * g.x_elems() * g.esz;
    a.ldx = g.ldx;
    a.x_f32 = f32;
    a.g_f32 = g_f32;
    a.rows = tall ? g.n : g.m;
    a.cols = tall ? g.m : g.n;
    a.transposed = tall ? 1 : 0;
    a.cnt = cnt;
    a.mu = h.mu;
    a.nesterov = h.nesterov;
    a.partials = at<float>(ch, ch.L.partials) + static_cast<size_t>(off) * ch.nblk;
    a.nblk = ch.nblk;
    a.aligned = ch.aligned;
    const double bytes = static_cast<double>(g.m) * g.n * cnt * ((g_f32 ? 4 : 2) + 8 + (f32 ? 4 : 2));
    cudaError_t e = launch_k(KIND_EW, 0.0, bytes, s, [&] { return launch_momentum(a, s); });
    if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "momentum kernel: %s", cudaGetErrorString(e));
    return DMUON_OK;
  };
  int rc;
  if (ch.nwide > 0 && (rc = part(0, ch.nwide, false))) return rc;
  if (ch.cnt > ch.nwide && (rc = part(ch.nwide, ch.cnt - ch.nwide, true))) return rc;
  cudaError_t e = launch_k(KIND_OTHER, 0.0, 0.0, s, [&] {
    return launch_norm_finalize(at<float>(ch, ch.L.partials), ch.nblk, ch.cnt, h.eps, at<float>(ch, ch.L.s),
                                at<float>(ch, ch.L.s2), s);
  });
  if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "norm finalize: %s", cudaGetErrorString(e));
  return DMUON_OK;
}

// Partial-sum slots per matrix for a chunk holding wide and/or tall
// matrices of the iterate geometry g (the larger of the two launches' grids).
int chunk_nblk(const Geo& g, bool wide, bool tall) {
  int nb = 1;
  if (wide) nb = std::max(nb, momentum_partials(g.m, g.n));
  if (tall) nb = std::max(nb, momentum_partials(g.n, g.m));
  return nb;
}

// The epilogue e for the matrices off, off+1, ... of its tables.
Epilogue shift_epi(Epilogue e, int off) {
  if (e.W) e.W += off;
  if (e.Out) e.Out += off;
  if (e.alpha_vec) e.alpha_vec += off;
  if (e.beta_vec) e.beta_vec += off;
  if (e.D) e.D = static_cast<uint8_t*>(e.D) + static_cast<size_t>(off) * e.sd * (e.d_f32 ? 4 : 2);
  return e;
}

// Newton-Schulz on X0 (unnormalised U, scale s folded into the first
// products), finishing with an epilogue (apply / out / store) on the result:
// fin_w for the chunk's first ch.nwide matrices (stored m x n), fin_t for the
// rest (stored n x m).  Every product but the last serves both orientations
// in one launch; the last runs once per orientation present.  Kernels that
// run every step in one launch (and the zero-step scale) run once per
// orientation part.  The launches are timed as one chain.
int run_ns(DeviceCtx& c, const Chunk& ch, bool f32, int variant, int tile, const Hyper& h, const Epilogue& fin_w,
           const Epilogue& fin_t, int cnt, cudaStream_t s) {
  const Geo& g = *ch.g;
  const int m = g.m, n = g.n;
  const long long sx = g.x_elems(), sq = g.q_elems();
  const float* sv = at<float>(ch, ch.L.s);
  const float* s2v = at<float>(ch, ch.L.s2);
  uint8_t* X0 = at<uint8_t>(ch, ch.L.X0);
  const int split = std::min(std::max(ch.nwide, 0), cnt);
  auto xoff = [&](int off) { return X0 + static_cast<size_t>(off) * sx * g.esz; };
  // runs one(off, count, epilogue) for each orientation part present
  auto parts = [&](auto&& one) -> int {
    int r = DMUON_OK;
    if (split > 0 && (r = one(0, split, shift_epi(fin_w, 0)))) return r;
    if (cnt > split) r = one(split, cnt - split, shift_epi(fin_t, split));
    return r;
  };
  int rc;
  TimedChain chain(s, !f32 && variant != DMUON_VARIANT_BATCHED && tile == 512 && h.steps > 0);
  if (h.steps == 0) {  // O = X0 = s U; the kernel folds s in
    return parts([&](int off, int nn, Epilogue fin) -> int {
      fin.alpha = 1.f;
      fin.alpha_vec = nullptr;
      fin.beta = 0.f;
      fin.C = nullptr;
      cudaError_t e = launch_k(KIND_OTHER, 0.0, 0.0, s, [&] {
        return launch_scale_epilogue(xoff(off), g.ldx, f32, m, n, nn, sv + off, fin, s);
      });
      if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "scale epilogue: %s", cudaGetErrorString(e));
      return DMUON_OK;
    });
  }
  if (variant == DMUON_VARIANT_BATCHED && f32) {  // fp32: every step in one cooperative launch
    return parts([&](int off, int nn, Epilogue fin) -> int {
      NsF32 a{reinterpret_cast<const float*>(xoff(off)), at<float>(ch, ch.L.Xp), at<float>(ch, ch.L.Xq),
              at<float>(ch, ch.L.A), at<float>(ch, ch.L.Bm), g.ldx, g.ldm, sx, sq, sv + off, s2v + off, nn, m, n,
              h.steps, h.a, h.b, h.c, fin, at<unsigned>(ch, ch.L.sync)};
      const double T = (m + 31) / 32;
      const double symf = (T * (T + 1) / 2) / (T * T);
      const double fl = 2.0 * h.steps * nn *
                        (symf * m * static_cast<double>(m) * n + symf * m * static_cast<double>(m) * m +
                         m * static_cast<double>(m) * n);
      cudaError_t e = launch_k(KIND_SIMT_GEMM, fl, 0.0, s, [&] { return launch_ns_f32(a, s, c.err_dev, c.num_sms); });
      if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "fp32 resident kernel: %s", cudaGetErrorString(e));
      return DMUON_OK;
    });
  }
  if (variant == DMUON_VARIANT_BATCHED && !ns_small_supported(m, n)) {  // bf16, medium: one CTA pair per matrix
    return parts([&](int off, int nn, Epilogue fin) -> int {
      cudaError_t e = launch_k(KIND_TC_GEMM, ns_mid_flops(m, n, h.steps, nn), 0.0, s, [&] {
        return launch_ns_mid(xoff(off), g.ldx, sv + off, s2v + off, nn, m, n, h.steps, h.a, h.b, h.c, fin, s,
                             c.err_dev, c.num_sms);
      });
      if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "resident medium-matrix kernel: %s", cudaGetErrorString(e));
      return DMUON_OK;
    });
  }
  if (variant == DMUON_VARIANT_BATCHED) {  // resident small-matrix kernel (bf16)
    return parts([&](int off, int nn, Epilogue fin) -> int {
      cudaError_t e = launch_k(KIND_TC_GEMM, 2.0 * h.steps * (2.0 * 128 * 128 * g.n + 2.0 * 128 * 128 * 128) *
                                                 ((nn + ns_small_group(m) - 1) / ns_small_group(m)),
                               0.0, s, [&] {
                                 return launch_ns_small(xoff(off), g.ldx, sv + off, s2v + off, nn, m, n, h.steps, h.a,
                                                        h.b, h.c, fin, s, c.err_dev);
                               });
      if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "resident small-matrix kernel: %s", cudaGetErrorString(e));
      return DMUON_OK;
    });
  }
  // On CTA-pair tiles every symmetric m x m matrix of the chain is kept as its
  // 256 x 256 blocks on and above the diagonal (no mirrored copy): the
  // products that make one pass UP_OUT, and every product that reads one as
  // its left (UP_A) or right (UP_B) operand reads the blocks below the
  // diagonal from the stored blocks across it.
  constexpr int UP_A = 1, UP_B = 2, UP_OUT = 4;
  // The last product O = scale * Aop Bx (m x n, K = m, Bx the MN-major iterate),
  // once per orientation part with its epilogue.
  auto final_product = [&](const void* Aop, const void* Bx, bool scale, int aflags) -> int {
    return parts([&](int off, int nn, Epilogue fin) -> int {
      fin.alpha = 1.f;
      fin.alpha_vec = scale ? sv + off : nullptr;
      fin.beta = 0.f;
      fin.beta_vec = nullptr;
      fin.C = nullptr;
      return gemm(c, nn, f32, tile, false, static_cast<const uint8_t*>(Aop) + static_cast<size_t>(off) * sq * g.esz,
                  g.ldm, sq, static_cast<const uint8_t*>(Bx) + static_cast<size_t>(off) * sx * g.esz, g.ldx, sx, false,
                  m, n, m, fin, s, aflags);
    });
  };
  if (variant == DMUON_VARIANT_GRAM) {
    // Every m x m product takes its right operand as stored (MN-major B), not
    // as the transpose of a matrix that is symmetric only up to rounding:
    // multiplying by transposes feeds the rounding's antisymmetric part back
    // into the recursion, where it grows from step to step (4e-2 instead of
    // 1e-2 relative error after 5 steps at 96 x 200 in bf16).
    void* A = at<void>(ch, ch.L.A);
    void* P = at<void>(ch, ch.L.P);
    void* T = at<void>(ch, ch.L.T);
    void* Q[2] = {at<void>(ch, ch.L.Q0), at<void>(ch, ch.L.Q1)};
    // G = s^2 U U^T  (A_0): both operands are rows of U (K-major)
    rc = gemm(c, cnt, f32, tile, true, X0, g.ldx, sx, X0, g.ldx, sx, true, m, m, n, store_epi(A, g.ldm, sq, f32, 1.f, s2v), s,
              UP_OUT);
    if (rc) return rc;
    int qi = 0;
    for (int k = 0; k < h.steps; ++k) {
      // P_k = c A_k^2 + b A_k + a I   (into Q[0] when k == 0: Q_1 = P_0)
      void* Pk = (k == 0) ? Q[0] : P;
      Epilogue ep = store_epi(Pk, g.ldm, sq, f32, h.c, nullptr);
      ep.C = A;
      ep.ldc = g.ldm;
      ep.sc = sq;
      ep.beta = h.b;
      ep.diag = h.a;
      // Q_1 = P_0 is the last Q when there is one step: stored in full
      rc = gemm(c, cnt, f32, tile, true, A, g.ldm, sq, A, g.ldm, sq, false, m, m, m, ep, s,
                UP_A | UP_B | (h.steps == 1 ? 0 : UP_OUT));
      if (rc) return rc;
      if (k > 0) {  // Q_{k+1} = P_k Q_k
        rc = gemm(c, cnt, f32, tile, true, Pk, g.ldm, sq, Q[qi], g.ldm, sq, false, m, m, m,
                  store_epi(Q[qi ^ 1], g.ldm, sq, f32, 1.f, nullptr), s,
                  UP_A | UP_B | (k == h.steps - 1 ? 0 : UP_OUT));
        if (rc) return rc;
        qi ^= 1;
      }
      if (k < h.steps - 1) {  // A_{k+1} = P_k A_k P_k
        rc = gemm(c, cnt, f32, tile, true, Pk, g.ldm, sq, A, g.ldm, sq, false, m, m, m,
                  store_epi(T, g.ldm, sq, f32, 1.f, nullptr), s, UP_A | UP_B | UP_OUT);
        if (rc) return rc;
        rc = gemm(c, cnt, f32, tile, true, T, g.ldm, sq, Pk, g.ldm, sq, false, m, m, m,
                  store_epi(A, g.ldm, sq, f32, 1.f, nullptr), s, UP_A | UP_B | UP_OUT);
        if (rc) return rc;
      }
    }
    // O = s * Q_K U; Q_K is stored in full (its blocks below the diagonal
    // mirrored), so the last and largest product reads it K-major
    return final_product(Q[qi], X0, true, 0);
  }
  // ---------------- direct form
  // Per step: A = X X^T, P = c A^2 + b A + a I, X' = P X.  Folding a X into
  // P (its identity term is the epilogue's diagonal add) leaves the X' product
  // without an addend; in bf16 it is as accurate as adding a X in fp32 (one
  // rounding fewer).  The scale s of the first step rides on alpha.
  void* A = at<void>(ch, ch.L.A);
  void* P = at<void>(ch, ch.L.Bm);
  void* bufs[2] = {at<void>(ch, ch.L.Xp), at<void>(ch, ch.L.Xq)};
  void* cur = X0;
  for (int k = 0; k < h.steps; ++k) {
    const bool first = (k == 0);
    const bool last = (k == h.steps - 1);
    // A = X X^T  (s^2 folded in on the first step)
    rc = gemm(c, cnt, f32, tile, true, cur, g.ldx, sx, cur, g.ldx, sx, true, m, m, n,
              store_epi(A, g.ldm, sq, f32, 1.f, first ? s2v : nullptr), s, UP_OUT);
    if (rc) return rc;
    // P = c A A + b A + a I   (right operand as stored, see the Gram form)
    Epilogue ep = store_epi(P, g.ldm, sq, f32, h.c, nullptr);
    ep.C = A;
    ep.ldc = g.ldm;
    ep.sc = sq;
    ep.beta = h.b;
    ep.diag = h.a;
    rc = gemm(c, cnt, f32, tile, true, A, g.ldm, sq, A, g.ldm, sq, false, m, m, m, ep, s, UP_A | UP_B | UP_OUT);
    if (rc) return rc;
    // X' = P X   (times s on the first step)
    if (last) return final_product(P, cur, first, UP_A);
    void* nxt = bufs[k & 1];
    rc = gemm(c, cnt, f32, tile, false, P, g.ldm, sq, cur, g.ldx, sx, false, m, n, m,
              store_epi(nxt, g.ldx, sx, f32, 1.f, first ? sv : nullptr), s, UP_A);
    if (rc) return rc;
    cur = nxt;
  }
  return DMUON_OK;
}

// ------------------------------------------------------------------ step
// A shape group: the matrices whose iterate is m x n (rows = m <= cols = n),
// whether stored m x n or n x m (a weight and a transposed weight of the
// same dimensions share every Newton-Schulz product).  idx lists the ones
// stored m x n first, then the ntall stored n x m.
struct Group {
  long long rows, cols;
  std::vector<int> idx;
  Plan plan;
  int chunk;
  int ntall;
  bool xf = false;  // the iterate is fp32 (iter_f32)
};

struct Request {
  void* const* params;
  const void* const* grads;
  void* const* moms;
  float* const* out;  // dmuon_compute_update
  const int64_t* shapes;
  int count;
  Hyper h;
  dmuon_options o;
  cudaStream_t s;
  bool grads_host = false;             // dmuon_step_host_io: grads in host memory
  void* const* params_host = nullptr;  // dmuon_step_host_io: updated params copied here
};

int validate(const Request& r) {
  if (r.count < 0) return fail(DMUON_ERR_INVALID, "count < 0");
  if (r.count == 0) return DMUON_OK;
  if (!r.grads || !r.moms || !r.shapes || (!r.params && !r.out))
    return fail(DMUON_ERR_INVALID, "null pointer array");
  if (r.h.steps < 0 || r.h.steps > 16) return fail(DMUON_ERR_INVALID, "ns_steps %d outside [0, 16]", r.h.steps);
  const float hs[] = {r.h.lr, r.h.wd, r.h.mu, r.h.eps, r.h.a, r.h.b, r.h.c};
  for (float v : hs)
    if (!std::isfinite(v)) return fail(DMUON_ERR_INVALID, "non-finite hyperparameter");
  if (r.h.eps < 0.f) return fail(DMUON_ERR_INVALID, "eps < 0");
  const dmuon_options& o = r.o;
  if (o.mom_dtype != DMUON_F32) return fail(DMUON_ERR_DTYPE, "momentum dtype must be F32");
  if (!((o.param_dtype == DMUON_BF16 && o.grad_dtype == DMUON_BF16) ||
        (o.param_dtype == DMUON_F32 && o.grad_dtype == DMUON_F32)))
    return fail(DMUON_ERR_DTYPE, "param/grad dtypes must both be BF16 or both F32");
  if (o.variant < 0 || o.variant > 3) return fail(DMUON_ERR_INVALID, "unknown variant %d", o.variant);
  for (int i = 0; i < r.count; ++i) {
    const int64_t rr = r.shapes[2 * i], cc = r.shapes[2 * i + 1];
    if (rr <= 0 || cc <= 0) return fail(DMUON_ERR_INVALID, "matrix %d has shape %lld x %lld", i, (long long)rr, (long long)cc);
    if (rr > (1 << 20) || cc > (1 << 20) || rr * cc > (1LL << 31))
      return fail(DMUON_ERR_INVALID, "matrix %d shape %lld x %lld too large", i, (long long)rr, (long long)cc);
    if (!r.grads[i] || !r.moms[i] || (r.params && !r.params[i]) || (r.out && !r.out[i]) ||
        (r.params_host && !r.params_host[i]))
      return fail(DMUON_ERR_INVALID, "null pointer for matrix %d", i);
  }
  return DMUON_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// DMUON_TILE=128|256|512 restricts the autotuner to one tile shape.
int forced_tile() {
  const char* b = getenv("DMUON_TILE");
  if (b) {
    int v = atoi(b);
    if (v == 128 || v == 256 || v == 512) return v;
  }
  return 0;
}

// The resident variant (DMUON_VARIANT_BATCHED) for this dtype and shape:
// bf16 stacks small matrices in shared memory and TMEM (m <= 128, n <= 512)
// or gives a medium matrix a CTA pair (m <= 256, n <= 1024); fp32 runs every
// step in one cooperative launch (m <= 1024).
bool resident_supported(bool f32, int m, int n) {
  return f32 ? ns_f32_supported(m, n) : (ns_small_supported(m, n) || ns_mid_supported(m, n));
}

double gate_tol() {
  const char* g = getenv("DMUON_GATE");
  return g ? atof(g) : 2e-2;
}

int upload_tables(DeviceCtx& c, const std::vector<void*>& host, void* dev, cudaStream_t s) {
  const size_t bytes = host.size() * sizeof(void*);
  if (bytes == 0) return DMUON_OK;
  const int slot = c.pin_next;
  if (c.pin_used[slot]) CUDA_TRY(cudaEventSynchronize(c.pin_ev[slot]));
  if (c.pin_cap[slot] < bytes) {
    if (c.pin[slot]) CUDA_TRY(cudaFreeHost(c.pin[slot]));
    c.pin[slot] = nullptr;
    size_t cap = std::max<size_t>(bytes, 64 << 10);
    CUDA_TRY(cudaHostAlloc(&c.pin[slot], cap, cudaHostAllocDefault));
    c.pin_cap[slot] = cap;
  }
  memcpy(c.pin[slot], host.data(), bytes);
  CUDA_TRY(cudaMemcpyAsync(dev, c.pin[slot], bytes, cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaEventRecord(c.pin_ev[slot], s));
  c.pin_used[slot] = true;
  c.pin_next ^= 1;
  return DMUON_OK;
}

// The last product's epilogue for the chunk's matrices stored m x n
// (tall = false) or n x m (tall = true; the update is written transposed).
Epilogue final_epilogue(const Request& r, const Geo& g, const Chunk& ch, bool f32, bool tall) {
  Epilogue e{};
  e.transposed = tall ? 1 : 0;
  e.ldw = tall ? g.m : g.n;
  e.w_f32 = f32;
  if (r.out) {
    e.mode = EPI_OUT;
    e.Out = ch.Ot;
  } else {
    e.mode = EPI_APPLY;
    e.W = ch.Wt;
    e.decay = 1.f - r.h.lr * r.h.wd;
    e.lr_scale = r.h.lr * 0.2f * std::sqrt(static_cast<float>(std::max(g.rows, g.cols)));
  }
  return e;
}

int time_ns(DeviceCtx& c, const Chunk& ch, bool f32, int variant, int tile, const Hyper& h, const Epilogue& fin,
            int cnt, cudaStream_t s, float* ms) {
  CUDA_TRY(cudaEventRecord(c.tune_a, s));
  int rc = run_ns(c, ch, f32, variant, tile, h, fin, fin, cnt, s);
  if (rc) return rc;
  CUDA_TRY(cudaEventRecord(c.tune_b, s));
  CUDA_TRY(cudaEventSynchronize(c.tune_b));
  CUDA_TRY(cudaEventElapsedTime(ms, c.tune_a, c.tune_b));
  if (*c.err_host) return fail(DMUON_ERR_DEVICE_TIMEOUT, "device wait timed out during autotune");
  return DMUON_OK;
}

// Chooses the plan for a group by timing candidates on the chunk's own data
// (after the momentum kernel produced X0).  Candidates write their result
// into scratch beyond the chunk layout, never into the caller's buffers.  The
// first candidate (direct form) is the accuracy reference of the gate.
int autotune(DeviceCtx& c, const Chunk& ch, bool f32, const Hyper& h, int forced_variant, Plan* plan,
             cudaStream_t s) {
  const Geo& g = *ch.g;
  std::vector<std::pair<int, int>> cands;  // (variant, tile)
  const int ft = forced_tile();
  std::vector<int> tiles;
  if (f32)
    tiles = {256};  // the SIMT path has one tile shape
  else if (ft)
    tiles = {ft};
  else if (g.m >= 256)
    tiles = {512, 256, 128};
  else
    tiles = {256, 128};
  std::vector<int> vars;
  if (forced_variant == DMUON_VARIANT_DIRECT || forced_variant == DMUON_VARIANT_GRAM)
    vars = {forced_variant};
  else if (forced_variant == DMUON_VARIANT_BATCHED)
    vars = {DMUON_VARIANT_DIRECT};  // reference for the gate; the batched candidate is added below
  else {
    vars = {DMUON_VARIANT_DIRECT};
    if (g.n * 4 >= g.m * 5 && h.steps > 0) vars.push_back(DMUON_VARIANT_GRAM);  // n >= 1.25 m
  }
  for (int v : vars)
    for (int t : tiles) cands.push_back({v, t});
  if (resident_supported(f32, g.m, g.n) && h.steps > 0 &&
      (forced_variant == DMUON_VARIANT_AUTO || forced_variant == DMUON_VARIANT_BATCHED))
    cands.push_back({DMUON_VARIANT_BATCHED, 128});
  if (forced_variant == DMUON_VARIANT_BATCHED && !cands.empty() && cands.back().first == DMUON_VARIANT_BATCHED)
    cands = {{DMUON_VARIANT_DIRECT, tiles[0]}, cands.back()};  // direct stays the gate's reference
  if (h.steps == 0) cands = {{DMUON_VARIANT_DIRECT, tiles[0]}};

  const int probe = ch.cnt;
  uint8_t* outbuf = ch.base + ch.L.total;  // two X-sized slots reserved by the caller
  const size_t xb = align256(static_cast<size_t>(probe) * g.x_elems() * g.esz);
  void* ref_out = outbuf;
  void* cand_out = outbuf + xb;
  double* dacc = reinterpret_cast<double*>(outbuf + 2 * xb);

  float best = 1e30f;
  Plan bestp;
  bool have_ref = false;
  bool forced_batched_ok = false;
  double forced_batched_ms = 0.0;
  for (auto [v, tile] : cands) {
    const bool is_ref = !have_ref;
    void* dst = is_ref ? ref_out : cand_out;
    Epilogue fin = store_epi(dst, g.ldx, g.x_elems(), f32, 1.f, nullptr);
    float ms = 0.f;
    // warm once (first launch of a kernel instance loads the module), then time
    int rc = run_ns(c, ch, f32, v, tile, h, fin, fin, probe, s);
    if (rc) return rc;
    rc = time_ns(c, ch, f32, v, tile, h, fin, probe, s, &ms);
    if (rc) return rc;
    bool pass = true;
    double relerr = 0.0;
    if (!is_ref) {
      CUDA_TRY(cudaMemsetAsync(dacc, 0, 2 * sizeof(double), s));
      cudaError_t e = launch_diff_norms(cand_out, ref_out, g.ldx, g.m, g.n, probe, f32, dacc, s);
      if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "diff norms: %s", cudaGetErrorString(e));
      double hacc[2];
      CUDA_TRY(cudaMemcpyAsync(hacc, dacc, sizeof(hacc), cudaMemcpyDeviceToHost, s));
      CUDA_TRY(cudaStreamSynchronize(s));
      relerr = hacc[1] > 0 ? std::sqrt(hacc[0] / hacc[1]) : std::sqrt(hacc[0]);
      pass = relerr <= gate_tol();
    }
    if (trace_on())
      fprintf(stderr, "[dmuon] tune %dx%d cnt=%d variant=%d tile=%d: %.3f ms%s gate=%.2e %s\n", g.rows, g.cols, probe,
              v, tile, ms, is_ref ? " (reference)" : "", relerr, pass ? "pass" : "REJECT");
    have_ref = true;
    if (v == DMUON_VARIANT_BATCHED && pass) {
      forced_batched_ok = true;
      forced_batched_ms = ms;
    }
    if (pass && ms < best) {
      best = ms;
      bestp.variant = v;
      bestp.tile = tile;
      bestp.cost_ms = ms;
    }
  }
  if (forced_variant == DMUON_VARIANT_BATCHED && forced_batched_ok) {
    bestp.variant = DMUON_VARIANT_BATCHED;
    bestp.tile = 128;
    bestp.cost_ms = forced_batched_ms;
  }
  *plan = bestp;
  return DMUON_OK;
}


// Host I/O pipeline: matrices per chunk (about DMUON_IO_CHUNK_MB, default 16,
// MB of gradients, at least one matrix) and the 256-byte aligned stride of one
// staged gradient.
long long io_chunk_bytes() {
  static const long long v = [] {
    const char* b = getenv("DMUON_IO_CHUNK_MB");
    const long long mb = b ? atoll(b) : 16;
    return std::max(1LL, mb) << 20;
  }();
  return v;
}
int io_chunk(long long rows, long long cols, bool g_f32) {
  const long long bytes = rows * cols * (g_f32 ? 4 : 2);
  const long long n = io_chunk_bytes() / std::max(bytes, 1LL);
  return static_cast<int>(std::max(1LL, std::min(n, 65535LL)));
}
size_t io_stride(long long rows, long long cols, bool g_f32) {
  return align256(static_cast<size_t>(rows * cols * (g_f32 ? 4 : 2)));
}

// Host I/O copies: "dma" (one copy-engine transfer per matrix), "kernel"
// (copy_tables_kernel through the SMs, one launch per chunk) or "auto".
// A copy-engine transfer costs about 4 us however small it is, so for
// matrices up to kIoKernelMaxBytes the kernel is far faster (32 KB
// matrices: 0.8 ms against 4.5 ms for 16 MB each way); for large matrices
// the copy engines win, because SM copies compete with the GEMMs running
// beside them (2 MB matrices: 4.0 ms against 6.0 ms).  "auto" takes the
// kernel for groups of small matrices whose host buffers allow it.
// DMUON_IO_COPY overrides.
enum IoCopy { IO_AUTO = 0, IO_DMA = 1, IO_KERNEL = 2, IO_OUT_KERNEL = 3 };
constexpr long long kIoKernelMaxBytes = 256 << 10;
constexpr double kIoLinkGBs = 50.0;  // host link, GB/s per direction (PCIe 5 x16 measures about 56)
IoCopy io_copy_mode() {
  static const IoCopy v = [] {
    const char* e = getenv("DMUON_IO_COPY");
    if (e && strcmp(e, "dma") == 0) return IO_DMA;
    if (e && strcmp(e, "kernel") == 0) return IO_KERNEL;
    if (e && strcmp(e, "out-kernel") == 0) return IO_OUT_KERNEL;
    return IO_AUTO;
  }();
  return v;
}

// The device address of pinned host memory mapped into the current
// device's address space, or null (pageable or unknown memory).
void* mapped_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  return a.devicePointer;
}

// The shape groups of a call: the matrices whose iterate is m x n (m the
// smaller, n the larger dimension, whichever way each is stored), in order of
// first appearance, those stored m x n first (ntall stored n x m); per group
// the iterate's dtype (iter_f32), its geometry and its chunk (matrices per
// chain of launches: scratch within the workspace budget, and with host I/O
// about DMUON_IO_CHUNK_MB of gradients).  Pure host logic: run_step and
// dmuon_debug_groups share it.
std::vector<Group> make_groups(const int64_t* shapes, int count, bool f32, bool io, bool g_f32,
                               std::vector<Geo>* geos) {
  std::vector<Group> groups;
  std::map<std::pair<long long, long long>, int> gi;
  for (int i = 0; i < count; ++i) {
    const long long rr = shapes[2 * i], cc = shapes[2 * i + 1];
    auto key = std::make_pair(std::min(rr, cc), std::max(rr, cc));
    auto it = gi.find(key);
    if (it == gi.end()) {
      it = gi.emplace(key, static_cast<int>(groups.size())).first;
      groups.push_back(Group{key.first, key.second, {}, Plan{}, 0, 0});
    }
    groups[it->second].idx.push_back(i);
  }
  geos->assign(groups.size(), Geo{});
  for (size_t k = 0; k < groups.size(); ++k) {
    Group& gr = groups[k];
    auto tall = [&](int i) { return shapes[2 * i] > shapes[2 * i + 1]; };
    std::stable_partition(gr.idx.begin(), gr.idx.end(), [&](int i) { return !tall(i); });
    gr.ntall = static_cast<int>(std::count_if(gr.idx.begin(), gr.idx.end(), tall));
    gr.xf = iter_f32(f32, gr.rows);
    (*geos)[k] = make_geo(gr.rows, gr.cols, gr.xf);
    gr.chunk = chunk_size((*geos)[k], static_cast<int>(gr.idx.size()));
    if (io) gr.chunk = std::min(gr.chunk, io_chunk(gr.rows, gr.cols, g_f32));
  }
  return groups;
}

// The order in which a call issues its chunks.  Pure host logic: run_step
// and dmuon_debug_io_order share it.
struct IoGroup {
  int count, chunk;  // matrices, matrices per chunk
  double cost_ms;    // measured time of one chunk's computation (its plan's cost)
  double bytes;      // bytes one matrix moves over the host link, the larger direction
  bool sm_copy;      // its copies run through copy_tables_kernel
};
struct Piece {
  int k, c0, cnt;  // group, its first matrix, matrices
};
// Group by group, in `order`, each group in chunks.  With host I/O and every
// plan cached (io_cached):
//  - when one group is copy-bound (a wide Gram group moves more bytes than it
//    computes for) and another compute-bound (a square direct one), the
//    chunks of the groups are merged, each group's spread evenly over the
//    call (chunk i of a group of n chunks at (i + 1/2) / n): group by group,
//    the copy engines would idle through the compute-bound groups and the
//    SMs through the copy-bound ones.  A chunk's cost is compared with its
//    copies at a nominal host-link rate of kIoLinkGBs per direction.  When
//    every group is copy-bound the group order stays (merging measured
//    slower there).  Groups copied through copy_tables_kernel stay out of the
//    merge and follow the merged chunks, in group order: that kernel needs
//    SMs, so between two big chunks it would wait for a GEMM to finish and
//    hold up the copy stream behind it.
//  - a quarter of the first chunk (at least one matrix) becomes a piece of
//    its own, so the first computation starts after a short copy-in, and so
//    does a quarter of the last chunk, so the last copy-out follows a short
//    computation (the pipeline's fill and drain).  A piece runs its group's
//    plan.
std::vector<Piece> chunk_order(const std::vector<IoGroup>& gs, const std::vector<int>& order, bool io_cached,
                               bool* merged) {
  std::vector<Piece> seq;
  for (int k : order)
    for (int c0 = 0; c0 < gs[k].count; c0 += gs[k].chunk) seq.push_back({k, c0, std::min(gs[k].chunk, gs[k].count - c0)});
  if (merged) *merged = false;
  if (!io_cached || seq.empty()) return seq;
  bool compute_bound = false, copy_bound = false;
  for (const IoGroup& g : gs) {
    if (g.sm_copy) continue;
    (g.cost_ms > g.chunk * g.bytes / (kIoLinkGBs * 1e6) ? compute_bound : copy_bound) = true;
  }
  if (compute_bound && copy_bound) {
    auto key = [&](const Piece& e) {
      const IoGroup& g = gs[e.k];
      if (g.sm_copy) return std::make_pair(1, 0.0);
      const double n = static_cast<double>((g.count + g.chunk - 1) / g.chunk);
      return std::make_pair(0, (e.c0 / g.chunk + 0.5) / n);
    };
    std::stable_sort(seq.begin(), seq.end(), [&](const Piece& x, const Piece& y) { return key(x) < key(y); });
    if (merged) *merged = true;
  }
  auto split = [&](size_t i, bool head) {
    const Piece e = seq[i];
    if (e.cnt < 2) return;
    const int a = std::max(1, e.cnt / 4);
    const Piece x{e.k, e.c0, head ? a : e.cnt - a};
    const Piece y{e.k, e.c0 + x.cnt, e.cnt - x.cnt};
    seq[i] = x;
    seq.insert(seq.begin() + static_cast<long>(i) + 1, y);
  };
  split(seq.size() - 1, false);
  split(0, true);
  return seq;
}

int run_step(Request& r) {
  int rc = validate(r);
  if (rc || r.count == 0) return rc;
  DeviceCtx* cp = nullptr;
  rc = get_ctx(&cp);
  if (rc) return rc;
  DeviceCtx& c = *cp;
  std::lock_guard<std::mutex> lk(c.mu);
  if (*c.err_host) {
    *c.err_host = 0;
    return fail(DMUON_ERR_DEVICE_TIMEOUT, "a previous launch on this device timed out on a device-side wait");
  }
  const bool f32 = r.o.param_dtype == DMUON_F32;
  const bool g_f32 = r.o.grad_dtype == DMUON_F32;

  std::vector<Geo> geos;
  std::vector<Group> groups = make_groups(r.shapes, r.count, f32, r.grads_host, g_f32, &geos);
  // plans: cache lookup; misses are tuned on this call's data below
  std::vector<bool> miss(groups.size(), false);
  std::vector<size_t> needs(groups.size(), 0);
  size_t ws_need = 0;
  size_t stage_slot = 0;  // host I/O: bytes of one staging slot for gradients
  for (size_t k = 0; k < groups.size(); ++k) {
    Group& gr = groups[k];
    Key key{gr.rows, gr.cols, gr.xf ? 1 : 0, r.h.steps, gr.chunk};
    {
      std::lock_guard<std::mutex> lk2(g_cache_mu);
      auto it = g_cache.find(key);
      // a forced variant the shape cannot take (see resident_supported)
      // runs as planned for AUTO
      const bool forced_ok =
          r.o.variant != DMUON_VARIANT_BATCHED || resident_supported(gr.xf, geos[k].m, geos[k].n);
      const int want = forced_ok ? r.o.variant : DMUON_VARIANT_AUTO;
      if (it != g_cache.end() && (want == DMUON_VARIANT_AUTO || it->second.variant == want)) {
        gr.plan = it->second;
      } else {
        miss[k] = true;
      }
    }
    const int nblk = chunk_nblk(geos[k], gr.ntall < static_cast<int>(gr.idx.size()), gr.ntall > 0);
    Layout L = make_layout(geos[k], gr.chunk, nblk);
    size_t need = L.total;
    if (miss[k]) need += 2 * align256(static_cast<size_t>(gr.chunk) * geos[k].x_elems() * geos[k].esz) + 256;
    needs[k] = align256(need);
    if (r.grads_host) stage_slot = std::max(stage_slot, static_cast<size_t>(gr.chunk) * io_stride(gr.rows, gr.cols, g_f32));
  }
  // Scheduler: groups run in descending measured cost.  Once every plan is
  // cached, groups whose largest product does not fill the GPU (under two
  // waves of output tiles) are spread over side streams, longest first onto
  // the least loaded stream, so they overlap each other and the big groups;
  // each stream has its own scratch region.
  const bool any_miss = std::find(miss.begin(), miss.end(), true) != miss.end();
  std::vector<int> lane(groups.size(), 0);  // 0: the caller's stream; 1..kSide: side streams
  auto group_cost = [&](int k) {
    return groups[k].plan.cost_ms * static_cast<double>((groups[k].idx.size() + groups[k].chunk - 1) / groups[k].chunk);
  };
  if (!any_miss && !f32 && groups.size() >= 2 && !r.grads_host) {
    std::vector<int> small;
    for (size_t k = 0; k < groups.size(); ++k) {
      const Geo& g = geos[k];
      const int tl = groups[k].plan.tile;
      const long long tiles = tc_gemm_tiles(g.m, g.n, groups[k].chunk, tl, false);
      const long long wave = tl >= 512 ? c.num_sms / 2 : c.num_sms;
      if (!groups[k].xf && groups[k].idx.size() <= static_cast<size_t>(groups[k].chunk) && tiles < 2 * wave)
        small.push_back(static_cast<int>(k));
    }
    std::stable_sort(small.begin(), small.end(), [&](int x, int y) { return group_cost(x) > group_cost(y); });
    double load[DeviceCtx::kSide] = {0, 0, 0};
    for (int k : small) {
      int best = 0;
      for (int i = 1; i < DeviceCtx::kSide; ++i)
        if (load[i] < load[best]) best = i;
      lane[k] = best + 1;
      load[best] += group_cost(k);
    }
  }
  // Host I/O with every plan cached: consecutive chunks alternate between
  // the caller's stream and side stream 1 (two scratch regions), so one
  // chunk's kernels fill the SMs the other's last wave leaves idle while the
  // copy streams run ahead through kIoSlots staging slots.
  bool io_two = r.grads_host && !any_miss;
  std::vector<size_t> region_need(DeviceCtx::kSide + 1, 0);
  std::vector<size_t> region_off(DeviceCtx::kSide + 1, 0);
  auto layout_regions = [&] {
    std::fill(region_need.begin(), region_need.end(), 0);
    for (size_t k = 0; k < groups.size(); ++k) region_need[lane[k]] = std::max(region_need[lane[k]], needs[k]);
    if (io_two) region_need[1] = std::max(region_need[1], region_need[0]);
    for (int i = 1; i <= DeviceCtx::kSide; ++i) region_off[i] = region_off[i - 1] + region_need[i - 1];
    ws_need = region_off[DeviceCtx::kSide] + region_need[DeviceCtx::kSide];
  };
  layout_regions();
  // pointer tables: G, B, W, O; with host I/O also the mapped host
  // gradients and the mapped host parameter outputs
  const int ntab = r.grads_host ? 6 : 4;
  const size_t tables_bytes = align256(ntab * sizeof(void*) * static_cast<size_t>(r.count));
  const int io_slots = r.grads_host ? DeviceCtx::kIoSlots : 0;
  auto ext_fits = [&] {
    return align256(ws_need) + static_cast<size_t>(io_slots) * align256(stage_slot) + tables_bytes <= g_ext_bytes;
  };
  if (g_ext_ptr && !ext_fits()) {
    std::fill(lane.begin(), lane.end(), 0);  // a caller buffer too small for side streams: one stream
    io_two = false;
    layout_regions();
  }
  // device pointer tables: 4 arrays of count pointers, after the chunk scratch
  const size_t stage_off = align256(ws_need);  // host I/O: the gradient staging slots
  const size_t tables_off = stage_off + static_cast<size_t>(io_slots) * align256(stage_slot);
  const size_t total_ws = tables_off + tables_bytes;
  rc = ensure_ws(c, total_ws, r.s);
  if (rc) return rc;

  // order GPU work after the previous call's (it may be on another stream)
  if (c.has_last) CUDA_TRY(cudaStreamWaitEvent(r.s, c.last_done, 0));

  // issue order: tuned groups first (they synchronise), then by cost
  std::vector<int> order(groups.size());
  for (size_t k = 0; k < order.size(); ++k) order[k] = static_cast<int>(k);
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) {
    if (miss[x] != miss[y]) return static_cast<bool>(miss[x]);
    return group_cost(x) > group_cost(y);
  });
  std::vector<Piece> seq;  // the chunks in issue order (chunk_order), once the copy kinds are known

  // pointer tables, grouped: for group k, its matrices are contiguous.  With
  // host gradients the G entries point at the staging slot of the matrix's
  // chunk (chunks take the kIoSlots slots in turn, in issue order).
  uint8_t* ws = static_cast<uint8_t*>(c.ws);
  std::vector<void*> host(ntab * static_cast<size_t>(r.count));
  std::vector<char> kin(groups.size(), 0), kout(groups.size(), 0);  // host I/O through copy_tables_kernel
  std::vector<int> gstart(groups.size());
  {
    int pos = 0;
    for (size_t k = 0; k < groups.size(); ++k) {
      gstart[k] = pos;
      for (int i : groups[k].idx) {
        host[pos] = const_cast<void*>(r.grads[i]);
        host[r.count + pos] = r.moms[i];
        host[2 * r.count + pos] = r.params ? r.params[i] : nullptr;
        host[3 * r.count + pos] = r.out ? static_cast<void*>(r.out[i]) : nullptr;
        ++pos;
      }
    }
    const IoCopy mode = io_copy_mode();
    if (r.grads_host && mode != IO_DMA) {
      for (size_t k = 0; k < groups.size(); ++k) {
        const Group& gr = groups[k];
        const long long gbytes = gr.rows * gr.cols * (g_f32 ? 4 : 2);
        const long long wbytes = gr.rows * gr.cols * (f32 ? 4 : 2);
        const bool small = std::max(gbytes, wbytes) <= kIoKernelMaxBytes;
        bool ok_in = gbytes % 16 == 0 && (mode == IO_KERNEL || small);
        bool ok_out = r.params_host && wbytes % 16 == 0 && (mode != IO_AUTO || small);
        for (size_t q = 0; q < gr.idx.size() && (ok_in || ok_out); ++q) {
          const int i = gr.idx[q];
          void* hs = ok_in ? mapped_host(r.grads[i]) : nullptr;
          void* hd = ok_out ? mapped_host(r.params_host[i]) : nullptr;
          ok_in = ok_in && hs && aligned16(hs);
          ok_out = ok_out && hd && aligned16(hd) && aligned16(r.params[i]);
          host[4 * r.count + gstart[k] + q] = hs;
          host[5 * r.count + gstart[k] + q] = hd;
        }
        kin[k] = ok_in ? 1 : 0;
        kout[k] = ok_out ? 1 : 0;
      }
    }
    std::vector<IoGroup> io(groups.size());
    for (size_t k = 0; k < groups.size(); ++k) {
      const Group& gr = groups[k];
      io[k] = {static_cast<int>(gr.idx.size()), gr.chunk, gr.plan.cost_ms,
               static_cast<double>(gr.rows) * gr.cols * std::max(g_f32 ? 4 : 2, r.params_host ? (f32 ? 4 : 2) : 0),
               kin[k] || kout[k]};
    }
    bool merged = false;
    seq = chunk_order(io, order, r.grads_host && !any_miss, &merged);
    if (merged && trace_on()) fprintf(stderr, "[dmuon] host I/O: chunks merged across shape groups\n");
    if (r.grads_host) {
      for (size_t j = 0; j < seq.size(); ++j) {
        const Piece& e = seq[j];
        const Group& gr = groups[e.k];
        const size_t stride = io_stride(gr.rows, gr.cols, g_f32);
        for (int q = 0; q < e.cnt; ++q)
          host[gstart[e.k] + e.c0 + q] = ws + stage_off + (j % io_slots) * align256(stage_slot) + q * stride;
      }
    }
  }
  void** dtab = reinterpret_cast<void**>(ws + tables_off);
  rc = upload_tables(c, host, dtab, r.s);
  if (rc) return rc;
  if (r.grads_host) {  // the copy streams start after everything before this call
    CUDA_TRY(cudaEventRecord(c.fork_ev, r.s));
    CUDA_TRY(cudaStreamWaitEvent(c.cin, c.fork_ev, 0));
    CUDA_TRY(cudaStreamWaitEvent(c.cout, c.fork_ev, 0));
  }
  int io_j = 0;  // host I/O: chunk counter in issue order
  bool side_used[DeviceCtx::kSide] = {false, false, false};
  for (size_t k = 0; k < groups.size(); ++k)
    if (lane[k] > 0) side_used[lane[k] - 1] = true;
  if (io_two) side_used[0] = true;
  const bool forked = side_used[0] || side_used[1] || side_used[2];
  if (forked) {
    CUDA_TRY(cudaEventRecord(c.fork_ev, r.s));
    for (int i = 0; i < DeviceCtx::kSide; ++i)
      if (side_used[i]) CUDA_TRY(cudaStreamWaitEvent(c.side[i], c.fork_ev, 0));
  }

  for (const Piece& e : seq) {
    const int k = e.k, c0 = e.c0;
    Group& gr = groups[k];
    const Geo& g = geos[k];
    const int total = static_cast<int>(gr.idx.size());
    {
      const int ln = io_two ? (io_j & 1) : lane[k];
      const cudaStream_t gs = ln == 0 ? r.s : c.side[ln - 1];
      Chunk ch;
      ch.g = &g;
      ch.cnt = e.cnt;
      ch.nwide = std::min(std::max(total - gr.ntall - c0, 0), ch.cnt);
      ch.base = ws + region_off[ln];
      ch.nblk = chunk_nblk(g, gr.ntall < total, gr.ntall > 0);
      ch.L = make_layout(g, gr.chunk, ch.nblk);
      const int p = gstart[k] + c0;
      ch.Gt = dtab + p;
      ch.Bt = dtab + r.count + p;
      ch.Wt = dtab + 2 * r.count + p;
      ch.Ot = reinterpret_cast<float* const*>(dtab + 3 * r.count + p);
      ch.aligned = 1;
      for (int q = 0; q < ch.cnt; ++q) {
        const int i = gr.idx[c0 + q];
        if (!aligned16(r.grads[i]) || !aligned16(r.moms[i])) ch.aligned = 0;
      }
      const int slot = r.grads_host ? io_j % io_slots : 0;
      if (r.grads_host) {
        // copy-in: this chunk's gradients into its staging slot, once the
        // chunk io_slots back has consumed that slot
        if (io_j >= io_slots) CUDA_TRY(cudaStreamWaitEvent(c.cin, c.g_free[slot], 0));
        const size_t bytes = static_cast<size_t>(g.rows) * g.cols * (g_f32 ? 4 : 2);
        if (kin[k]) {
          CUDA_TRY(launch_k(KIND_OTHER, 0.0, 0.0, c.cin, [&] {
            return launch_copy_tables(dtab + 4 * r.count + p, dtab + p, static_cast<long long>(bytes), ch.cnt,
                                      c.num_sms, c.cin);
          }));
        } else {
          for (int q = 0; q < ch.cnt; ++q)
            CUDA_TRY(cudaMemcpyAsync(host[p + q], r.grads[gr.idx[c0 + q]], bytes, cudaMemcpyHostToDevice, c.cin));
        }
        CUDA_TRY(cudaEventRecord(c.g_ready[slot], c.cin));
        CUDA_TRY(cudaStreamWaitEvent(gs, c.g_ready[slot], 0));
      }
      rc = run_momentum(ch, gr.xf, g_f32, r.h, gs);
      if (rc) return rc;
      if (r.grads_host) CUDA_TRY(cudaEventRecord(c.g_free[slot], gs));
      if (miss[k] && c0 == 0) {
        Plan pl;
        rc = autotune(c, ch, gr.xf, r.h, r.o.variant, &pl, gs);
        if (rc) return rc;
        gr.plan = pl;
        Key key{gr.rows, gr.cols, gr.xf ? 1 : 0, r.h.steps, gr.chunk};
        std::lock_guard<std::mutex> lk2(g_cache_mu);
        if (r.o.variant == DMUON_VARIANT_AUTO || !g_cache.count(key)) g_cache[key] = pl;
      }
      rc = run_ns(c, ch, gr.xf, gr.plan.variant, gr.plan.tile, r.h, final_epilogue(r, g, ch, f32, false),
                  final_epilogue(r, g, ch, f32, true), ch.cnt, gs);
      if (rc) return rc;
      if (r.grads_host) {
        if (r.params_host) {  // copy-out: the chunk's updated parameters
          CUDA_TRY(cudaEventRecord(c.w_done[slot], gs));
          CUDA_TRY(cudaStreamWaitEvent(c.cout, c.w_done[slot], 0));
          const size_t bytes = static_cast<size_t>(g.rows) * g.cols * (f32 ? 4 : 2);
          if (kout[k]) {
            CUDA_TRY(launch_k(KIND_OTHER, 0.0, 0.0, c.cout, [&] {
              return launch_copy_tables(dtab + 2 * r.count + p, dtab + 5 * r.count + p,
                                        static_cast<long long>(bytes), ch.cnt, c.num_sms, c.cout);
            }));
          } else {
            for (int q = 0; q < ch.cnt; ++q) {
              const int i = gr.idx[c0 + q];
              CUDA_TRY(cudaMemcpyAsync(r.params_host[i], r.params[i], bytes, cudaMemcpyDeviceToHost, c.cout));
            }
          }
        }
        ++io_j;
      }
    }
    if (trace_on() && c0 + e.cnt >= total)
      fprintf(stderr, "[dmuon] group %lldx%lld x%d (%d stored transposed): variant=%d tile=%d chunk=%d cost=%.3f ms stream=%d\n",
              gr.rows, gr.cols, total, gr.ntall, gr.plan.variant, gr.plan.tile, gr.chunk, gr.plan.cost_ms, lane[k]);
  }
  if (forked) {
    for (int i = 0; i < DeviceCtx::kSide; ++i)
      if (side_used[i]) {
        CUDA_TRY(cudaEventRecord(c.side_done[i], c.side[i]));
        CUDA_TRY(cudaStreamWaitEvent(r.s, c.side_done[i], 0));
      }
  }
  if (r.grads_host) {  // join the copy streams back into the caller's stream
    CUDA_TRY(cudaEventRecord(c.io_done, c.cout));
    CUDA_TRY(cudaStreamWaitEvent(r.s, c.io_done, 0));
    CUDA_TRY(cudaEventRecord(c.io_done, c.cin));
    CUDA_TRY(cudaStreamWaitEvent(r.s, c.io_done, 0));
  }
  CUDA_TRY(cudaEventRecord(c.last_done, r.s));
  c.has_last = true;
  return DMUON_OK;
}

Hyper hyper_from(float lr, float wd, float mu, int steps, const dmuon_options& o) {
  Hyper h;
  h.mu = mu;
  h.lr = lr;
  h.wd = wd;
  h.eps = o.eps;
  h.a = o.ns_a;
  h.b = o.ns_b;
  h.c = o.ns_c;
  h.steps = steps;
  h.nesterov = o.nesterov;
  return h;
}

}  // namespace

// ------------------------------------------------------------------ no-alloc entry point
// Scratch of dmuon_compute_update_noalloc: a fixed array in the library's own
// device image, so that entry point never allocates.  Every GPU that loads
// the library holds these 64 MiB until the process exits.  Host code must not
// use the symbol's name as an address; it asks the runtime for the device
// address once per device (static_scratch below).
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device; looked up with
// cudaGetSymbolAddress on the first call per device (with that device current).
int static_scratch(void** out, int* device) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return fail(DMUON_ERR_INVALID, "device ordinal %d not supported", dev);
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return fail(DMUON_ERR_CUDA, "cudaGetSymbolAddress(static scratch) on device %d: %s", dev, cudaGetErrorString(e));
    g_static_addr[dev] = p;
  }
  *out = g_static_addr[dev];
  *device = dev;
  return DMUON_OK;
}

}  // namespace
}  // namespace dmuon

using namespace dmuon;

extern "C" {

void dmuon_options_init(dmuon_options* o) {
  if (!o) return;
  o->param_dtype = DMUON_BF16;
  o->grad_dtype = DMUON_BF16;
  o->mom_dtype = DMUON_F32;
  o->eps = 1e-7f;
  o->nesterov = 1;
  o->variant = DMUON_VARIANT_AUTO;
  o->ns_a = 3.4445f;
  o->ns_b = -4.7750f;
  o->ns_c = 2.0315f;
}

int dmuon_step_ex(void* const* params, const void* const* grads, void* const* momenta, const int64_t* shapes,
                  int count, float lr, float wd, float mu, int ns_steps, const dmuon_options* opts, void* stream) {
  t_err.clear();
  dmuon_options o;
  dmuon_options_init(&o);
  if (opts) o = *opts;
  if (!params && count > 0) return fail(DMUON_ERR_INVALID, "params is NULL");
  Request r{params, grads, momenta, nullptr, shapes, count, hyper_from(lr, wd, mu, ns_steps, o), o,
            static_cast<cudaStream_t>(stream)};
  return run_step(r);
}

int dmuon_step(void* const* params, const void* const* grads, void* const* momenta, const int64_t* shapes, int count,
               float lr, float wd, float mu, int ns_steps, void* stream) {
  return dmuon_step_ex(params, grads, momenta, shapes, count, lr, wd, mu, ns_steps, nullptr, stream);
}

int dmuon_step_host_io(void* const* params, const void* const* grads_host, void* const* momenta,
                       void* const* params_host_out, const int64_t* shapes, int count, float lr, float wd, float mu,
                       int ns_steps, const dmuon_options* opts, void* stream) {
  t_err.clear();
  dmuon_options o;
  dmuon_options_init(&o);
  if (opts) o = *opts;
  if (!params && count > 0) return fail(DMUON_ERR_INVALID, "params is NULL");
  Request r{params, grads_host, momenta, nullptr, shapes, count, hyper_from(lr, wd, mu, ns_steps, o), o,
            static_cast<cudaStream_t>(stream)};
  r.grads_host = true;
  r.params_host = params_host_out;
  return run_step(r);
}

int dmuon_compute_update(const void* const* grads, void* const* momenta, const int64_t* shapes, int count, float mu,
                         int ns_steps, const dmuon_options* opts, float* const* out, void* stream) {
  t_err.clear();
  dmuon_options o;
  dmuon_options_init(&o);
  if (opts) o = *opts;
  if (!out && count > 0) return fail(DMUON_ERR_INVALID, "out is NULL");
  Request r{nullptr, grads, momenta, out, shapes, count, hyper_from(0.f, 0.f, mu, ns_steps, o), o,
            static_cast<cudaStream_t>(stream)};
  return run_step(r);
}

int dmuon_compute_update_noalloc(const void* grad, void* momentum, int64_t rows, int64_t cols, float mu,
                                 int ns_steps, const dmuon_options* opts, float* out, void* stream) {
  t_err.clear();
  dmuon_options o;
  dmuon_options_init(&o);
  if (opts) o = *opts;
  if (!grad || !momentum || !out) return fail(DMUON_ERR_INVALID, "null pointer");
  const int64_t shape[2] = {rows, cols};
  void* gp = const_cast<void*>(grad);
  float* op = out;
  Request r{nullptr, reinterpret_cast<const void* const*>(&gp), &momentum, &op, shape, 1,
            hyper_from(0.f, 0.f, mu, ns_steps, o), o, static_cast<cudaStream_t>(stream)};
  int rc = validate(r);
  if (rc) return rc;
  const bool f32 = o.param_dtype == DMUON_F32;
  const bool xf = iter_f32(f32, std::min(rows, cols));
  const bool tall = rows > cols;
  const Geo g = make_geo(std::min(rows, cols), std::max(rows, cols), xf);  // the iterate, m x n
  // plan: the resident kernel when it is asked for and the shape fits it;
  // else the plan the autotuner cached for this shape (count 1), else the
  // direct form (a forced variant the shape cannot take runs as AUTO)
  Plan plan;
  if (o.variant == DMUON_VARIANT_BATCHED && resident_supported(xf, g.m, g.n)) {
    plan.variant = DMUON_VARIANT_BATCHED;
    plan.tile = 128;
  } else {
    const int want = o.variant == DMUON_VARIANT_BATCHED ? DMUON_VARIANT_AUTO : o.variant;
    if (want == DMUON_VARIANT_DIRECT || want == DMUON_VARIANT_GRAM) plan.variant = want;
    std::lock_guard<std::mutex> lk(g_cache_mu);
    auto it = g_cache.find(Key{g.m, g.n, xf ? 1 : 0, ns_steps, 1});
    if (it != g_cache.end() && (want == DMUON_VARIANT_AUTO || it->second.variant == want)) plan = it->second;
  }
  void* base = nullptr;
  int dev = 0;
  rc = static_scratch(&base, &dev);
  if (rc) return rc;
  int sms = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int nblk = chunk_nblk(g, !tall, tall);
  const Layout L = make_layout(g, 1, nblk);
  const size_t header = 256;  // 4 pointer slots and the device error word
  const size_t need = header + L.total;
  if (need > kStaticScratchBytes)
    return fail(DMUON_ERR_INVALID,
                "a %lld x %lld %s matrix needs %zu bytes of scratch; dmuon_compute_update_noalloc has %zu",
                (long long)rows, (long long)cols, f32 ? "fp32" : "bf16", need, kStaticScratchBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* sb = static_cast<uint8_t*>(base);
  int* dev_err = reinterpret_cast<int*>(sb + 64);
  // A bounded device wait that gave up in an earlier call left its code in
  // the error word, which no call clears unread.  The word is read here
  // (4 bytes on the per-thread stream, which does not wait for `stream`),
  // except while `stream` is being captured; a code found is reported now,
  // and the word cleared, before any launch.
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  CUDA_TRY(cudaStreamIsCapturing(s, &cap));
  if (cap == cudaStreamCaptureStatusNone) {
    int word = 0;
    CUDA_TRY(cudaMemcpyAsync(&word, dev_err, sizeof(int), cudaMemcpyDeviceToHost, cudaStreamPerThread));
    CUDA_TRY(cudaStreamSynchronize(cudaStreamPerThread));
    if (word != 0) {
      CUDA_TRY(cudaMemsetAsync(dev_err, 0, sizeof(int), s));
      return fail(DMUON_ERR_DEVICE_TIMEOUT, "a device-side wait of an earlier dmuon_compute_update_noalloc call timed out");
    }
  }
  // pointer table (G, B, W, O) written on the device from kernel arguments
  void** dtab = reinterpret_cast<void**>(sb);
  cudaError_t e = launch_k(KIND_OTHER, 0.0, 0.0, s, [&] { return launch_store_ptrs(dtab, gp, momentum, nullptr, out, s); });
  if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "pointer table: %s", cudaGetErrorString(e));
  DeviceCtx c;  // launch parameters only: nothing is allocated for it
  c.device = dev;
  c.num_sms = sms;
  c.err_dev = dev_err;
  Chunk ch;
  ch.g = &g;
  ch.cnt = 1;
  ch.nwide = tall ? 0 : 1;
  ch.base = sb + header;
  ch.L = L;
  ch.Gt = dtab;
  ch.Bt = dtab + 1;
  ch.Wt = dtab + 2;
  ch.Ot = reinterpret_cast<float* const*>(dtab + 3);
  ch.nblk = nblk;
  ch.aligned = aligned16(grad) && aligned16(momentum);
  rc = run_momentum(ch, xf, o.grad_dtype == DMUON_F32, r.h, s);
  if (rc) return rc;
  Epilogue fin{};
  fin.mode = EPI_OUT;
  fin.Out = ch.Ot;
  fin.transposed = tall ? 1 : 0;
  fin.ldw = tall ? g.m : g.n;
  fin.w_f32 = f32;
  rc = run_ns(c, ch, xf, plan.variant, plan.tile, r.h, fin, fin, 1, s);
  if (rc) return rc;
  if (fault_wait()) {  // DMUON_FAULT=wait: a bounded wait that runs out, as a stalled pipeline would
    e = launch_wait_selftest(dev_err, 20000000ull, s);
    if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "injected wait: %s", cudaGetErrorString(e));
  }
  return DMUON_OK;
}

int dmuon_gemm_bf16(const void* A, int64_t lda, int64_t sa, const void* B, int64_t ldb, int64_t sb, int b_kmajor,
                    const void* C, int64_t ldc, int64_t sc, void* D, int64_t ldd, int64_t sd, int M, int N, int K,
                    int batch, float alpha, float beta, int tile, int sym, void* stream) {
  t_err.clear();
  if (!A || !B || !D) return fail(DMUON_ERR_INVALID, "null operand");
  if (M <= 0 || N <= 0 || K <= 0 || batch <= 0) return fail(DMUON_ERR_INVALID, "bad GEMM size");
  if ((lda | ldb | ldd | sa | sb | sd) & 7 || (C && ((ldc | sc) & 7)))
    return fail(DMUON_ERR_INVALID, "leading dims / batch strides must be multiples of 8");
  if (lda < K || ldd < N || (b_kmajor ? ldb < K : ldb < N) || (C && ldc < N))
    return fail(DMUON_ERR_INVALID, "leading dim smaller than the row");
  if (tile != 0 && tile != 128 && tile != 256 && tile != 512) return fail(DMUON_ERR_INVALID, "tile must be 0, 128, 256 or 512");
  if (sym && M != N) return fail(DMUON_ERR_INVALID, "sym needs M == N");
  DeviceCtx* cp = nullptr;
  int rc = get_ctx(&cp);
  if (rc) return rc;
  Epilogue e{};
  e.mode = EPI_STORE;
  e.alpha = alpha;
  e.beta = beta;
  e.C = C;
  e.ldc = ldc;
  e.sc = sc;
  e.D = D;
  e.ldd = ldd;
  e.sd = sd;
  const int tl = tile == 0 ? 256 : tile;
  TcGemm t{A, lda, sa, B, ldb, sb, b_kmajor != 0, M, N, K, batch, tl, sym != 0, e};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const double frac = static_cast<double>(tc_gemm_tiles(M, N, batch, tl, sym != 0)) / tc_gemm_tiles(M, N, batch, tl, false);
  cudaError_t err = launch_k(KIND_TC_GEMM, 2.0 * M * N * static_cast<double>(K) * batch * frac, 0.0, s,
                             [&] { return launch_tc_gemm(t, s, cp->err_dev, cp->num_sms); });
  if (err != cudaSuccess) return fail(DMUON_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(err));
  return DMUON_OK;
}

int dmuon_adamw_step(void* const* params, const void* const* grads, float* const* exp_avg, float* const* exp_avg_sq,
                     const int64_t* numels, int count, float lr, float beta1, float beta2, float eps, float wd,
                     int64_t step, int dtype, void* stream) {
  t_err.clear();
  if (count < 0) return fail(DMUON_ERR_INVALID, "count < 0");
  if (count == 0) return DMUON_OK;
  if (!params || !grads || !exp_avg || !exp_avg_sq || !numels) return fail(DMUON_ERR_INVALID, "null pointer array");
  if (dtype != DMUON_BF16 && dtype != DMUON_F32) return fail(DMUON_ERR_DTYPE, "dtype must be BF16 or F32");
  if (step < 1) return fail(DMUON_ERR_INVALID, "step counts from 1 (got %lld)", static_cast<long long>(step));
  const float hs[] = {lr, beta1, beta2, eps, wd};
  for (float v : hs)
    if (!std::isfinite(v)) return fail(DMUON_ERR_INVALID, "non-finite hyperparameter");
  if (beta1 < 0.f || beta1 >= 1.f || beta2 < 0.f || beta2 >= 1.f || eps < 0.f)
    return fail(DMUON_ERR_INVALID, "betas must be in [0, 1) and eps >= 0");
  // live tensors (numel > 0) and their chunk offsets
  std::vector<int> live;
  std::vector<long long> starts;
  long long chunks = 0;
  bool aligned = true;
  for (int i = 0; i < count; ++i) {
    if (numels[i] < 0) return fail(DMUON_ERR_INVALID, "tensor %d has numel %lld", i, static_cast<long long>(numels[i]));
    if (numels[i] == 0) continue;
    if (!params[i] || !grads[i] || !exp_avg[i] || !exp_avg_sq[i]) return fail(DMUON_ERR_INVALID, "null pointer for tensor %d", i);
    aligned = aligned && aligned16(params[i]) && aligned16(grads[i]) && aligned16(exp_avg[i]) && aligned16(exp_avg_sq[i]);
    live.push_back(i);
    starts.push_back(chunks);
    chunks += adamw_chunks(numels[i]);
  }
  const int n = static_cast<int>(live.size());
  if (n == 0) return DMUON_OK;
  if (chunks > 0x7fffffffLL) return fail(DMUON_ERR_INVALID, "too many elements for one launch");
  DeviceCtx* cp = nullptr;
  int rc = get_ctx(&cp);
  if (rc) return rc;
  DeviceCtx& c = *cp;
  std::lock_guard<std::mutex> lk(c.mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // tables: P, G, M, V pointers, chunk starts, numels (8 bytes each)
  std::vector<void*> host(6 * static_cast<size_t>(n));
  for (int k = 0; k < n; ++k) {
    const int i = live[k];
    host[k] = params[i];
    host[n + k] = const_cast<void*>(grads[i]);
    host[2 * n + k] = exp_avg[i];
    host[3 * n + k] = exp_avg_sq[i];
    host[4 * n + k] = reinterpret_cast<void*>(static_cast<intptr_t>(starts[k]));
    host[5 * n + k] = reinterpret_cast<void*>(static_cast<intptr_t>(numels[i]));
  }
  const size_t bytes = host.size() * sizeof(void*);
  if (c.adam_used) CUDA_TRY(cudaStreamWaitEvent(s, c.adam_done, 0));  // the previous launch has read the tables
  if (bytes > c.adam_cap) {
    if (fault_alloc()) return fail(DMUON_ERR_OOM, "injected allocation failure (DMUON_FAULT=alloc)");
    if (c.adam_tab) {
      CUDA_TRY(cudaStreamSynchronize(s));
      CUDA_TRY(cudaFree(c.adam_tab));
      c.adam_tab = nullptr;
      c.adam_cap = 0;
    }
    const size_t cap = std::max<size_t>(bytes, 64 << 10);
    if (cudaMalloc(&c.adam_tab, cap) != cudaSuccess) {
      cudaGetLastError();
      return fail(DMUON_ERR_OOM, "AdamW tables: cannot allocate %zu bytes", cap);
    }
    c.adam_cap = cap;
  }
  rc = upload_tables(c, host, c.adam_tab, s);
  if (rc) return rc;
  void** tab = static_cast<void**>(c.adam_tab);
  AdamwArgs a{};
  a.P = tab;
  a.G = tab + n;
  a.M = reinterpret_cast<float* const*>(tab + 2 * n);
  a.V = reinterpret_cast<float* const*>(tab + 3 * n);
  a.chunk_start = reinterpret_cast<const long long*>(tab + 4 * n);
  a.numel = reinterpret_cast<const long long*>(tab + 5 * n);
  a.count = n;
  a.p_f32 = dtype == DMUON_F32 ? 1 : 0;
  a.aligned = aligned ? 1 : 0;
  a.lr = lr;
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.eps = eps;
  a.omb1 = static_cast<float>(1.0 - static_cast<double>(beta1));
  a.omb2 = static_cast<float>(1.0 - static_cast<double>(beta2));
  a.decay = static_cast<float>(1.0 - static_cast<double>(lr) * static_cast<double>(wd));
  a.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step)));
  a.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step)));
  if (!(a.bc1 > 0.f) || !(a.bc2 > 0.f)) return fail(DMUON_ERR_INVALID, "bias correction 1 - beta^t is not positive");
  long long elems = 0;
  for (int k = 0; k < n; ++k) elems += numels[live[k]];
  const double ebytes = static_cast<double>(elems) * (dtype == DMUON_F32 ? 32.0 : 22.0);
  cudaError_t e = launch_k(KIND_EW, 0.0, ebytes, s, [&] { return launch_adamw(a, chunks, s); });
  if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "AdamW kernel: %s", cudaGetErrorString(e));
  CUDA_TRY(cudaEventRecord(c.adam_done, s));
  c.adam_used = true;
  return DMUON_OK;
}

int dmuon_selftest_wait(int limit_ms, void* stream) {
  t_err.clear();
  if (limit_ms < 1 || limit_ms > 2000) return fail(DMUON_ERR_INVALID, "limit_ms must be in [1, 2000]");
  DeviceCtx* cp = nullptr;
  int rc = get_ctx(&cp);
  if (rc) return rc;
  std::lock_guard<std::mutex> lk(cp->mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  *cp->err_host = 0;
  cudaError_t e = launch_wait_selftest(cp->err_dev, static_cast<unsigned long long>(limit_ms) * 1000000ull, s);
  if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  CUDA_TRY(cudaStreamSynchronize(s));
  const int word = *cp->err_host;
  *cp->err_host = 0;  // reported here: the next call starts clean
  if (word == DMUON_ERR_DEVICE_TIMEOUT)
    return fail(DMUON_ERR_DEVICE_TIMEOUT, "device wait gave up after %d ms (expected by the self-test)", limit_ms);
  return DMUON_OK;
}

int dmuon_cache_save(const char* path) {
  t_err.clear();
  if (!path) return fail(DMUON_ERR_INVALID, "null path");
  DeviceCtx* cp = nullptr;
  int rc = get_ctx(&cp);
  if (rc) return rc;
  FILE* f = fopen(path, "w");
  if (!f) return fail(DMUON_ERR_INVALID, "cannot open %s", path);
  std::string gpu = cp->name;
  for (char& ch : gpu)
    if (ch == ' ') ch = '_';
  fprintf(f, "dmuon-cache %d %s %d\n", DMUON_VERSION, gpu.c_str(), cp->num_sms);
  std::lock_guard<std::mutex> lk(g_cache_mu);
  for (auto& kv : g_cache)
    fprintf(f, "%lld %lld %d %d %d %d %d %.6f\n", kv.first.rows, kv.first.cols, kv.first.f32, kv.first.steps,
            kv.first.cnt, kv.second.variant, kv.second.tile, kv.second.cost_ms);
  fclose(f);
  return DMUON_OK;
}

int dmuon_cache_load(const char* path) {
  t_err.clear();
  if (!path) return fail(DMUON_ERR_INVALID, "null path");
  DeviceCtx* cp = nullptr;
  int rc = get_ctx(&cp);
  if (rc) return rc;
  FILE* f = fopen(path, "r");
  if (!f) return fail(DMUON_ERR_INVALID, "cannot open %s", path);
  int ver = 0, sms = 0;
  char gpu[256] = {0};
  if (fscanf(f, "dmuon-cache %d %255s %d", &ver, gpu, &sms) != 3) {
    fclose(f);
    return fail(DMUON_ERR_INVALID, "%s: not a dmuon cache file", path);
  }
  std::string mine = cp->name;
  for (char& ch : mine)
    if (ch == ' ') ch = '_';
  if (ver != DMUON_VERSION || mine != gpu || sms != cp->num_sms) {
    fclose(f);
    return fail(DMUON_ERR_INVALID, "%s was tuned for %s (%d SMs, v%d), not this GPU", path, gpu, sms, ver);
  }
  std::map<Key, Plan> loaded;
  long long rr, cc;
  int f32, steps, cnt, var, tile;
  double cost;
  while (fscanf(f, "%lld %lld %d %d %d %d %d %lf", &rr, &cc, &f32, &steps, &cnt, &var, &tile, &cost) == 8) {
    if (rr <= 0 || cc <= 0 || cnt <= 0 || var < 1 || var > 3 || (tile != 128 && tile != 256 && tile != 512) ||
        rr > cc || rr > INT32_MAX || cc > INT32_MAX ||
        (var == DMUON_VARIANT_BATCHED && !resident_supported(f32 != 0, static_cast<int>(rr), static_cast<int>(cc)))) {
      fclose(f);
      return fail(DMUON_ERR_INVALID, "%s: malformed entry", path);
    }
    Plan p;
    p.variant = var;
    p.tile = tile;
    p.cost_ms = cost;
    loaded[Key{rr, cc, f32, steps, cnt}] = p;
  }
  fclose(f);
  std::lock_guard<std::mutex> lk(g_cache_mu);
  for (auto& kv : loaded) g_cache[kv.first] = kv.second;
  return DMUON_OK;
}

void dmuon_cache_clear(void) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  g_cache.clear();
}

int dmuon_cache_size(void) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  return static_cast<int>(g_cache.size());
}

int dmuon_cache_entry(int i, char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_cache_mu);
  if (i < 0 || i >= static_cast<int>(g_cache.size()) || !buf || len == 0)
    return fail(DMUON_ERR_INVALID, "bad cache index");
  auto it = g_cache.begin();
  std::advance(it, i);
  snprintf(buf, len, "%lld %lld %s %d %s %d %d %.4f", it->first.rows, it->first.cols, it->first.f32 ? "f32" : "bf16",
           it->first.steps, it->second.variant == DMUON_VARIANT_GRAM ? "gram" : (it->second.variant == DMUON_VARIANT_BATCHED ? "batched" : "direct"),
           it->second.tile, it->first.cnt,
           it->second.cost_ms);
  return DMUON_OK;
}

int dmuon_set_workspace(void* dev_ptr, size_t bytes) {
  t_err.clear();
  if (dev_ptr && (reinterpret_cast<uintptr_t>(dev_ptr) & 255))
    return fail(DMUON_ERR_INVALID, "workspace must be 256-byte aligned");
  g_ext_ptr = bytes ? dev_ptr : nullptr;
  g_ext_bytes = dev_ptr ? bytes : 0;
  return DMUON_OK;
}

int dmuon_workspace_size(const int64_t* shapes, int count, int param_dtype, size_t* bytes) {
  t_err.clear();
  if (!bytes || (count > 0 && !shapes) || count < 0) return fail(DMUON_ERR_INVALID, "bad arguments");
  const bool f32 = param_dtype == DMUON_F32;
  std::map<std::pair<long long, long long>, std::pair<int, int>> counts;  // (m, n) -> (stored m x n, stored n x m)
  for (int i = 0; i < count; ++i) {
    const long long rr = shapes[2 * i], cc = shapes[2 * i + 1];
    if (rr <= 0 || cc <= 0) return fail(DMUON_ERR_INVALID, "bad shape");
    auto& e = counts[{std::min(rr, cc), std::max(rr, cc)}];
    (rr > cc ? e.second : e.first)++;
  }
  // the first call runs every group on one stream (with autotune scratch);
  // later calls may give up to three small groups a region each
  size_t need = 0, small_need = 0;
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  for (auto& kv : counts) {
    const bool xf = iter_f32(f32, kv.first.first);
    Geo g = make_geo(kv.first.first, kv.first.second, xf);
    const int total = kv.second.first + kv.second.second;
    int ch = chunk_size(g, total);
    Layout L = make_layout(g, ch, chunk_nblk(g, kv.second.first > 0, kv.second.second > 0));
    const size_t n_tune = align256(L.total + 2 * align256(static_cast<size_t>(ch) * g.x_elems() * g.esz) + 256);
    need = std::max(need, n_tune);
    const bool maybe_small = !xf && total <= ch && (tc_gemm_tiles(g.m, g.n, ch, 128, false) < 2LL * sms ||
                                                     tc_gemm_tiles(g.m, g.n, ch, 512, false) < sms);
    if (maybe_small) small_need = std::max(small_need, align256(L.total));
  }
  *bytes = need + 3 * small_need + align256(4 * sizeof(void*) * static_cast<size_t>(count));
  return DMUON_OK;
}

void dmuon_timing_enable(int enable) { g_timing.store(enable ? 1 : 0); }

void dmuon_timing_reset(void) {
  std::lock_guard<std::mutex> lk(g_tmu);
  for (auto& t : g_timed) {
    g_event_pool.push_back(t.a);
    g_event_pool.push_back(t.b);
  }
  g_timed.clear();
}

int dmuon_timing_get(int kind, int64_t* launches, double* ms, double* flops, double* bytes) {
  std::lock_guard<std::mutex> lk(g_tmu);
  int64_t n = 0;
  double t = 0, f = 0, b = 0;
  for (auto& x : g_timed) {
    if (kind == KIND_TC_GEMM_PAIR ? !(x.kind == KIND_TC_GEMM && x.pair) : x.kind != kind) continue;
    cudaError_t e = cudaEventSynchronize(x.b);
    if (e != cudaSuccess) return fail(DMUON_ERR_CUDA, "timing event: %s", cudaGetErrorString(e));
    float d = 0.f;
    cudaEventElapsedTime(&d, x.a, x.b);
    n += x.launches;
    t += d;
    f += x.flops;
    b += x.bytes;
  }
  if (launches) *launches = n;
  if (ms) *ms = t;
  if (flops) *flops = f;
  if (bytes) *bytes = b;
  return DMUON_OK;
}

int64_t dmuon_launch_count(void) { return g_launches.load(); }

const char* dmuon_last_error(void) { return t_err.c_str(); }

int dmuon_version(void) { return DMUON_VERSION; }

int dmuon_debug_groups(const int64_t* shapes, int count, int param_dtype, int grads_host, int64_t* out, int cap,
                       int* members) {
  t_err.clear();
  if (count < 0 || (count > 0 && !shapes) || cap < 0 || (cap > 0 && !out))
    return fail(DMUON_ERR_INVALID, "bad arguments");
  if (param_dtype != DMUON_BF16 && param_dtype != DMUON_F32) return fail(DMUON_ERR_DTYPE, "bad dtype");
  for (int i = 0; i < count; ++i)
    if (shapes[2 * i] <= 0 || shapes[2 * i + 1] <= 0 || shapes[2 * i] > INT32_MAX || shapes[2 * i + 1] > INT32_MAX)
      return fail(DMUON_ERR_INVALID, "bad shape of matrix %d", i);
  const bool f32 = param_dtype == DMUON_F32;
  std::vector<Geo> geos;
  const std::vector<Group> groups = make_groups(shapes, count, f32, grads_host != 0, f32, &geos);
  int pos = 0;
  for (size_t k = 0; k < groups.size(); ++k) {
    const Group& gr = groups[k];
    if (static_cast<long long>(k) < cap) {
      int64_t* o = out + 6 * k;
      o[0] = gr.rows;
      o[1] = gr.cols;
      o[2] = static_cast<int64_t>(gr.idx.size());
      o[3] = gr.ntall;
      o[4] = gr.chunk;
      o[5] = gr.xf ? 1 : 0;
    }
    if (members)
      for (int i : gr.idx) members[pos++] = i;
  }
  return static_cast<int>(groups.size());
}

int dmuon_debug_io_order(const int* counts, const int* chunks, const double* cost_ms, const double* bytes,
                         const int* sm_copy, int ngroups, int cached, int* out, int cap) {
  t_err.clear();
  if (ngroups < 0 || cap < 0 || (cap > 0 && !out) ||
      (ngroups > 0 && (!counts || !chunks || !cost_ms || !bytes || !sm_copy)))
    return fail(DMUON_ERR_INVALID, "bad arguments");
  std::vector<IoGroup> gs(ngroups);
  std::vector<int> order(ngroups);
  for (int g = 0; g < ngroups; ++g) {
    if (counts[g] < 0 || chunks[g] < 1 || !std::isfinite(cost_ms[g]) || !std::isfinite(bytes[g]) || bytes[g] < 0)
      return fail(DMUON_ERR_INVALID, "bad description of group %d", g);
    gs[g] = {counts[g], chunks[g], cost_ms[g], bytes[g], sm_copy[g] != 0};
    order[g] = g;
  }
  const std::vector<Piece> seq = chunk_order(gs, order, cached != 0, nullptr);
  for (size_t i = 0; i < seq.size() && static_cast<long long>(i) < cap; ++i) {
    out[3 * i] = seq[i].k;
    out[3 * i + 1] = seq[i].c0;
    out[3 * i + 2] = seq[i].cnt;
  }
  return static_cast<int>(seq.size());
}

}  // extern "C"
