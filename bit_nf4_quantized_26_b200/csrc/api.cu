// api.cu — the C ABI declared in include/qlora_nf4.h: argument checks,
// workspace planning, TMA descriptor creation and kernel launches.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "../../include/qlora_optim.h"

using namespace qnf4;

namespace {

// ------------------------------------------------------------ NF4 constants
//
// "QLoRA" encyclopedia entry (tonho.wtf), section "como funciona": a 4-bit
// type from standard-normal quantiles, normalised to [-1, 1] by the absolute
// maximum, asymmetric so that zero is exact.  Positive levels are the N(0,1)
// quantiles at 8 probabilities evenly spaced from DELTA towards 1/2, negative
// levels minus the quantiles at 7 such probabilities, plus 0; all divided by
// the largest magnitude.  DELTA is the mean of 1-1/30 and 1-1/32.  The
// quantile is found by bisection on Phi(x) = erfc(-x/sqrt 2)/2 in double
// precision, then rounded once to fp32.

double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

double normal_quantile(double p) {
  double lo = -12.0, hi = 12.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (normal_cdf(mid) < p) lo = mid;
    else hi = mid;
  }
  return 0.5 * (lo + hi);
}

// Set when the bucket table below fails its construction checks (a midpoint
// on or next to a bucket edge, or two midpoints in one bucket); every compute
// entry point then returns QLORA_ERR_INTERNAL.  The checks are on fixed
// constants, so this never happens with the NF4 levels.
bool g_tables_bad = false;

Nf4Tables build_tables() {
  const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
  std::vector<double> lv;
  const double step_pos = (0.5 - delta) / 8.0, step_neg = (0.5 - delta) / 7.0;
  for (int i = 0; i < 8; ++i) lv.push_back(normal_quantile(i * step_pos + delta));
  for (int i = 0; i < 7; ++i) lv.push_back(-normal_quantile(i * step_neg + delta));
  lv.push_back(0.0);
  std::sort(lv.begin(), lv.end());
  double amax = 0.0;
  for (double v : lv) amax = std::max(amax, std::fabs(v));
  Nf4Tables t{};
  for (int i = 0; i < 16; ++i) t.q[i] = static_cast<float>(lv[i] / amax);
  float mid[15];
  for (int i = 0; i < 15; ++i)
    mid[i] = static_cast<float>((static_cast<double>(t.q[i]) + static_cast<double>(t.q[i + 1])) / 2.0);
  for (int b = 0; b < 64; ++b) {
    t.thr[b] = INFINITY;
    t.base[b] = 0;
  }
  for (int b = 0; b <= 32; ++b) {
    const double lo = -1.0 + (b - 0.5) / 16.0, hi = -1.0 + (b + 0.5) / 16.0;
    int below = 0, inside = 0;
    float thr = INFINITY;
    for (int i = 0; i < 15; ++i) {
      const double m = mid[i];
      if (m < lo) ++below;
      else if (m <= hi) { ++inside; thr = mid[i]; }
      // A midpoint on (or next to) a bucket edge would make the bucket
      // choice matter; the NF4 midpoints sit at least 4e-3 from every edge.
      if (std::fabs(m - lo) < 1e-6 || std::fabs(m - hi) < 1e-6) g_tables_bad = true;
    }
    if (inside > 1) g_tables_bad = true;
    t.base[b] = below;
    t.thr[b] = thr;
  }
  return t;
}

const Nf4Tables& tables() {
  static const Nf4Tables t = build_tables();
  return t;
}

// ------------------------------------------------------------ TMA descriptors

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major tensor [outer, inner] of elements of `esize` bytes, row
// stride `row_bytes`, copied in boxes of [box_outer, box_inner].
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                               : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                     : CU_TENSOR_MAP_SWIZZLE_NONE;
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows, cols] row-major; the box's inner extent times 2 bytes must equal
// the swizzle span (128 or 64 bytes).
bool map_bf16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_cols, uint32_t box_rows,
              int swizzle_bytes = 128) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cols, rows, cols * 2, box_cols, box_rows,
                  swizzle_bytes);
}

bool map_u8(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, uint32_t box_cols, uint32_t box_rows,
            int swizzle_bytes = 0) {
  return make_map(m, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, cols, rows, cols, box_cols, box_rows, swizzle_bytes);
}

}  // namespace

bool qnf4::pdl_enabled() {
  static const bool enabled = [] {
    const char* e = getenv("QLORA_PDL");
    return !(e && e[0] == '0');
  }();
  return enabled;
}

namespace {

// Token count above which the 512-token kernels run.
constexpr int64_t kWideM = 256;

// CTA-pair (cta_group::2) kernels for large M when the W-side extent is a
// multiple of 256; QLORA_PAIR=0 selects the single-CTA 512-token kernel.
bool use_pair(int64_t rows) {
  static const bool enabled = [] {
    const char* e = getenv("QLORA_PAIR");
    return !(e && e[0] == '0');
  }();
  return enabled && rows % 256 == 0;
}

// QLORA_TMEM_A=1 selects the CTA-pair forward that keeps the dequantised
// tile in tensor memory (exact, but measured slower than the shared-memory
// kernel, which stays the default).
bool use_tmem_a() {
  static const bool enabled = [] {
    const char* e = getenv("QLORA_TMEM_A");
    return e && e[0] == '1';
  }();
  return enabled;
}

// A slots of that kernel: QLORA_TMEM_A_SLOTS = 4 (448-token tiles, the
// default) or 8 (384-token tiles).
int tmem_a_slots() {
  static const int v = [] {
    const char* e = getenv("QLORA_TMEM_A_SLOTS");
    return (e && atoi(e) == 8) ? 8 : 4;
  }();
  return v;
}

// ------------------------------------------------------------ checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status check_device() {
  (void)tables();
  if (g_tables_bad) return QLORA_ERR_INTERNAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  static int arch_ok[64] = {0};  // 0 unknown, 1 ok, 2 not sm_100
  if (dev < 0 || dev >= 64) return QLORA_ERR_ARCH;
  if (arch_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    arch_ok[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return arch_ok[dev] == 1 ? QLORA_OK : QLORA_ERR_ARCH;
}

constexpr int32_t kChunkRank = 64;  // largest rank the rank-r kernels take in one CTA
constexpr int32_t kMaxRank = 256;

qlora_status check_linear_shape(int64_t M, const nf4_weight& W, int32_t r) {
  const int64_t N = W.n_out, K = W.k_in;
  if (M < 0 || M >= (int64_t(1) << 31)) return QLORA_ERR_SHAPE;
  if (N < 64 || K < 64 || N % 64 != 0 || K % 64 != 0) return QLORA_ERR_SHAPE;
  if (N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N * K >= (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  if (r < 16 || r % 16 != 0 || r > kMaxRank) return QLORA_ERR_SHAPE;
  return QLORA_OK;
}

qlora_status check_weight_ptrs(const nf4_weight& W) {
  if (!W.codes || !W.c8 || !W.s2) return QLORA_ERR_NULL;
  if (!aligned16(W.codes) || !aligned16(W.c8) || !aligned16(W.s2) || (W.mean && !aligned16(W.mean)))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

qlora_status from_cuda(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

// ------------------------------------------------------------ kernel timing

enum KernelId {
  kKQuantize = 0, kKDequantize, kKDown, kKFusedFwd, kKFinishFwd, kKLowFwd, kKLowFinish, kKDU, kKDB, kKFusedDX,
  kKDA, kKAdamW8, kKDropout, kKDropoutDx, kKCount
};
const char* const kKernelNames[kKCount] = {
    "nf4_quantize", "nf4_dequantize", "lora_down", "fused_fwd", "finish_fwd", "lowm_fwd", "lowm_finish",
    "lora_du", "lora_db", "fused_dx", "lora_da", "adamw8", "dropout", "dropout_dx"};

struct ProfRecord {
  int id;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_prof_pool;

cudaEvent_t prof_event() {
  if (!g_prof_pool.empty()) {
    cudaEvent_t e = g_prof_pool.back();
    g_prof_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one kernel launch with events on its stream while profiling is on.
class ProfScope {
 public:
  ProfScope(int id, cudaStream_t s) : s_(s) {
    if (!g_prof_on) return;
    std::lock_guard<std::mutex> g(g_prof_mu);
    rec_.id = id;
    rec_.start = prof_event();
    rec_.stop = prof_event();
    if (rec_.start && rec_.stop) {
      cudaEventRecord(rec_.start, s_);
      active_ = true;
    }
  }
  ~ProfScope() {
    if (!active_) return;
    cudaEventRecord(rec_.stop, s_);
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_records.push_back(rec_);
  }

 private:
  cudaStream_t s_;
  ProfRecord rec_{};
  bool active_ = false;
};

// ------------------------------------------------------------ side stream
//
// The backward's dB and dA products depend on dU (and dY, X) but not on the
// dX GEMM, so they run on a second stream of the same device while dX runs:
// they are HBM-bound and fill the SMs that the dX GEMM's last wave of tiles
// leaves idle.  The fork and join are event edges on the caller's stream, so
// ordering for the caller (and stream capture) is unchanged.  QLORA_FORK=0
// keeps everything on the caller's stream.

struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool failed = false;
};
std::mutex g_side_mu;
SideStream g_side[64];

bool fork_enabled() {
  static const bool enabled = [] {
    const char* e = getenv("QLORA_FORK");
    return !(e && e[0] == '0');
  }();
  return enabled;
}

// The current device's side stream, created on first use; `lk` holds the
// lock (one fork/join sequence at a time).  nullptr: no fork.  While kernel
// timing is on there is no fork either, so that each kernel's event pair
// brackets that kernel alone rather than its overlap with the dX GEMM.
SideStream* side_stream(std::unique_lock<std::mutex>& lk) {
  if (!fork_enabled() || g_prof_on) return nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  lk = std::unique_lock<std::mutex>(g_side_mu);
  SideStream& ss = g_side[dev];
  if (ss.failed) return nullptr;
  if (!ss.s) {
    if (cudaStreamCreateWithFlags(&ss.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      ss.failed = true;
      return nullptr;
    }
  }
  return &ss;
}

// Fork on construction (side waits for everything issued on `main` so far),
// join on destruction (`main` waits for everything issued on the side).
class Fork {
 public:
  explicit Fork(cudaStream_t main) : main_(main), side_(main) {
    ss_ = side_stream(lk_);
    if (ss_ && cudaEventRecord(ss_->fork, main_) == cudaSuccess &&
        cudaStreamWaitEvent(ss_->s, ss_->fork, 0) == cudaSuccess) {
      side_ = ss_->s;
    } else {
      ss_ = nullptr;
    }
  }
  ~Fork() {
    if (ss_ && cudaEventRecord(ss_->join, side_) == cudaSuccess) cudaStreamWaitEvent(main_, ss_->join, 0);
  }
  cudaStream_t side() const { return side_; }

 private:
  std::unique_lock<std::mutex> lk_;
  cudaStream_t main_, side_;
  SideStream* ss_ = nullptr;
};

// ------------------------------------------------------------ planning
//
// Split counts depend only on the shape (sized against the 148 SMs of a
// B200), so the workspace query is a pure host function.

constexpr int kSms = 148;
constexpr int64_t kMaxCluster = 8;  // portable cluster size: splits reduced in-cluster

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Number of slices for `stages` contraction steps over `tiles` output tiles so
// that tiles * slices stays within `cta_budget` CTAs, with at least `min_per`
// steps per slice; every slice is non-empty.
void split_plan(int64_t tiles, int64_t stages, int64_t min_per, int64_t cta_budget, int& splits, int& per) {
  int64_t s = std::max<int64_t>(1, cta_budget / std::max<int64_t>(tiles, 1));
  s = std::min<int64_t>(s, std::max<int64_t>(1, stages / std::max<int64_t>(min_per, 1)));
  s = std::min<int64_t>(s, kMaxCluster);
  const int64_t p = cdiv(stages, s);
  per = static_cast<int>(p);
  splits = static_cast<int>(cdiv(stages, p));
}

// Slices of the contraction for the mid-size kernels (M <= 256, 128 W-side
// rows x bn tokens per tile, kst 64-deep stages).  The weight streams through
// once; splitting the contraction (a cluster, reduced in distributed shared
// memory) fills the SMs, but every slice adds a reduction and its cluster
// must be placed whole: s minimises waves(s) x (stages per slice + 3 s), with
// 2 CTAs per SM for tiles of up to 128 tokens (s <= 4) and 1 for 256
// (s <= 2), at least 8 stages per slice.  This model picked the measured best
// (or within a few percent of it) for 64-256 tokens on 22016x8192,
// 8192x22016, 4096x4096 and 11008x4096 weights.
void mid_splits(int64_t tiles, int64_t kst, int bn, int& splits, int& per) {
  const int64_t slots = (bn <= 128 ? 2 : 1) * kSms;
  const int64_t smax = std::min<int64_t>(bn <= 128 ? 4 : 2, std::max<int64_t>(1, kst / 8));
  int64_t best_s = 1, best_cost = -1;
  for (int64_t sl = 1; sl <= smax; ++sl) {
    const int64_t cost = cdiv(tiles * sl, slots) * (cdiv(kst, sl) + (sl > 1 ? 3 * sl : 0));
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = sl;
    }
  }
  per = static_cast<int>(cdiv(kst, best_s));
  splits = static_cast<int>(cdiv(kst, per));
}

struct FwdPlan {
  int s_down, per_down;
  int bn, s_fwd, per_fwd;
  bool low;                  // few-token path (lowm.cu)
  int low_tiles, low_kc, low_ctas, low_mpad;
  size_t off_ucat, off_pfwd, off_cnt, total;
};

// Few tokens: U = X A^T by the rank-r kernel (one 128-token tile per member,
// the contraction split over a cluster), then persistent CTAs (two per SM,
// and at least one per row tile so that no CTA's range spans more than two
// tiles) over tiles * kc units of W.
FwdPlan plan_fwd_low(int64_t M, int64_t N, int64_t K, int32_t r, int G) {
  FwdPlan p{};
  p.low = true;
  split_plan(G, K / 64, 4, 2 * kSms, p.s_down, p.per_down);
  p.low_mpad = M <= 8 ? 8 : 16;
  p.low_tiles = static_cast<int>(cdiv(N, kLowmRows));
  p.low_kc = static_cast<int>(cdiv(K / 64, 4));
  const int64_t units = static_cast<int64_t>(p.low_tiles) * p.low_kc;
  // Two CTAs per SM, less the slots the rank-r kernel's CTAs hold while it
  // runs beside this one (so that no persistent CTA starts late).
  const int64_t slots = 2 * kSms - static_cast<int64_t>(p.s_down) * G;
  p.low_ctas = static_cast<int>(std::min<int64_t>(units, std::max<int64_t>(slots, p.low_tiles)));
  size_t off = 0;
  p.off_pfwd = off;
  off += align256(static_cast<size_t>(p.low_ctas) * 2 * kLowmRows * p.low_mpad * 4);
  p.off_cnt = off;
  off += align256(static_cast<size_t>(p.low_tiles) * 4);
  p.off_ucat = off;
  off += align256(static_cast<size_t>(M) * 2 * G * r * 2);
  p.total = off;
  return p;
}

// Few tokens run the register-path kernel only on a large weight: it streams
// the weight at a higher rate there (22016x8192 at 1 token: 68.6 us against
// 83.0 for the mid-size kernel), while on smaller weights its fixed costs
// dominate and the mid-size kernel is faster (4096x4096: 25.6 against 20.5
// us).  The threshold is a process-wide setting (qlora_set_few_token_threshold).
std::atomic<int64_t> g_few_token_min_elems{int64_t(1) << 26};

bool few_token_path(int64_t M, int64_t N, int64_t K) {
  return M <= kLowmMaxM && N * K >= g_few_token_min_elems.load(std::memory_order_relaxed);
}

FwdPlan plan_fwd(int64_t M, int64_t N, int64_t K, int32_t r, int G) {
  if (r <= kChunkRank && few_token_path(M, N, K)) return plan_fwd_low(M, N, K, r, G);
  FwdPlan p{};
  const int64_t kst = K / 64;
  split_plan(cdiv(M, 128) * G, kst, 4, 2 * kSms, p.s_down, p.per_down);
  if (M > kWideM) {
    // The wide GEMM needs U only in its last stages and does not wait for it
    // before then, so U = X A^T runs beside the GEMM's main loop: one CTA per
    // 128-token tile over the whole contraction (about half as long as a GEMM
    // tile's main loop) holds few SMs and leaves the rest to the GEMM.
    p.s_down = 1;
    p.per_down = static_cast<int>(kst);
  }
  p.bn = M > 128 ? 256 : (M > 64 ? 128 : (M > 32 ? 64 : 32));
  const int64_t tiles = cdiv(N, 128) * cdiv(M, p.bn);
  if (M <= 256) {
    mid_splits(tiles, kst, p.bn, p.s_fwd, p.per_fwd);
  } else {
    p.s_fwd = 1;
    p.per_fwd = static_cast<int>(kst);
  }
  size_t off = 0;
  p.off_ucat = off;
  off += align256(static_cast<size_t>(M) * 2 * G * r * 2);
  p.off_pfwd = off;
  p.total = off;
  return p;
}

struct BwdPlan {
  int s_du, per_du, s_db, per_db, s_da, per_da, bn, s_dx, per_dx;
  size_t off_sucat, off_ducat, total;
};

// G members, the longest with n_max outputs (the dU contraction); sizes
// depend on M, G and r only.
BwdPlan plan_bwd(int64_t M, int64_t N, int64_t K, int32_t r, int G, int64_t n_max) {
  BwdPlan p{};
  split_plan(cdiv(M, 128) * G, n_max / 64, 4, 2 * kSms, p.s_du, p.per_du);
  if (M > kWideM) {  // dU runs beside the wide dX GEMM's main loop (as U beside Y)
    p.s_du = 1;
    p.per_du = static_cast<int>(n_max / 64);
  }
  // dB and dA run on the side stream beside dX: few CTAs with long
  // contractions take fewer SM-cycles from it than many short ones.
  split_plan(cdiv(N, 128), cdiv(M, 64), 4, kSms / 2, p.s_db, p.per_db);
  split_plan(cdiv(K, 128) * G, cdiv(M, 64), 4, kSms / 2, p.s_da, p.per_da);
  p.bn = M > 128 ? 256 : 128;
  // the mid-size dX GEMM (M <= 256): contraction over the N outputs
  p.s_dx = 1;
  p.per_dx = static_cast<int>(n_max / 64);
  if (M <= kWideM) mid_splits(cdiv(K, 128) * cdiv(M, p.bn), N / 64, p.bn, p.s_dx, p.per_dx);
  size_t off = 0;
  p.off_sucat = off;
  off += align256(static_cast<size_t>(M) * 2 * G * r * 2);
  p.off_ducat = off;
  off += align256(static_cast<size_t>(M) * 2 * G * r * 2);
  p.total = off;
  return p;
}

// A group of linears that read the same input, stacked along the output
// dimension: member g owns rows off[g] .. off[g+1]-1 of the stacked weight,
// B, Y, dY and dB.  A single linear is the group of one.
struct Group {
  int G = 1;
  int64_t off[5] = {0, 0, 0, 0, 0};
  int64_t n_max = 0;
};

Group single_group(int64_t N) {
  Group g;
  g.off[1] = N;
  g.n_max = N;
  return g;
}

// A single linear of rank r > 64 runs its rank-r products as ceil(r / 64)
// chunks of rank 64 (the last one r - 64 (chunks - 1) wide), laid out as a
// group's members: U [M, r], the hi/lo of s U [M, 2 r], dA [r, K].  The GEMMs
// take the whole rank in their adapter stages.
bool rank_chunks(const Group& g, int32_t r) { return g.G == 1 && r > kChunkRank; }

// Members 1..4, each a multiple of 128 rows (tiles never straddle members),
// summing to the stacked weight's rows.
qlora_status make_group(int32_t members, const int64_t* n_member, int64_t N, Group* out) {
  if (members < 1 || members > 4) return QLORA_ERR_SHAPE;
  if (!n_member) return QLORA_ERR_NULL;
  Group g;
  g.G = members;
  for (int i = 0; i < members; ++i) {
    const int64_t n = n_member[i];
    if (n < 64 || n % 64 != 0 || (members > 1 && n % 128 != 0)) return QLORA_ERR_SHAPE;
    g.off[i + 1] = g.off[i] + n;
    g.n_max = std::max(g.n_max, n);
  }
  if (g.off[members] != N) return QLORA_ERR_SHAPE;
  *out = g;
  return QLORA_OK;
}

// CTA-pair tiles (256 W rows) need every member boundary on a tile boundary.
bool group_pairs(const Group& g) {
  for (int i = 0; i <= g.G; ++i)
    if (g.off[i] % 256 != 0) return false;
  return true;
}

void fill_group(const Group& g, FusedArgs* fa) {
  fa->groups = g.G;
  for (int i = 0; i < 3; ++i) fa->grp_end[i] = static_cast<int>(i + 1 < g.G ? g.off[i + 1] : g.off[g.G]);
}
void fill_group(const Group& g, SkinnyArgs* sa) {
  sa->groups = g.G;
  for (int i = 0; i < 5; ++i) sa->grp_n[i] = static_cast<int>(i <= g.G ? g.off[i] : g.off[g.G]);
}
void fill_group(const Group& g, LowmArgs* la, int32_t r) {
  la->ra = g.G * r;
  la->groups = g.G;
  for (int i = 0; i < 3; ++i) la->grp_end[i] = static_cast<int>(i + 1 < g.G ? g.off[i + 1] : g.off[g.G]);
}

}  // namespace

// =================================================================== C ABI

extern "C" {

void qlora_profile_enable(int32_t enable) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = enable != 0;
}

int32_t qlora_profile_collect(int32_t* kernel_ids, float* ms, int32_t capacity) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  int32_t n = 0;
  bool ok = true;
  for (const ProfRecord& r : g_prof_records) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      ok = false;
    if (n < capacity) {
      if (kernel_ids) kernel_ids[n] = r.id;
      if (ms) ms[n] = t;
    }
    ++n;
    g_prof_pool.push_back(r.start);
    g_prof_pool.push_back(r.stop);
  }
  g_prof_records.clear();
  return ok ? n : -1;
}

const char* qlora_kernel_name(int32_t id) {
  return (id >= 0 && id < kKCount) ? kKernelNames[id] : "unknown";
}

int64_t qlora_set_few_token_threshold(int64_t min_weight_elems) {
  return g_few_token_min_elems.exchange(min_weight_elems < 0 ? 0 : min_weight_elems);
}

const char* qlora_strerror(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_NULL: return "a required pointer is NULL";
    case QLORA_ERR_SHAPE: return "a size violates the documented constraints";
    case QLORA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_NONFINITE: return "non-finite input";
    case QLORA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case QLORA_ERR_CUDA: return "a CUDA call failed";
    case QLORA_ERR_ARCH: return "the current device is not sm_100";
    case QLORA_ERR_DTYPE: return "unknown output dtype";
    case QLORA_ERR_INTERNAL: return "an internal constant table failed its construction check";
  }
  return "unknown status";
}

void nf4_levels(float out[16]) {
  if (out) std::memcpy(out, tables().q, sizeof(float) * 16);
}

size_t qlora_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
  return plan_fwd(M, N, K, r, 1).total;
}

size_t qlora_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
  return plan_bwd(M, N, K, r, 1, N).total;
}

qlora_status nf4_quantize(const uint16_t* w_bf16, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                          int32_t* d_status, void* stream) {
  if (numel < 0 || numel >= (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  if (numel == 0) return QLORA_OK;
  if (!w_bf16 || !codes || !c8 || !s2) return QLORA_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(c8) || !aligned16(s2) ||
      (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  ProfScope ps(kKQuantize, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_nf4_quantize(w_bf16, numel, codes, c8, s2, d_status, tables(),
                                       static_cast<cudaStream_t>(stream)));
}

qlora_status nf4_dequantize(const uint8_t* codes, const uint8_t* c8, const float* s2, int64_t numel,
                            uint16_t* w_bf16, void* stream) {
  if (numel < 0 || numel >= (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  if (numel == 0) return QLORA_OK;
  if (!w_bf16 || !codes || !c8 || !s2) return QLORA_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(c8) || !aligned16(s2)) return QLORA_ERR_ALIGN;
  if (numel >= (int64_t(1) << 37)) return QLORA_ERR_SHAPE;  // the output tensor map holds < 2^31 rows of 64
  if (qlora_status st = check_device()) return st;
  const int64_t nfull = numel / 64;
  CUtensorMap tm_out;
  if (nfull > 0 && !map_bf16(&tm_out, w_bf16, nfull, 64, 64, 32, 128)) return QLORA_ERR_CUDA;
  ProfScope ps(kKDequantize, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_nf4_dequantize(codes, c8, s2, nullptr, numel, w_bf16, nfull > 0 ? &tm_out : nullptr,
                                         tables(), static_cast<cudaStream_t>(stream)));
}

size_t nf4_centered_workspace_size(int64_t numel) {
  if (numel <= 0) return 0;
  const int64_t nblocks = cdiv(numel, 64), ngroups = cdiv(numel, 16384);
  // fp32 constants, fp64 group sums, two buffers for the pairwise passes
  return align256(static_cast<size_t>(nblocks) * 4) + align256(static_cast<size_t>(ngroups) * 8) +
         2 * align256(static_cast<size_t>(cdiv(ngroups, 2048)) * 8);
}

qlora_status nf4_quantize_centered(const uint16_t* w_bf16, int64_t numel, uint8_t* codes, uint8_t* c8, float* s2,
                                   float* mean, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (numel < 0 || numel >= (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  if (numel == 0) return QLORA_OK;
  if (!w_bf16 || !codes || !c8 || !s2 || !mean) return QLORA_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(c8) || !aligned16(s2) || !aligned16(mean) ||
      (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  if (!ws || ws_bytes < nf4_centered_workspace_size(numel)) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  float* cbuf = static_cast<float*>(ws);
  uint8_t* wp = static_cast<uint8_t*>(ws) + align256(static_cast<size_t>(cdiv(numel, 64)) * 4);
  double* gsum = reinterpret_cast<double*>(wp);
  wp += align256(static_cast<size_t>(cdiv(numel, 16384)) * 8);
  double* lvl0 = reinterpret_cast<double*>(wp);
  double* lvl1 = reinterpret_cast<double*>(wp + align256(static_cast<size_t>(cdiv(cdiv(numel, 16384), 2048)) * 8));
  ProfScope ps(kKQuantize, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_nf4_quantize_centered(w_bf16, numel, codes, c8, s2, mean, cbuf, gsum, lvl0, lvl1, d_status,
                                                tables(), static_cast<cudaStream_t>(stream)));
}

qlora_status nf4_dequantize_centered(const uint8_t* codes, const uint8_t* c8, const float* s2, const float* mean,
                                     int64_t numel, uint16_t* w_bf16, void* stream) {
  if (numel < 0 || numel >= (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  if (numel == 0) return QLORA_OK;
  if (!w_bf16 || !codes || !c8 || !s2 || !mean) return QLORA_ERR_NULL;
  if (!aligned16(w_bf16) || !aligned16(codes) || !aligned16(c8) || !aligned16(s2) || !aligned16(mean))
    return QLORA_ERR_ALIGN;
  if (numel >= (int64_t(1) << 37)) return QLORA_ERR_SHAPE;
  if (qlora_status st = check_device()) return st;
  const int64_t nfull = numel / 64;
  CUtensorMap tm_out;
  if (nfull > 0 && !map_bf16(&tm_out, w_bf16, nfull, 64, 64, 32, 128)) return QLORA_ERR_CUDA;
  ProfScope ps(kKDequantize, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_nf4_dequantize(codes, c8, s2, mean, numel, w_bf16, nfull > 0 ? &tm_out : nullptr, tables(),
                                         static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

qlora_status qnf4::check_fwd_args(const uint16_t* X, const uint16_t* Xa, int64_t M, const nf4_weight& W,
                                  const uint16_t* A, const uint16_t* B, int32_t r, const void* Y, int32_t y_dtype,
                                  const float* U_out, const int32_t* d_status) {
  if (qlora_status st = check_linear_shape(M, W, r)) return st;
  if (y_dtype != QLORA_DTYPE_BF16 && y_dtype != QLORA_DTYPE_F32) return QLORA_ERR_DTYPE;
  if (M == 0) return QLORA_OK;
  if (!X || !Xa || !A || !B || !Y || !U_out) return QLORA_ERR_NULL;
  if (qlora_status st = check_weight_ptrs(W)) return st;
  if (!aligned16(X) || !aligned16(Xa) || !aligned16(A) || !aligned16(B) || !aligned16(Y) || !aligned16(U_out) ||
      (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  return QLORA_OK;
}

extern "C" {

// The forward of a group of linears sharing X (a single linear is the group
// of one); Xa is the adapter's input: X itself, or X after dropout.  A is the
// members' adapters stacked [G r, K], B stacked [N, r], Y [M, N], U [M, G r].
static qlora_status linear_fwd_impl(const uint16_t* X, const uint16_t* Xa, int64_t M, nf4_weight W, const Group& grp,
                                    const uint16_t* A, const uint16_t* B, int32_t r, float s, void* Y,
                                    int32_t y_dtype, float* U_out, void* ws, size_t ws_bytes, int32_t* d_status,
                                    void* stream) {
  if (qlora_status st = check_fwd_args(X, Xa, M, W, A, B, r, Y, y_dtype, U_out, d_status)) return st;
  if (M == 0) return QLORA_OK;
  const int64_t N = W.n_out, K = W.k_in;
  const int G = grp.G;
  const int ra = G * r;
  const FwdPlan p = plan_fwd(M, N, K, r, G);
  if (!ws || ws_bytes < p.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* ucat = reinterpret_cast<uint16_t*>(wsb + p.off_ucat);
  float* pfwd = reinterpret_cast<float*>(wsb + p.off_pfwd);

  // U = Xa A^T for every member (contraction split over a cluster), plus the
  // bf16 hi/lo of s*U; the G CTAs of a token tile read the same X rows.
  CUtensorMap mx_down, ma_down;
  if (!map_bf16(&mx_down, Xa, M, K, 64, 128) || !map_bf16(&ma_down, A, ra, K, 64, 64)) return QLORA_ERR_CUDA;
  // A rank above 64 runs as ceil(r / 64) chunks of rank 64: the G CTAs of a
  // token tile are then the chunks instead of the members.
  const bool chunks = rank_chunks(grp, r);
  const int Gd = chunks ? (r + kChunkRank - 1) / kChunkRank : G;
  SkinnyArgs sa{};
  sa.M = static_cast<int>(M);
  sa.N = static_cast<int>(N);
  sa.K = static_cast<int>(K);
  sa.r = chunks ? kChunkRank : r;
  sa.stages_total = static_cast<int>(K / 64);
  sa.stages_per_split = p.per_down;
  sa.s = s;
  sa.out_f32 = U_out;
  sa.out_cat = ucat;
  sa.status = d_status;
  fill_group(grp, &sa);
  sa.groups = Gd;
  sa.chunks = chunks ? 1 : 0;
  sa.r_total = r;
  uint32_t* tile_count = reinterpret_cast<uint32_t*>(wsb + p.off_cnt);
  if (p.low) {  // the few-token kernel's tile counters start at zero
    sa.zero = tile_count;
    sa.zero_count = p.low_tiles;
  }
  {
    ProfScope ps(kKDown, cs);
    if (qlora_status st = from_cuda(launch_skinny(kSkDown, mx_down, ma_down, sa,
                                                  static_cast<int>(cdiv(M, 128)) * Gd, p.s_down, cs)))
      return st;
  }

  if (p.low) {
    LowmArgs la{};
    la.codes = W.codes;
    la.c8 = W.c8;
    la.s2 = W.s2;
    la.mean = W.mean;
    la.B = B;
    la.part = pfwd;
    la.Y = Y;
    la.y_f32 = y_dtype == QLORA_DTYPE_F32;
    la.U = U_out;
    la.tile_count = tile_count;
    la.s = s;
    la.M = static_cast<int>(M);
    la.N = static_cast<int>(N);
    la.K = static_cast<int>(K);
    la.r = r;
    la.tiles = p.low_tiles;
    la.atiles = 0;
    la.kc = p.low_kc;
    la.ctas = p.low_ctas;
    la.mpad = p.low_mpad;
    la.status = d_status;
    la.tab = tables();
    fill_group(grp, &la, r);
    CUtensorMap lc, lx;
    if (!map_u8(&lc, W.codes, N, K / 2, 128, kLowmRows, 128) ||
        !map_bf16(&lx, X, M, K, 64, static_cast<uint32_t>(p.low_mpad), 128))
      return QLORA_ERR_CUDA;
    ProfScope ps(kKLowFwd, cs);
    return from_cuda(launch_lowm_fwd(lc, lx, la, cs));
  }


  // Y = X W'^T + (sU) B^T, W' dequantised inside the GEMM.
  if (M > kWideM) {
    const bool pair = use_pair(N) && group_pairs(grp);
    const bool tmem_a = pair && use_tmem_a() && r <= kChunkRank;  // its adapter buffers hold r <= 64
    const uint32_t tok_box = tmem_a ? static_cast<uint32_t>(pair_fwd_tokens(tmem_a_slots()) / 4) : (pair ? 128 : 256);
    CUtensorMap wx, wc, wu, wb;
    if (!map_bf16(&wx, X, M, K, 32, tok_box, 64) || !map_u8(&wc, W.codes, N, K / 2, 16, 128) ||
        !map_bf16(&wu, ucat, M, 2 * ra, 32, tok_box, 64) || !map_bf16(&wb, B, N, r, 32, 128, 64))
      return QLORA_ERR_CUDA;
    FusedArgs fa{};
    fa.c8 = W.c8;
    fa.s2 = W.s2;
    fa.mean = W.mean;
    fa.out = Y;
    fa.out_f32 = y_dtype == QLORA_DTYPE_F32;
    fa.ld_out = N;
    fa.M = static_cast<int>(M);
    fa.rows = static_cast<int>(N);
    fa.n_out = static_cast<int>(N);
    fa.k_in = static_cast<int>(K);
    fa.r = r;
    fa.kt_total = static_cast<int>(K / 32);
    fa.kt_per_split = fa.kt_total;
    fa.status = d_status;
    fa.tab = tables();
    fill_group(grp, &fa);
    ProfScope ps(kKFusedFwd, cs);
    if (tmem_a) return from_cuda(launch_fused_pair_fwd(wx, wc, wu, wb, fa, tmem_a_slots(), cs));
    return from_cuda(pair ? launch_fused_pair(false, wx, wc, wu, wb, fa, cs)
                          : launch_fused2x(false, wx, wc, wu, wb, fa, cs));
  }
  CUtensorMap mx, mc, mu, mb;
  if (!map_bf16(&mx, X, M, K, 64, p.bn) || !map_u8(&mc, W.codes, N, K / 2, 32, 128) ||
      !map_bf16(&mu, ucat, M, 2 * ra, 64, p.bn) || !map_bf16(&mb, B, N, r, 64, 128))
    return QLORA_ERR_CUDA;
  FusedArgs fa{};
  fa.c8 = W.c8;
  fa.s2 = W.s2;
  fa.mean = W.mean;
  fa.out = Y;
  fa.out_f32 = y_dtype == QLORA_DTYPE_F32;
  fa.ld_out = N;
  fa.M = static_cast<int>(M);
  fa.rows = static_cast<int>(N);
  fa.n_out = static_cast<int>(N);
  fa.k_in = static_cast<int>(K);
  fa.r = r;
  fa.kt_total = static_cast<int>(K / 64);
  fa.kt_per_split = p.per_fwd;
  fa.status = d_status;
  fa.tab = tables();
  fill_group(grp, &fa);
  ProfScope ps(kKFusedFwd, cs);
  return from_cuda(launch_fused_fwd(p.bn, mx, mc, mu, mb, fa, p.s_fwd, cs));
}

qlora_status qlora_linear_fwd(const uint16_t* X, int64_t M, nf4_weight W, const uint16_t* A, const uint16_t* B,
                              int32_t r, float s, void* Y, int32_t y_dtype, float* U_out, void* ws,
                              size_t ws_bytes, int32_t* d_status, void* stream) {
  return linear_fwd_impl(X, X, M, W, single_group(W.n_out), A, B, r, s, Y, y_dtype, U_out, ws, ws_bytes, d_status,
                         stream);
}

// The backward of a group (a single linear is the group of one); X is the
// adapter's input (X itself, or X after dropout, for dA).  dY [M, N] stacked,
// U [M, G r], A [G r, K], B [N, r], dA [G r, K], dB [N, r]; dX [M, K] is the
// sum over the members.  With `drop`, the GEMM's adapter stages are left out:
// dX's frozen-path term goes to an fp32 buffer after the caller's workspace
// and a second pass adds keep * c * (dU A) and writes dX.
static qlora_status linear_bwd_impl(const uint16_t* dY, const uint16_t* X, const float* U, int64_t M, nf4_weight W,
                                    const Group& grp, const uint16_t* A, const uint16_t* B, int32_t r, float s,
                                    void* dX, int32_t dx_dtype, float* dA, float* dB, void* ws, size_t ws_bytes,
                                    int32_t* d_status, void* stream, const DropoutArgs* drop) {
  if (qlora_status st = check_linear_shape(M, W, r)) return st;
  if (dx_dtype != QLORA_DTYPE_BF16 && dx_dtype != QLORA_DTYPE_F32) return QLORA_ERR_DTYPE;
  if (M == 0) return QLORA_OK;
  if (!dY || !X || !U || !A || !B || !dX || !dA || !dB) return QLORA_ERR_NULL;
  if (qlora_status st = check_weight_ptrs(W)) return st;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(U) || !aligned16(A) || !aligned16(B) || !aligned16(dX) ||
      !aligned16(dA) || !aligned16(dB) || (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  const int64_t N = W.n_out, K = W.k_in;
  const int G = grp.G;
  const int ra = G * r;
  const BwdPlan p = plan_bwd(M, N, K, r, G, grp.n_max);
  const size_t need = p.total + (drop ? align256(static_cast<size_t>(M) * K * 4) : 0);
  if (!ws || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* sucat = reinterpret_cast<uint16_t*>(wsb + p.off_sucat);
  uint16_t* ducat = reinterpret_cast<uint16_t*>(wsb + p.off_ducat);
  float* dx32 = drop ? reinterpret_cast<float*>(wsb + p.total) : nullptr;
  void* dx_gemm = drop ? static_cast<void*>(dx32) : dX;           // where the GEMM writes
  const int gemm_f32 = drop ? 1 : (dx_dtype == QLORA_DTYPE_F32);
  const int gemm_r = drop ? 0 : ra;                               // adapter stages in the GEMM (all members)
  const int Mi = static_cast<int>(M), Ni = static_cast<int>(N), Ki = static_cast<int>(K);

  // A rank above 64: ceil(r / 64) chunks of rank 64 (DU and DA: G CTAs per
  // tile; DB: G CTAs per row tile, each writing its columns of dB).
  const bool chunks = rank_chunks(grp, r);
  const int Gs = chunks ? (r + kChunkRank - 1) / kChunkRank : G;
  SkinnyArgs sa{};
  sa.M = Mi;
  sa.N = Ni;
  sa.K = Ki;
  sa.r = chunks ? kChunkRank : r;
  sa.status = d_status;
  fill_group(grp, &sa);
  sa.groups = Gs;
  sa.chunks = chunks ? 1 : 0;
  sa.r_total = r;

  // dU = s dY B per member (contraction over the member's outputs, split over
  // a cluster) -> bf16 hi/lo, and the bf16 hi/lo of s*U for dB from the saved U.
  CUtensorMap mdy128, mbl;
  if (!map_bf16(&mdy128, dY, M, N, 64, 128) || !map_bf16(&mbl, B, N, r, 64, 64)) return QLORA_ERR_CUDA;
  sa.stages_total = static_cast<int>(grp.n_max / 64);
  sa.stages_per_split = p.per_du;
  sa.s = s;
  sa.out_f32 = nullptr;
  sa.out_cat = ducat;
  sa.in_u = U;
  sa.out_cat2 = sucat;
  {
    ProfScope ps(kKDU, cs);
    if (qlora_status st =
            from_cuda(launch_skinny(kSkDU, mdy128, mbl, sa, static_cast<int>(cdiv(M, 128)) * Gs, p.s_du, cs)))
      return st;
  }

  // dB and dA go to the side stream (they need dU, not dX) and are issued
  // after dX, so dX's tiles take the SMs first and dB / dA fill the ones its
  // last wave leaves idle; the join at the end of this scope makes the
  // caller's stream wait for them.
  Fork fork(cs);
  const cudaStream_t side = fork.side();

  // dX = dY W' + dU A (summed over the members: one contraction over the
  // stacked outputs, then one over the stacked adapter rank), W' dequantised
  // inside the GEMM.
  if (M > kWideM) {
    const bool pair = use_pair(K);
    const uint32_t tok_box = pair ? 128 : 256;
    CUtensorMap wdy, wc, wdu, wal;
    if (!map_bf16(&wdy, dY, M, N, 32, tok_box, 64) || !map_u8(&wc, W.codes, N, K / 2, 64, 32) ||
        !map_bf16(&wdu, ducat, M, 2 * ra, 32, tok_box, 64) || !map_bf16(&wal, A, ra, K, 64, 16, 128))
      return QLORA_ERR_CUDA;
    FusedArgs fa{};
    fa.c8 = W.c8;
    fa.s2 = W.s2;
    fa.mean = W.mean;
    fa.out = dx_gemm;
    fa.out_f32 = gemm_f32;
    fa.ld_out = K;
    fa.M = Mi;
    fa.rows = Ki;
    fa.n_out = Ni;
    fa.k_in = Ki;
    fa.r = gemm_r;
    fa.kt_total = static_cast<int>(N / 32);
    fa.kt_per_split = fa.kt_total;
    fa.status = d_status;
    fa.tab = tables();
    fa.groups = 1;
    ProfScope ps(kKFusedDX, cs);
    if (qlora_status st = from_cuda(pair ? launch_fused_pair(true, wdy, wc, wdu, wal, fa, cs)
                                         : launch_fused2x(true, wdy, wc, wdu, wal, fa, cs)))
      return st;
  } else {
    CUtensorMap mdy, mc, mdu, mal;
    if (!map_bf16(&mdy, dY, M, N, 64, p.bn) || !map_u8(&mc, W.codes, N, K / 2, 64, 64) ||
        !map_bf16(&mdu, ducat, M, 2 * ra, 64, p.bn) || !map_bf16(&mal, A, ra, K, 64, 64))
      return QLORA_ERR_CUDA;
    FusedArgs fa{};
    fa.c8 = W.c8;
    fa.s2 = W.s2;
    fa.mean = W.mean;
    fa.out = dx_gemm;
    fa.out_f32 = gemm_f32;
    fa.ld_out = K;
    fa.M = Mi;
    fa.rows = Ki;
    fa.n_out = Ni;
    fa.k_in = Ki;
    fa.r = gemm_r;
    fa.kt_total = static_cast<int>(N / 64);
    fa.kt_per_split = p.per_dx;
    fa.status = d_status;
    fa.tab = tables();
    fa.groups = 1;
    ProfScope ps(kKFusedDX, cs);
    if (qlora_status st = from_cuda(launch_fused_dx(p.bn, mdy, mc, mdu, mal, fa, p.s_dx, cs))) return st;
  }
  if (drop) {  // dX = dX_main + keep * c * (dU A), on the caller's stream after the GEMM
    ProfScope ps(kKDropoutDx, cs);
    if (qlora_status st = from_cuda(
            launch_dropout_dx(dx32, ducat, A, dX, dx_dtype == QLORA_DTYPE_F32, Mi, Ki, r, *drop, cs)))
      return st;
  }

  // dB = s dY^T U per member (contraction over M split over a cluster)
  CUtensorMap mdy64, msu;
  if (!map_bf16(&mdy64, dY, M, N, 64, 64) || !map_bf16(&msu, sucat, M, 2 * ra, 64, 64)) return QLORA_ERR_CUDA;
  sa.stages_total = static_cast<int>(cdiv(M, 64));
  sa.stages_per_split = p.per_db;
  sa.s = 1.0f;
  sa.out_f32 = dB;
  sa.out_cat = nullptr;
  sa.in_u = nullptr;
  sa.out_cat2 = nullptr;
  {
    ProfScope ps(kKDB, side);
    if (qlora_status st =
            from_cuda(launch_skinny(kSkDB, mdy64, msu, sa, static_cast<int>(cdiv(N, 128)) * (chunks ? Gs : 1), p.s_db,
                                    side)))
      return st;
  }

  // dA = dU^T X per member (contraction over M split over a cluster)
  CUtensorMap mduc, mx;
  if (!map_bf16(&mduc, ducat, M, 2 * ra, 64, 64) || !map_bf16(&mx, X, M, K, 64, 64)) return QLORA_ERR_CUDA;
  {
    SkinnyArgs da = sa;
    da.stages_total = static_cast<int>(cdiv(M, 64));
    da.stages_per_split = p.per_da;
    da.s = 1.0f;
    da.out_f32 = dA;
    da.out_cat = nullptr;
    ProfScope ps(kKDA, side);
    if (qlora_status st = from_cuda(
            launch_skinny(kSkDA, mduc, mx, da, static_cast<int>(cdiv(K, 128)) * Gs, p.s_da, side)))
      return st;
  }

  return QLORA_OK;
}

qlora_status qlora_linear_bwd(const uint16_t* dY, const uint16_t* X, const float* U, int64_t M, nf4_weight W,
                              const uint16_t* A, const uint16_t* B, int32_t r, float s, void* dX, int32_t dx_dtype,
                              float* dA, float* dB, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  return linear_bwd_impl(dY, X, U, M, W, single_group(W.n_out), A, B, r, s, dX, dx_dtype, dA, dB, ws, ws_bytes,
                         d_status, stream, nullptr);
}

// ------------------------------------------------------------ grouped linears

size_t qlora_group_fwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t members, int32_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0 || members < 1 || members > 4) return 0;
  return plan_fwd(M, N, K, r, members).total;
}

size_t qlora_group_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int32_t members, int32_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0 || members < 1 || members > 4) return 0;
  return plan_bwd(M, N, K, r, members, N).total;
}

qlora_status qlora_group_fwd(const uint16_t* X, int64_t M, nf4_weight W, int32_t members, const int64_t* n_member,
                             const uint16_t* A, const uint16_t* B, int32_t r, float s, void* Y, int32_t y_dtype,
                             float* U_out, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (qlora_status st = check_linear_shape(M, W, r)) return st;
  if (members > 1 && r > kChunkRank) return QLORA_ERR_SHAPE;  // members' ranks are at most 64
  Group grp;
  if (qlora_status st = make_group(members, n_member, W.n_out, &grp)) return st;
  return linear_fwd_impl(X, X, M, W, grp, A, B, r, s, Y, y_dtype, U_out, ws, ws_bytes, d_status, stream);
}

qlora_status qlora_group_bwd(const uint16_t* dY, const uint16_t* X, const float* U, int64_t M, nf4_weight W,
                             int32_t members, const int64_t* n_member, const uint16_t* A, const uint16_t* B,
                             int32_t r, float s, void* dX, int32_t dx_dtype, float* dA, float* dB, void* ws,
                             size_t ws_bytes, int32_t* d_status, void* stream) {
  if (qlora_status st = check_linear_shape(M, W, r)) return st;
  if (members > 1 && r > kChunkRank) return QLORA_ERR_SHAPE;  // members' ranks are at most 64
  Group grp;
  if (qlora_status st = make_group(members, n_member, W.n_out, &grp)) return st;
  return linear_bwd_impl(dY, X, U, M, W, grp, A, B, r, s, dX, dx_dtype, dA, dB, ws, ws_bytes, d_status, stream,
                         nullptr);
}

qlora_status qlora_selftest_timeout(int32_t* d_status, int64_t limit_ns, void* stream) {
  if (!d_status) return QLORA_ERR_NULL;
  if (limit_ns < 1000 || limit_ns > 2000000000) return QLORA_ERR_SHAPE;
  if (!aligned16(d_status)) return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  return from_cuda(launch_selftest_timeout(d_status, static_cast<uint64_t>(limit_ns), static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------ LoRA dropout

// Host constants of the mask: keep when the Philox word is below
// T = floor((1 - p) 2^32) (fp64), every element for p = 0; c = fp32(1/(1-p)).
static bool dropout_args(float p, uint64_t seed, DropoutArgs* d) {
  if (!(p >= 0.0f && p < 1.0f)) return false;
  const double keep = 1.0 - static_cast<double>(p);
  const double t = std::floor(keep * 4294967296.0);
  d->seed = seed;
  d->keep_all = t >= 4294967296.0 ? 1 : 0;
  d->threshold = d->keep_all ? 0xFFFFFFFFu : static_cast<uint32_t>(t);
  d->c = static_cast<float>(1.0 / keep);
  return true;
}

size_t qlora_bwd_dropout_workspace_size(int64_t M, int64_t N, int64_t K, int32_t r) {
  if (M <= 0 || N <= 0 || K <= 0 || r <= 0) return 0;
  return plan_bwd(M, N, K, r, 1, N).total + align256(static_cast<size_t>(M) * K * 4);
}

qlora_status qlora_linear_fwd_dropout(const uint16_t* X, int64_t M, nf4_weight W, const uint16_t* A,
                                      const uint16_t* B, int32_t r, float s, float p, uint64_t seed,
                                      uint16_t* X_drop, void* Y, int32_t y_dtype, float* U_out, void* ws,
                                      size_t ws_bytes, int32_t* d_status, void* stream) {
  DropoutArgs d{};
  if (!dropout_args(p, seed, &d)) return QLORA_ERR_SHAPE;
  if (qlora_status st = check_linear_shape(M, W, r)) return st;
  if (y_dtype != QLORA_DTYPE_BF16 && y_dtype != QLORA_DTYPE_F32) return QLORA_ERR_DTYPE;
  if (M == 0) return QLORA_OK;
  if (!X || !X_drop || !A || !B || !Y || !U_out) return QLORA_ERR_NULL;
  if (qlora_status st = check_weight_ptrs(W)) return st;
  if (!aligned16(X) || !aligned16(X_drop) || !aligned16(A) || !aligned16(B) || !aligned16(Y) ||
      !aligned16(U_out) || (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  const FwdPlan pl = plan_fwd(M, W.n_out, W.k_in, r, 1);
  if (!ws || ws_bytes < pl.total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  {
    ProfScope ps(kKDropout, static_cast<cudaStream_t>(stream));
    if (qlora_status st =
            from_cuda(launch_dropout_apply(X, X_drop, M * W.k_in, d, static_cast<cudaStream_t>(stream))))
      return st;
  }
  return linear_fwd_impl(X, X_drop, M, W, single_group(W.n_out), A, B, r, s, Y, y_dtype, U_out, ws, ws_bytes,
                         d_status, stream);
}

qlora_status qlora_linear_bwd_dropout(const uint16_t* dY, const uint16_t* X_drop, const float* U, int64_t M,
                                      nf4_weight W, const uint16_t* A, const uint16_t* B, int32_t r, float s, float p,
                                      uint64_t seed, void* dX, int32_t dx_dtype, float* dA, float* dB, void* ws,
                                      size_t ws_bytes, int32_t* d_status, void* stream) {
  DropoutArgs d{};
  if (!dropout_args(p, seed, &d)) return QLORA_ERR_SHAPE;
  return linear_bwd_impl(dY, X_drop, U, M, W, single_group(W.n_out), A, B, r, s, dX, dx_dtype, dA, dB, ws, ws_bytes,
                         d_status, stream, &d);
}

// ------------------------------------------------------------------ optimizer

qlora_status qlora_adamw8_step(uint16_t* p, const float* grad, uint8_t* m8, uint8_t* u8, float* m_scale,
                               float* u_scale, int64_t n, float lr, float beta1, float beta2, float eps,
                               float weight_decay, int64_t step, int32_t* d_status, void* stream) {
  if (n < 0 || n >= (int64_t(1) << 40) || step < 1) return QLORA_ERR_SHAPE;
  if (!std::isfinite(lr) || !std::isfinite(eps) || !std::isfinite(weight_decay) || eps < 0.0f ||
      !(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f))
    return QLORA_ERR_SHAPE;
  if (n == 0) return QLORA_OK;
  if (!p || !grad || !m8 || !u8 || !m_scale || !u_scale) return QLORA_ERR_NULL;
  if (!aligned16(p) || !aligned16(grad) || !aligned16(m8) || !aligned16(u8) || !aligned16(m_scale) ||
      !aligned16(u_scale) || (d_status && !aligned16(d_status)))
    return QLORA_ERR_ALIGN;
  if (qlora_status st = check_device()) return st;
  AdamW8Args a{};
  a.p = p;
  a.g = grad;
  a.m8 = m8;
  a.u8 = u8;
  a.m_scale = m_scale;
  a.u_scale = u_scale;
  a.n = n;
  a.lr = lr;
  a.b1 = beta1;
  a.b2 = beta2;
  a.omb1 = 1.0f - beta1;  // one fp32 subtraction (exact for beta in [0.5, 1))
  a.omb2 = 1.0f - beta2;
  a.eps = eps;
  a.wd = weight_decay;
  // Bias corrections in fp64 from the fp32 betas, rounded once to fp32.
  const double t = static_cast<double>(step);
  a.bc1 = static_cast<float>(1.0 / (1.0 - std::pow(static_cast<double>(beta1), t)));
  a.bc2 = static_cast<float>(1.0 / std::sqrt(1.0 - std::pow(static_cast<double>(beta2), t)));
  a.status = d_status;
  ProfScope ps(kKAdamW8, static_cast<cudaStream_t>(stream));
  return from_cuda(launch_adamw8(a, static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_paged_alloc(void** ptr, size_t bytes) {
  if (!ptr) return QLORA_ERR_NULL;
  *ptr = nullptr;
  if (bytes == 0) return QLORA_ERR_SHAPE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  void* q = nullptr;
  if (cudaMallocManaged(&q, bytes, cudaMemAttachGlobal) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemAdvise(q, bytes, cudaMemAdviseSetPreferredLocation, dev) != cudaSuccess ||
      cudaMemset(q, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(q);
    return QLORA_ERR_CUDA;
  }
  *ptr = q;
  return QLORA_OK;
}

qlora_status qlora_paged_prefetch(const void* ptr, size_t bytes, int32_t to_host, void* stream) {
  if (!ptr) return QLORA_ERR_NULL;
  if (bytes == 0) return QLORA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_CUDA;
  return from_cuda(cudaMemPrefetchAsync(ptr, bytes, to_host ? cudaCpuDeviceId : dev,
                                        static_cast<cudaStream_t>(stream)));
}

qlora_status qlora_paged_free(void* ptr) {
  if (!ptr) return QLORA_OK;
  return from_cuda(cudaFree(ptr));
}

}  // extern "C"
