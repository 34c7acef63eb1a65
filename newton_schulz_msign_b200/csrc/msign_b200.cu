// msign_b200.cu - C ABI of the library (declared in include/msign_b200.h):
// argument checks, workspace layout, TMA descriptor construction and the
// launch sequences of msign_ns, gram_xxt, gram_ns and muon_step.
//
// Every step of every entry point runs in the kernels of gemm_sm100.cuh and
// elementwise.cuh; the host only plans and enqueues.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "msign_b200.h"
#include "elementwise.cuh"
#include "gemm_sm100.cuh"

namespace msb {

// Device error word raised by bounded waits (bit 0).
__device__ int g_err_word;

constexpr float kJordanA = 3.4445f, kJordanB = -4.7750f, kJordanC = 2.0315f;  // [P2] eq. 7
constexpr int kJordanSteps = 5;
constexpr float kNsEps = 1e-20f;    // [P2] section 参考实现, under the square root
constexpr float kGramEps = 1e-7f;   // [P3] Algorithm 2 step 1, added to the norm
constexpr int kMaxSteps = 64;
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // 4 s per wait

// ---------------------------------------------------------------- device state

struct DeviceState {
  bool ready = false;
  int sms = 0;
  int max_pairs = 0;  // CTA pairs of the GEMM kernel that fit on the GPU at once
  int ingest_blocks = 0;  // ingest_kernel blocks resident at once on the whole GPU
  int* err = nullptr;
};

std::mutex g_mu;
DeviceState g_dev[64];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

msign_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MSIGN_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return MSIGN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return MSIGN_ERR_CUDA;
    if (major != 10 || minor != 0) return MSIGN_ERR_UNSUPPORTED;  // built for sm_100a only
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MSIGN_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.err), g_err_word) != cudaSuccess) return MSIGN_ERR_CUDA;
    if (cudaFuncSetAttribute(gemm_sm100_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_sm100_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_sm100_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_sm100_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return MSIGN_ERR_CUDA;
    {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(static_cast<unsigned>(d.sms & ~1), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = kSmemBytes;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, gemm_sm100_kernel<false, false>, &cfg) != cudaSuccess ||
          clusters < 1) {
        (void)cudaGetLastError();
        clusters = d.sms / 2;
      }
      d.max_pairs = clusters;
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, ingest_kernel, 256, 0) != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        per_sm = 4;
      }
      d.ingest_blocks = per_sm * d.sms;
    }
    if (g_encode == nullptr) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return MSIGN_ERR_CUDA;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ready = true;
  }
  *out = &d;
  return MSIGN_OK;
}

// ---------------------------------------------------------------- launch records
//
// While enabled (msign_profile_enable), every kernel the library enqueues is
// bracketed by two CUDA events on its own stream, tagged with its kind and
// its algorithmic work (useful FLOPs, compulsory HBM bytes).

struct ProfRec {
  int kind;
  cudaEvent_t e0, e1;
  double flops, bytes;
};

bool g_prof = false;
std::vector<ProfRec> g_prof_recs;
std::vector<cudaEvent_t> g_event_pool;
cudaEvent_t g_pending = nullptr;

cudaEvent_t pool_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

void prof_begin(cudaStream_t s) {
  if (!g_prof) return;
  g_pending = pool_event();
  cudaEventRecord(g_pending, s);
}

void prof_end(int kind, cudaStream_t s, double flops, double bytes) {
  if (!g_prof || g_pending == nullptr) return;
  cudaEvent_t e1 = pool_event();
  cudaEventRecord(e1, s);
  g_prof_recs.push_back({kind, g_pending, e1, flops, bytes});
  g_pending = nullptr;
}

// ---------------------------------------------------------------- helpers

inline int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// NS steps per chained launch: 3 phases each, within kMaxClasses classes.
constexpr int kChainSteps = 5;
static_assert(3 * kChainSteps <= kMaxClasses, "a chain of kChainSteps steps fits one launch");

int to_dt(msign_dtype d) { return d == MSIGN_BF16 ? DT_BF16 : d == MSIGN_FP16 ? DT_FP16 : DT_FP32; }

bool valid_dtype(msign_dtype d) { return d == MSIGN_BF16 || d == MSIGN_FP16 || d == MSIGN_FP32; }

// Batch strides: 0 (matrices back to back) or at least one matrix, so that
// the matrices of a batch never overlap.
bool valid_strides(int64_t rows, int64_t cols, int64_t in_stride, int64_t out_stride) {
  const int64_t per = rows * cols;
  return in_stride >= 0 && out_stride >= 0 && (in_stride == 0 || in_stride >= per) &&
         (out_stride == 0 || out_stride >= per);
}

// Workspace carving: the same routine sizes and slices the workspace.
struct Carver {
  char* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  void* take(size_t bytes) {
    off = (off + 1023) & ~size_t(1023);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
};

struct Schedule {
  std::vector<float> abc;
  float eps;
  int init = 0;    // 1: sharper step-0 normalisation (msign_coeffs.init)
  int method = 0;  // 1: msign_ns may run Gram NS (msign_coeffs.method)
  int steps() const { return static_cast<int>(abc.size() / 3); }
};

msign_status read_schedule(const msign_coeffs* c, float default_eps, Schedule* s) {
  int T = kJordanSteps;
  const float* abc = nullptr;
  float eps = default_eps;
  if (c != nullptr) {
    if (c->abc != nullptr) {
      if (c->steps <= 0) return MSIGN_ERR_INVALID_ARG;
      T = c->steps;
      abc = c->abc;
    } else if (c->steps > 0) {
      T = c->steps;
    }
    if (c->eps >= 0.0f) eps = c->eps;
    if (!std::isfinite(eps)) return MSIGN_ERR_INVALID_ARG;
    if (c->init != 0 && c->init != 1) return MSIGN_ERR_INVALID_ARG;
    s->init = c->init;
    if (c->method != 0 && c->method != 1) return MSIGN_ERR_INVALID_ARG;
    s->method = c->method;
  }
  if (T > kMaxSteps) return MSIGN_ERR_UNSUPPORTED;
  s->abc.resize(3 * T);
  for (int t = 0; t < T; ++t) {
    s->abc[3 * t + 0] = abc ? abc[3 * t + 0] : kJordanA;
    s->abc[3 * t + 1] = abc ? abc[3 * t + 1] : kJordanB;
    s->abc[3 * t + 2] = abc ? abc[3 * t + 2] : kJordanC;
    for (int j = 0; j < 3; ++j)
      if (!std::isfinite(s->abc[3 * t + j])) return MSIGN_ERR_INVALID_ARG;
  }
  s->eps = eps;
  return MSIGN_OK;
}

// A dense batched matrix: rows x cols, leading dimension ld, batch stride bs
// (both in elements).
struct Mat {
  const void* ptr;
  int dt;
  int64_t rows, cols, ld, bs;
};

bool tma_ok(const Mat& m) {
  const int es = dtype_size(m.dt);
  return (reinterpret_cast<uintptr_t>(m.ptr) % 16) == 0 && (m.ld * es) % 16 == 0 && (m.bs * es) % 16 == 0;
}

// 3-D tensor map (cols, rows, batch) with a box of one 128-byte swizzle row
// (64 16-bit or 32 fp32 elements) by box_rows.  For split operands the
// batch coordinate counts planes (2 per matrix) and m.bs is the plane stride.
// mn_major: the box feeds an MN-major operand; fp32 words then take the
// 32-byte-chunk form of the 128-byte swizzle, the only MN-major form the
// tf32 MMA reads.
bool encode(CUtensorMap* tm, const Mat& m, int box0, int box_rows, int64_t batch, bool mn_major = false) {
  const int es = dtype_size(m.dt);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(m.cols), static_cast<cuuint64_t>(m.rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(m.ld * es), static_cast<cuuint64_t>(m.bs * es)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapDataType dt = m.dt == DT_BF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : m.dt == DT_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                   : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapSwizzle sw =
      (mn_major && es == 4) ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = g_encode(tm, dt, 3, const_cast<void*>(m.ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D tensor map (cols, rows, batch) of a 16-bit output for the epilogue's
// staged bulk stores: a 32 x 32 box (64-byte rows) in the 64-byte swizzle.
bool encode_out(CUtensorMap* tm, const Mat& m, int64_t batch) {
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(m.cols), static_cast<cuuint64_t>(m.rows),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(m.ld * 2), static_cast<cuuint64_t>(m.bs * 2)};
  cuuint32_t box[3] = {32u, 32u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapDataType dt = m.dt == DT_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = g_encode(tm, dt, 3, const_cast<void*>(m.ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 in the blocked layout of blk_off(): padded width and per-matrix size
inline int64_t blk_ld(int64_t cols) { return round_up(cols, 32); }
inline int64_t blk_size(int64_t rows, int64_t cols) { return round_up(rows, 32) * round_up(cols, 32); }

EpiOut out_to(void* ptr, int dt, int64_t ld, int64_t bs, bool transposed, float gamma = 0.0f) {
  EpiOut e;
  std::memset(&e, 0, sizeof(e));
  e.ptr = ptr;
  e.dtype = dt;
  e.ld = ld;
  e.bs = bs;
  e.transposed = transposed ? 1 : 0;
  e.gamma = gamma;
  return e;
}

// A direct fp32 output in the blocked layout (ld = padded width, bs = matrix size).
EpiOut out_blocked(float* ptr, int64_t ld, int64_t bs) {
  EpiOut e = out_to(ptr, DT_FP32, ld, bs, false);
  e.blocked = 1;
  return e;
}

// One class of a grouped launch: D (M x N) = epilogue(A_op * B_op^T).
//   A: rows M, cols K (K-major).
//   B: if !b_mn: rows N, cols K (K-major); if b_mn: rows K, cols N.
struct ClassSpec {
  Mat A, B;
  bool b_mn = false;
  bool symmetric = false;  // triangle schedule (M == N)
  bool mirror = false;     // symmetric: write exact mirrors (else upper 256-blocks only)
  bool a_sym = false;      // A is a symmetric matrix stored by upper 256-blocks
  bool b_sym = false;      // B likewise
  bool split = false;      // fp32-accurate: A and B are tf32 hi/lo planes (Mat.bs = plane stride)
  int bn = kBN;            // tile width (output columns per CTA pair): 256, or 128 (see pick_bn)
  int64_t c_plane = 0;     // > 0: C is split, lo plane at C + c_plane elements
  int64_t M = 0, N = 0, K = 0, batch = 0;
  float alpha = 1.0f, beta = 0.0f;
  const float* alpha_scale = nullptr;
  const float* beta_scale = nullptr;
  const void* C = nullptr;
  int c_dt = DT_FP32;
  int64_t ldc = 0, c_bs = 0;
  bool c_blocked = false;  // C is fp32 in the blocked layout
  const float* row_beta = nullptr;  // per-row term of the C coefficient (see ClassInfo)
  int64_t row_beta_bs = 0;
  std::vector<EpiOut> outs;
  // in-launch dependencies (see ClassInfo): row-block counters of earlier classes
  std::vector<RowDep> deps;
  int c_dep = -1;  // the entry of deps that produced C
  int* sig = nullptr;
  float* sumsq = nullptr;  // see ClassInfo
  int64_t sumsq_bs = 0;
  // split K (see ClassInfo): K slices [k_begin, k_begin + K) of a product of
  // inner dimension k_total (0: K), plus the other parts' partials to add
  int64_t k_begin = 0, k_total = 0;
  std::vector<const float*> addends;
  int64_t add_ld = 0, add_bs = 0;
};

// Tile order of large classes (see decode_tile): bands of kBand tile rows
// when one batch entry's operands exceed kBandBytes.
constexpr int kBand = 8;
constexpr double kBandBytes = 96.0 * (1 << 20);

// Square kBM x kBN tiles on or above the diagonal.
int64_t triangle_tiles(int64_t n) {
  const int64_t t = (n + kBN - 1) / kBN;
  return t * (t + 1) / 2;
}

int64_t class_tiles(const ClassSpec& s) {
  if (s.M <= 0 || s.N <= 0 || s.batch <= 0) return 0;
  const int64_t tm = (s.M + kBM - 1) / kBM, tn = (s.N + s.bn - 1) / s.bn;
  // symmetric: row block r keeps the column tiles from its diagonal 256-block on
  const int64_t per = s.symmetric ? tm * tn - (kBM / s.bn) * tm * (tm - 1) / 2 : tm * tn;
  return per * s.batch;
}

// Tile width of a product of an M x N output (batch entries): 128 where its
// 256-wide tiles would leave CTA pairs idle (fewer tiles than kPlanPairs),
// which halves each tile's MMA and epilogue time and doubles the tiles a
// dependent phase can spread over.  A symmetric output takes 128 only when
// every 256-row block holds two column tiles, so that each row block is
// touched by the same number of tiles.  From the shapes alone (kPlanPairs,
// not the device), like the split-K plans.
int pick_bn(int64_t M, int64_t N, int64_t batch, bool symmetric);

// Encodes and launches up to kMaxClasses classes of one operand dtype.
// `ordered`: the classes form a chain (later classes read earlier outputs
// through dep/sig counters) and keep their order; otherwise the longest
// reductions go first.
// `sched`: kSchedBytes of zeroed device memory for a dynamic tile schedule
// (null: static round robin).
msign_status launch_grouped(std::vector<ClassSpec> specs, int ab_dt, cudaStream_t stream, bool ordered = false,
                            void* sched = nullptr) {
  DeviceState* dev = nullptr;
  msign_status st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  specs.erase(std::remove_if(specs.begin(), specs.end(), [](const ClassSpec& s) { return class_tiles(s) == 0; }),
              specs.end());
  if (specs.empty()) return MSIGN_OK;
  if (specs.size() > static_cast<size_t>(kMaxClasses)) return MSIGN_ERR_UNSUPPORTED;
  // longest reduction first: its tiles are the longest-running work items
  if (!ordered)
    std::stable_sort(specs.begin(), specs.end(), [](const ClassSpec& a, const ClassSpec& b) { return a.K > b.K; });

  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  int64_t total = 0;
  for (size_t i = 0; i < specs.size(); ++i) {
    const ClassSpec& s = specs[i];
    GemmClass& c = p.cls[i];
    if (s.K <= 0 || s.outs.empty() || s.outs.size() > static_cast<size_t>(kMaxOuts)) return MSIGN_ERR_INVALID_ARG;
    if (s.symmetric && s.M != s.N) return MSIGN_ERR_INVALID_ARG;
    if (!tma_ok(s.A) || !tma_ok(s.B) || s.A.dt != ab_dt || s.B.dt != ab_dt) return MSIGN_ERR_UNSUPPORTED;
    if ((ab_dt == DT_FP32) != s.split) return MSIGN_ERR_INVALID_ARG;
    if (s.M > INT32_MAX || s.N > INT32_MAX || s.K > INT32_MAX || s.batch > 65535) return MSIGN_ERR_UNSUPPORTED;
    const int bke = kRowBytes / dtype_size(ab_dt);  // K elements per stage row
    const int64_t zb = s.split ? 2 * s.batch : s.batch;
    const int64_t kt = s.k_total > 0 ? s.k_total : s.K;  // the product's whole inner dimension
    if (s.k_begin < 0 || s.k_begin % kBM != 0 || s.k_begin + s.K > kt || s.addends.size() > kMaxAddends)
      return MSIGN_ERR_INVALID_ARG;
    Mat a = s.A;
    a.rows = s.M;
    a.cols = kt;
    if (!encode(&c.tmA, a, bke, kHalfM, zb)) return MSIGN_ERR_CUDA;
    if (s.a_sym && (s.M != kt || !encode(&c.tmA2, a, bke, bke, zb, true))) return MSIGN_ERR_INVALID_ARG;
    Mat b = s.B;
    if (s.b_sym) {
      if (s.b_mn || s.N != kt) return MSIGN_ERR_INVALID_ARG;
      b.rows = s.N;
      b.cols = kt;
      if (!encode(&c.tmB2, b, bke, bke, zb, true)) return MSIGN_ERR_CUDA;
    }
    if (!s.b_mn) {
      b.rows = s.N;
      b.cols = kt;
      if (!encode(&c.tmB, b, bke, s.bn / 2, zb)) return MSIGN_ERR_CUDA;
    } else {
      b.rows = kt;
      b.cols = s.N;
      if (!encode(&c.tmB, b, bke, bke, zb, true)) return MSIGN_ERR_CUDA;
    }
    ClassInfo& ci = c.info;
    ci.M = static_cast<int>(s.M);
    ci.N = static_cast<int>(s.N);
    ci.K = static_cast<int>(s.K);
    ci.batch = static_cast<int>(s.batch);
    ci.tiles_m = static_cast<int>((s.M + kBM - 1) / kBM);
    if (s.bn != kBN && (s.bn != kBN / 2 || (s.symmetric && ((s.N + s.bn - 1) / s.bn) % 2 != 0) || s.sumsq != nullptr))
      return MSIGN_ERR_INVALID_ARG;
    ci.bn = s.bn;
    ci.tiles_n = static_cast<int>((s.N + s.bn - 1) / s.bn);
    ci.tiles_per_batch = static_cast<int>(class_tiles(s) / s.batch);
    ci.tile_begin = static_cast<int>(total);
    ci.symmetric = s.symmetric ? 1 : 0;
    {
      // operands of one batch entry larger than about 3/4 of the L2: walk the
      // tiles in bands of 8 tile rows so that a wave's operands stay in L2
      // (measured: the row-by-row order re-read X 5x from DRAM in 8192^2 X X^T)
      const double fp = static_cast<double>(dtype_size(ab_dt)) * (s.split ? 2.0 : 1.0) *
                        (static_cast<double>(s.M) * kt + (s.A.ptr == s.B.ptr ? 0.0 : static_cast<double>(s.N) * kt));
      ci.group = (fp > kBandBytes && s.bn == kBN) ? kBand : 1;
    }
    ci.mirror = (s.symmetric && s.mirror) ? 1 : 0;
    ci.a_sym = s.a_sym ? 1 : 0;
    ci.b_sym = s.b_sym ? 1 : 0;
    ci.b_mn_major = s.b_mn ? 1 : 0;
    ci.split = s.split ? 1 : 0;
    ci.c_plane = s.c_plane;
    ci.num_out = static_cast<int>(s.outs.size());
    ci.alpha = s.alpha;
    ci.beta = s.beta;
    ci.alpha_scale = s.alpha_scale;
    ci.beta_scale = s.beta_scale;
    ci.C = s.C;
    ci.c_dtype = s.c_dt;
    ci.ldc = s.ldc;
    ci.c_bs = s.c_bs;
    ci.c_blocked = s.c_blocked ? 1 : 0;
    ci.row_beta = s.row_beta;
    ci.row_beta_bs = s.row_beta_bs;
    if (s.c_blocked && (s.c_dt != DT_FP32 || s.c_plane != 0 || s.symmetric || s.ldc % 32 != 0))
      return MSIGN_ERR_INVALID_ARG;
    for (const EpiOut& e : s.outs)
      if (e.blocked && (e.dtype != DT_FP32 || e.transposed || e.ld % 32 != 0)) return MSIGN_ERR_INVALID_ARG;
    for (size_t o = 0; o < s.outs.size(); ++o) {
      EpiOut& e = ci.out[o];
      e = s.outs[o];
      // 16-bit row-major outputs leave by staged bulk stores where the
      // buffer's address and strides allow a tensor map (16-byte multiples);
      // the rest, and transposed outputs of symmetric classes, by lane stores
      e.tma = 0;
      if (!e.blocked && (e.dtype == DT_BF16 || e.dtype == DT_FP16) && !(e.transposed && s.symmetric)) {
        Mat d{e.ptr, e.dtype, e.transposed ? s.N : s.M, e.transposed ? s.M : s.N, e.ld, e.bs};
        if (s.batch == 1) d.bs = d.rows * d.ld;
        if (d.ld >= d.cols && d.bs > 0 && tma_ok(d) && encode_out(&c.tmOut[o], d, s.batch)) e.tma = 1;
      }
    }
    if (s.deps.size() > static_cast<size_t>(kMaxDeps) || s.c_dep >= static_cast<int>(s.deps.size()))
      return MSIGN_ERR_INVALID_ARG;
    for (size_t e = 0; e < s.deps.size(); ++e) ci.deps[e] = s.deps[e];
    ci.num_deps = static_cast<int>(s.deps.size());
    ci.c_dep = s.c_dep;
    ci.sig = s.sig;
    ci.sumsq = s.sumsq;
    ci.sumsq_bs = s.sumsq_bs;
    ci.k_begin = static_cast<int>(s.k_begin);
    ci.num_addends = static_cast<int>(s.addends.size());
    for (size_t e = 0; e < s.addends.size(); ++e) ci.addend[e] = s.addends[e];
    ci.add_ld = s.add_ld;
    ci.add_bs = s.add_bs;
    if (s.sumsq != nullptr && !s.symmetric) return MSIGN_ERR_INVALID_ARG;
    total += class_tiles(s);
  }
  if (total > INT32_MAX) return MSIGN_ERR_UNSUPPORTED;
  p.num_classes = static_cast<int>(specs.size());
  p.total_tiles = static_cast<int>(total);
  const uint32_t fmt = (ab_dt == DT_BF16) ? 1u : (ab_dt == DT_FP16 ? 0u : 2u);  // bf16, f16 or tf32
  p.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (static_cast<uint32_t>(kBN >> 3) << 17) |
            (static_cast<uint32_t>(kBM >> 4) << 24);
  p.err = dev->err;
  p.timeout_ns = kWaitLimitNs;
  if (sched != nullptr && dev->max_pairs <= kMaxSchedPairs) {
    p.claim = static_cast<int*>(sched);
    p.ring = reinterpret_cast<unsigned long long*>(static_cast<char*>(sched) + 256);
  }
  // one CTA pair per co-resident cluster slot, never more pairs than tiles
  const int grid = 2 * static_cast<int>(std::min<int64_t>(total, dev->max_pairs));
  double flops = 0.0, bytes = 0.0;
  for (const ClassSpec& s : specs) {
    const double bt = static_cast<double>(s.batch);
    // useful FLOPs: the triangle only for symmetric outputs
    flops += s.symmetric ? bt * s.K * static_cast<double>(s.M) * (s.M + 1) : bt * 2.0 * s.M * s.N * s.K;
    // compulsory traffic: both operands once, C once, every output once
    const double es = dtype_size(s.A.dt);
    bytes += bt * es * (static_cast<double>(s.M) * s.K + (s.A.ptr == s.B.ptr ? 0.0 : static_cast<double>(s.N) * s.K));
    if (s.C) bytes += bt * dtype_size(s.c_dt) * static_cast<double>(s.M) * s.N;
    for (const EpiOut& e : s.outs)
      bytes += bt * dtype_size(e.dtype) * static_cast<double>(s.M) * s.N * (s.symmetric ? 0.5 : 1.0);
  }
  if (ab_dt == DT_FP32) flops *= 3.0;  // three tf32 products per fp32-accurate product
  prof_begin(stream);
  // the kernel built with per-class tile widths only where a class is narrow
  bool narrow = false;
  for (const ClassSpec& s : specs) narrow = narrow || s.bn != kBN;
  // a programmatic dependent launch: the CTAs set up while the previous
  // kernel drains, then wait for it (griddepcontrol.wait in the kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (ab_dt == DT_FP32)
    (void)cudaLaunchKernelEx(&cfg, narrow ? gemm_sm100_kernel<true, true> : gemm_sm100_kernel<true, false>, p);
  else
    (void)cudaLaunchKernelEx(&cfg, narrow ? gemm_sm100_kernel<false, true> : gemm_sm100_kernel<false, false>, p);
  prof_end(0, stream, flops, bytes);
  return cudaGetLastError() == cudaSuccess ? MSIGN_OK : MSIGN_ERR_CUDA;
}

msign_status launch_ok() { return cudaGetLastError() == cudaSuccess ? MSIGN_OK : MSIGN_ERR_CUDA; }

// The failure path of every bounded wait, made to fire on purpose: one
// thread waits on an mbarrier that no one arrives on and on a counter that
// no one increments.  Each wait gives up after limit_ns, sets the device
// error word and returns; the kernel then ends normally.
__device__ int g_never_signalled = 0;

__global__ void selftest_timeout_kernel(int* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  (void)wait_bounded(&bar, 0, nullptr, err, limit_ns);
  (void)wait_counter(&g_never_signalled, 1, nullptr, err, limit_ns);
}

// Frobenius normalisation factor of every matrix of a batch into scale[].
// Matrix b of the batch starts at element b * bs of `in`.
msign_status launch_norm(const void* in, int in_dt, int64_t per, int64_t bs, int64_t batch, int cast_dt, float eps,
                         int mode, float* partials, float* scale, cudaStream_t stream) {
  const int parts = norm_parts(per);
  dim3 g(static_cast<unsigned>(parts), static_cast<unsigned>(batch));
  prof_begin(stream);
  sumsq_partial_kernel<<<g, kNormThreads, 0, stream>>>(in, in_dt, per, bs, cast_dt, partials);
  prof_end(1, stream, 0.0, static_cast<double>(batch) * per * dtype_size(in_dt));
  prof_begin(stream);
  norm_finalize_kernel<<<static_cast<unsigned>(batch), 1024, 0, stream>>>(partials, parts, eps, mode, scale);
  prof_end(1, stream, 0.0, static_cast<double>(batch) * parts * 4);
  return launch_ok();
}

// Launches ingest_kernel over `batch` matrices (see IngestArgs).
msign_status launch_ingest(const IngestArgs& a, int64_t batch, cudaStream_t stream) {
  const int64_t n = a.transpose ? a.cols : a.rows, m = a.transpose ? a.rows : a.cols;
  if (a.G != nullptr && a.in_dt != DT_FP32) return MSIGN_ERR_INVALID_ARG;
  const double e = static_cast<double>(batch) * a.rows * a.cols;
  double bytes = e * (dtype_size(a.in_dt) + dtype_size(a.op_dt) * (a.op_dt == DT_TF32_HI ? 2 : 1));
  if (a.master) bytes += e * 4;
  if (a.G) bytes += e * (dtype_size(a.g_dt) + 4);
  DeviceState* dev = nullptr;
  msign_status st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  // one full wave of resident blocks over the whole batch, grid-striding
  // over the tiles: no partial last wave
  const int64_t tiles = ceil_div(n, 32) * ceil_div(m, 64);
  const int64_t wave = std::max<int64_t>(1, dev->ingest_blocks / std::max<int64_t>(batch, 1));
  dim3 g(static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>({tiles, wave, int64_t(kIngestParts)}))),
         static_cast<unsigned>(batch));
  prof_begin(stream);
  ingest_kernel<<<g, dim3(32, 8), 0, stream>>>(a);
  prof_end(2, stream, 0.0, bytes);
  return launch_ok();
}

// Ingest arguments with everything optional left off.
IngestArgs ingest_args(const void* in, int in_dt, int64_t rows, int64_t cols, bool transpose, int cast_dt, void* xop,
                       int op_dt, int64_t ld_op, int64_t op_bs) {
  IngestArgs a;
  std::memset(&a, 0, sizeof(a));
  a.in = const_cast<void*>(in);
  a.in_dt = in_dt;
  a.rows = static_cast<int>(rows);
  a.cols = static_cast<int>(cols);
  a.transpose = transpose ? 1 : 0;
  a.cast_dt = cast_dt;
  a.xop = xop;
  a.op_dt = op_dt;
  a.ld_op = ld_op;
  a.op_bs = op_bs;
  return a;
}

// ---------------------------------------------------------------- msign_ns plan

struct NsBuffers {
  float* partials;
  float* scale;   // s per matrix, then s^2 per matrix
  void* P[2];     // bf16 operand copies of X (n x ldm)
  float* master;  // fp32 X, blocked layout (blk_ld(m) wide, blk_size(n, m) per matrix)
  void* A;        // bf16 n x ldn
  void* B;        // bf16 n x ldn (zero diagonal; the diagonal is in `diag`)
  float* diag;    // fp32 diagonal of B, n per matrix
  float* sumsq;   // sharper initial normalisation: ||A^2||_F^2 partials, [batch][tiles^2][kTileSignals]
  float* scale_n; // and the step-0 factor s / n per matrix
  int syrk_parts;  // K parts of the X X^T product (see syrk_parts()), 1 = whole
  float* part[kMaxAddends];  // their fp32 partials (blocked), parts - 1 of them
  int* cnt;       // state zeroed before use: kSchedBytes of dynamic-schedule state,
                  // the ingest tickets (ns_tickets(batch) ints), then the row-block
                  // counters of a chained launch [kChainSteps][3 phases][batch][tiles]
};

inline int64_t ns_tickets(int64_t batch) { return round_up(batch, 64); }
inline int* ns_ticket_ptr(const NsBuffers& w) { return w.cnt + kSchedBytes / sizeof(int); }
inline int* ns_counter_base(const NsBuffers& w, int64_t batch) { return ns_ticket_ptr(w) + ns_tickets(batch); }
// Bytes of the state region in use with `items` chained phases.
inline size_t state_bytes(int64_t batch, int64_t n, int items) {
  return kSchedBytes + sizeof(int) * (ns_tickets(batch) + items * batch * ceil_div(n, kBM));
}

// CTA pairs the split-K plan assumes (a B200: 148 SMs).  The plan must not
// depend on the device, because the workspace size is a host-only query.
constexpr int kPlanPairs = 74;

int pick_bn(int64_t M, int64_t N, int64_t batch, bool symmetric) {
  ClassSpec s;
  s.M = M, s.N = N, s.batch = batch, s.symmetric = symmetric;
  if (class_tiles(s) >= kPlanPairs) return kBN;
  if (symmetric && ceil_div(N, kBN / 2) % 2 != 0) return kBN;
  return kBN / 2;
}

// K parts of the X X^T product (K = m) of a class whose triangle tiles
// leave CTA pairs idle: whole 256-blocks, each at least 4096 long.  In the
// chained iteration the split pays only there: measured on 1 x 2048 x 4096
// (two parts of 2048) it was 9% slower, on 1 x 1024 x 16384 (four parts of
// 4096) 16% faster.
inline int syrk_parts(int64_t batch, int64_t n, int64_t m) {
  const int64_t want = std::min<int64_t>({kMaxAddends + 1,
                                          std::max<int64_t>(1, kPlanPairs / std::max<int64_t>(1, triangle_tiles(n) * batch)),
                                          std::max<int64_t>(1, m / 4096)});
  return static_cast<int>(ceil_div(m, round_up(ceil_div(m, want), kBM)));
}
inline int64_t syrk_part_len(int64_t m, int parts) { return round_up(ceil_div(m, parts), kBM); }

// fp32: the operand copies P, A and B hold two fp32 planes (tf32 hi, lo)
// per matrix, [batch][plane][rows][ld].
void carve_ns(Carver& cv, int64_t batch, int64_t n, int64_t m, NsBuffers* b, bool fp32 = false) {
  const int64_t ldm = round_up(m, 8), ldn = round_up(n, 8);
  const uint64_t op = fp32 ? 8ull : 2ull;  // bytes per operand element (two fp32 planes, or bf16)
  b->partials = static_cast<float*>(cv.take(sizeof(float) * kNormParts * batch));
  b->scale = static_cast<float*>(cv.take(sizeof(float) * 2 * batch));
  b->P[0] = cv.take(op * batch * n * ldm);
  b->P[1] = cv.take(op * batch * n * ldm);
  b->master = static_cast<float*>(cv.take(4ull * batch * blk_size(n, m)));
  b->A = cv.take(op * batch * n * ldn);
  b->B = cv.take(op * batch * n * ldn);
  b->diag = static_cast<float*>(cv.take(sizeof(float) * batch * n));
  b->sumsq = static_cast<float*>(cv.take(sizeof(float) * batch * ceil_div(n, kBM) * ceil_div(n, kBM) * kTileSignals));
  b->scale_n = static_cast<float*>(cv.take(sizeof(float) * batch));
  b->syrk_parts = fp32 ? 1 : syrk_parts(batch, n, m);
  for (int q = 0; q < kMaxAddends; ++q)
    b->part[q] = q + 1 < b->syrk_parts ? static_cast<float*>(cv.take(4ull * batch * blk_size(n, n))) : nullptr;
  b->cnt = static_cast<int*>(cv.take(state_bytes(batch, n, kMaxClasses)));
}

// Launches a list of classes of one operand dtype, kMaxClasses at a time.
msign_status launch_all(const std::vector<ClassSpec>& specs, int ab_dt, cudaStream_t stream) {
  for (size_t i = 0; i < specs.size(); i += kMaxClasses) {
    std::vector<ClassSpec> chunk(specs.begin() + i, specs.begin() + std::min(specs.size(), i + kMaxClasses));
    msign_status st = launch_grouped(chunk, ab_dt, stream);
    if (st != MSIGN_OK) return st;
  }
  return MSIGN_OK;
}

// One shape class of a standard-NS run: `batch` oriented n x m matrices.
struct NsClass {
  NsBuffers w;
  int64_t batch, n, m;
  std::vector<EpiOut> final_outs;  // outputs of the last step's B X product
  bool fp32 = false;               // fp32-accurate products (3xTF32 on split planes)
  int op_dt = DT_BF16;             // 16-bit operand type otherwise (bf16 or fp16)
  // set when P[0] and master hold the unscaled x (fused ingest): the first
  // step applies X0 = s x through its epilogues (s^2 on X X^T, s on a X + B X)
  const float* s = nullptr;
  const float* s2 = nullptr;
  bool improved = false;  // sharper step-0 normalisation (Schedule::init)
  // the first step's a X term reads the 16-bit operand copy P[0] instead of
  // the fp32 master: the fused ingest writes the unscaled x rounded to the
  // operand type, which the copy holds exactly, so the ingest skips the
  // master and the first B X epilogue writes it
  bool c0_op = false;
};

// Hi and lo plane outputs of a split matrix at `p` (planes of `plane` elements).
std::vector<EpiOut> split_out(void* p, int64_t ld, int64_t plane) {
  return {out_to(p, DT_TF32_HI, ld, 2 * plane, false),
          out_to(static_cast<char*>(p) + 4 * plane, DT_TF32_LO, ld, 2 * plane, false)};
}

// The three products of one NS step ([P2] eq. 6, left form) for one class:
//   SYRK   A = X X^T                  (symmetric, upper 256-blocks)
//   SQR    B = b A + c A A            (symmetric; A A = A A^T as A = A^T),
//                                      stored as E = B - diag(B) plus the
//                                      diagonal d in fp32
//   BX     X' = E X~ + (a + d) . X    (d scales the rows of the fp32 copy X;
//                                      X~ is its rounding, the MMA operand)
// which is a X + B X.  Near convergence B is close to (b + c) I, about -2.7
// I for Jordan's triple, while a X + B X is about 0.7 X: stored in bf16, the
// diagonal's rounding would be amplified about 4x in the result.  Keeping
// it in fp32 leaves only the small off-diagonal part to bf16, and X~ is
// multiplied by that part only, so rounding noise never reaches the null
// space of X (zero singular values stay zero).  Against the fp64 iteration
// this lowers the largest error over the test matrices (Gaussian, rank-one,
// momentum-like) from 2.2e-2 to 1.2e-2 with bf16 operands.  The
// fp32-accurate class runs the plain products on tf32 hi/lo planes.
void ns_specs(const NsClass& k, int cur, float a, float b, float c, bool first, bool last, ClassSpec* syrk,
              ClassSpec* sqr, ClassSpec* bx) {
  const int64_t n = k.n, m = k.m, ldm = round_up(m, 8), ldn = round_up(n, 8);
  const int od = k.fp32 ? DT_FP32 : k.op_dt;
  const bool sp = k.fp32;
  const int64_t pm = n * ldm, pn = n * ldn;        // matrix (or plane) strides
  const int64_t zn = sp ? 2 * pn : pn;             // batch stride of A and B
  const Mat X{k.w.P[cur], od, n, m, ldm, pm};
  const Mat A{k.w.A, od, n, n, ldn, pn};
  const Mat B{k.w.B, od, n, n, ldn, pn};
  auto outs = [&](void* p, int64_t ld, int64_t plane) {
    return sp ? split_out(p, ld, plane) : std::vector<EpiOut>{out_to(p, od, ld, plane, false)};
  };
  ClassSpec& s = *syrk;
  s = ClassSpec();
  s.A = X, s.B = X, s.symmetric = true, s.split = sp;
  // 128-wide tiles where 256-wide ones would leave CTA pairs idle (X X^T
  // split in K parts keeps 256); step 0's A A of the sharper normalisation
  // keeps 256 for its per-tile sums of squares
  s.bn = k.w.syrk_parts > 1 ? kBN : pick_bn(n, n, k.batch, true);
  s.M = n, s.N = n, s.K = m, s.batch = k.batch;
  s.outs = outs(k.w.A, ldn, pn);

  ClassSpec& q = *sqr;  // both operands read from A's upper blocks
  q = ClassSpec();
  q.A = A, q.B = A, q.symmetric = true, q.a_sym = true, q.b_sym = true, q.split = sp;
  q.bn = (first && k.improved) ? kBN : pick_bn(n, n, k.batch, true);
  q.M = n, q.N = n, q.K = n, q.batch = k.batch;
  q.alpha = c, q.beta = b;
  q.C = k.w.A, q.c_dt = od, q.ldc = ldn, q.c_bs = zn, q.c_plane = sp ? pn : 0;
  q.outs = outs(k.w.B, ldn, pn);
  if (!sp) q.outs[0].diag = k.w.diag, q.outs[0].diag_bs = n;

  ClassSpec& x = *bx;  // B read from its upper blocks
  x = ClassSpec();
  x.A = B, x.a_sym = true, x.B = X, x.b_mn = true, x.split = sp;
  x.bn = pick_bn(n, m, k.batch, false);
  x.M = n, x.N = m, x.K = n, x.batch = k.batch;
  x.alpha = 1.0f, x.beta = a;
  if (!sp) x.row_beta = k.w.diag, x.row_beta_bs = n;
  x.C = k.w.master, x.c_dt = DT_FP32, x.ldc = blk_ld(m), x.c_bs = blk_size(n, m), x.c_blocked = true;
  if (first && k.c0_op && !sp) x.C = k.w.P[cur], x.c_dt = k.op_dt, x.ldc = ldm, x.c_bs = pm, x.c_blocked = false;
  if (!last) {
    x.outs = outs(k.w.P[cur ^ 1], ldm, pm);
    x.outs.insert(x.outs.begin(), out_blocked(k.w.master, blk_ld(m), blk_size(n, m)));
  } else {
    x.outs = k.final_outs;
  }
  if (first && k.s != nullptr) {
    s.alpha_scale = k.s2;
    x.alpha_scale = k.s;
    x.beta_scale = k.s;
  }
  if (first && k.improved) {
    // step 0 of the sharper normalisation: the SQR product stores A^2 itself
    // (and the partials of ||A^2||_F^2); improved_init_kernel then forms B,
    // and B X runs with X0 / n, i.e. with s / n on both of its terms
    q.alpha = 1.0f, q.beta = 0.0f, q.C = nullptr;
    q.sumsq = k.w.sumsq, q.sumsq_bs = ceil_div(n, kBM) * ceil_div(n, kBM) * kTileSignals;
    x.alpha_scale = k.w.scale_n;
    x.beta_scale = k.w.scale_n;
  }
}

// Operand dtype of a class's products.
int ns_op_dt(const NsClass& k) { return k.fp32 ? DT_FP32 : k.op_dt; }

// Between step 0's SQR (which stored A^2) and its B X product: the sharper
// normalisation's B and s / n (improved_init_kernel).
msign_status launch_improved_init(const NsClass& k, const Schedule& sch, cudaStream_t stream) {
  const int64_t nb = ceil_div(k.n, kBM), ldn = round_up(k.n, 8);
  dim3 g(static_cast<unsigned>(nb * nb), static_cast<unsigned>(k.batch), 8);
  prof_begin(stream);
  improved_init_kernel<<<g, 256, 0, stream>>>(k.w.A, k.w.B, k.op_dt, k.w.diag, ldn, k.n * ldn, static_cast<int>(k.n),
                                              static_cast<int>(nb), k.w.sumsq, nb * nb * kTileSignals, kTileSignals, sch.abc[1], sch.abc[2],
                                              sch.eps, k.s, k.w.scale_n);
  prof_end(3, stream, 0.0, static_cast<double>(k.batch) * k.n * k.n * 3.0);
  return launch_ok();
}

// One NS step as three launches (one per phase), each over all classes.
msign_status ns_step(const std::vector<NsClass>& cls, const Schedule& sch, int cur, float a, float b, float c,
                     bool first, bool last, cudaStream_t stream) {
  std::vector<ClassSpec> ph[3];
  std::vector<int> dts;
  for (const NsClass& k : cls)
    if (std::find(dts.begin(), dts.end(), ns_op_dt(k)) == dts.end()) dts.push_back(ns_op_dt(k));
  for (int p = 0; p < 3; ++p)
    for (int dt : dts) {
      std::vector<ClassSpec> v;
      for (const NsClass& k : cls) {
        if (ns_op_dt(k) != dt) continue;
        ClassSpec sp[3];
        ns_specs(k, cur, a, b, c, first, last, &sp[0], &sp[1], &sp[2]);
        v.push_back(sp[p]);
      }
      msign_status st = launch_all(v, dt, stream);
      if (st != MSIGN_OK) return st;
      if (p == 1 && first)
        for (const NsClass& k : cls)
          if (k.improved && ns_op_dt(k) == dt) {
            st = launch_improved_init(k, sch, stream);
            if (st != MSIGN_OK) return st;
          }
    }
  return MSIGN_OK;
}

// Runs all steps of the schedule on classes whose P[0] / master already hold X0.
//
// When every class shares one operand dtype and 3 x classes x steps fit in
// one launch, up to kChainSteps steps run as ONE launch: the classes are the
// phases in order, and each phase's tiles wait only for the row blocks they
// read (SYRK on rows tm, tn of X; SQR on rows tm, tn of A; BX on row tm of
// B) instead of for the whole previous phase.  This removes the launch gaps
// and lets the last wave of one phase overlap the first tiles of the next.
//   The write-after-read hazards of the reused buffers are covered by the
// same counters: a tile that overwrites A, B or an X copy transitively waits
// for every reader of the old contents (e.g. SYRK of step t+1 on A[i][j]
// needs B rows i and j of step t, i.e. every SQR tile that read A rows i, j).
//   `zeroed`: the classes' state regions were zeroed for this call (and only
// the tickets used since), so the first chained launch needs no memset.
// msign_set_chaining(0): every phase as a launch of its own (diagnostics)
std::atomic<int> g_chaining{1};

msign_status ns_iterate(const std::vector<NsClass>& cls, const Schedule& sch, cudaStream_t stream,
                        bool zeroed = false) {
  const int T = sch.steps();
  const int ncls = static_cast<int>(cls.size());
  bool uniform = !cls.empty(), improved = false;
  for (const NsClass& k : cls) uniform = uniform && ns_op_dt(k) == ns_op_dt(cls.front()), improved |= k.improved;
  // classes a phase takes in a launch: X X^T may run as several K parts
  auto phase_classes = [&](int p) {
    int c = 0;
    for (const NsClass& k : cls) c += p == 0 ? k.w.syrk_parts : 1;
    return c;
  };
  const bool chained = g_chaining.load() != 0 && uniform && std::max({phase_classes(0), phase_classes(1), phase_classes(2)}) <= kMaxClasses &&
                       3 * ncls <= kMaxClasses;
  if (!chained) {
    for (int t = 0; t < T; ++t) {
      msign_status st = ns_step(cls, sch, t & 1, sch.abc[3 * t], sch.abc[3 * t + 1], sch.abc[3 * t + 2], t == 0,
                                t == T - 1, stream);
      if (st != MSIGN_OK) return st;
    }
    return MSIGN_OK;
  }
  // The phases (t, p) in order, p = 0 SYRK, 1 SQR, 2 BX, packed into chained
  // launches of at most kMaxClasses classes.  With the sharper normalisation
  // the first launch ends after step 0's SQR, and improved_init_kernel runs
  // before the launch that starts with step 0's B X.
  const int total = 3 * T;
  for (int i = 0; i < total;) {
    int j = i, used = 0;
    while (j < total && used + phase_classes(j % 3) <= kMaxClasses) {
      used += phase_classes(j % 3);
      ++j;
      if (improved && j - 1 == 1) break;  // just placed step 0's SQR
    }
    if (!(zeroed && i == 0))
      for (const NsClass& k : cls)
        if (cudaMemsetAsync(k.w.cnt, 0, state_bytes(k.batch, k.n, used), stream) != cudaSuccess) return MSIGN_ERR_CUDA;
    std::vector<ClassSpec> chain;
    std::vector<int> slots(cls.size(), 0);                // next counter slot of each class
    std::vector<std::vector<int>> done(cls.size());       // counter slot of each phase's final class
    for (int it = i; it < j; ++it) {
      const int t = it / 3, p = it % 3;
      for (size_t ci = 0; ci < cls.size(); ++ci) {
        const NsClass& k = cls[ci];
        ClassSpec sp[3];
        ns_specs(k, t & 1, sch.abc[3 * t], sch.abc[3 * t + 1], sch.abc[3 * t + 2], t == 0, t == T - 1, &sp[0], &sp[1],
                 &sp[2]);
        ClassSpec q = sp[p];
        const int64_t rb = ceil_div(k.n, kBM);  // 256-row blocks of X, A and B
        int* const base = ns_counter_base(k.w, k.batch);
        auto ctr = [&](int slot) { return base + static_cast<int64_t>(slot) * k.batch * rb; };
        const int rows = static_cast<int>(rb);
        // arrivals that complete a row block of a phase's output: kTileSignals
        // per tile touching it, i.e. per column tile of the phase's width
        auto per_block = [&](int ph) {
          return static_cast<int>(kTileSignals * ceil_div(ph == 2 ? k.m : k.n, sp[ph].bn));
        };
        const int per_block_sym = per_block(0);  // the X X^T parts below
        // the phase this one reads: the previous one in the order (the B X of
        // the step before has the same shape and tile width as this step's)
        std::vector<RowDep> reads;
        if (it - 1 >= i) {
          const int ps = done[ci][it - 1 - i];
          if (p == 0) reads = {RowDep{ctr(ps), rows, per_block(2), DEP_TM | DEP_TN}};
          if (p == 1) reads = {RowDep{ctr(ps), rows, per_block(0), DEP_TM | DEP_TN}};
          if (p == 2) reads = {RowDep{ctr(ps), rows, per_block(1), DEP_TM}};
        }
        if (p == 0 && k.w.syrk_parts > 1) {
          // split K (see Chain::add_split): parts 0 .. P-2 store fp32
          // partials, the final part adds them in its epilogue
          const int P = k.w.syrk_parts;
          const int64_t len = syrk_part_len(k.m, P);
          std::vector<RowDep> epi;
          for (int qq = 0; qq + 1 < P; ++qq) {
            ClassSpec c;
            c.A = q.A, c.B = q.B, c.symmetric = true, c.split = q.split, c.bn = q.bn;
            c.M = q.M, c.N = q.N, c.batch = q.batch;
            c.K = len, c.k_begin = qq * len, c.k_total = k.m;
            c.outs = {out_blocked(k.w.part[qq], blk_ld(k.n), blk_size(k.n, k.n))};
            c.deps = reads;
            c.sig = ctr(slots[ci]);
            epi.push_back(RowDep{ctr(slots[ci]), rows, per_block_sym, DEP_EPI | DEP_TM | DEP_TN});
            ++slots[ci];
            chain.push_back(c);
          }
          q.k_begin = (P - 1) * len, q.K = k.m - q.k_begin, q.k_total = k.m;
          for (int qq = 0; qq + 1 < P; ++qq) q.addends.push_back(k.w.part[qq]);
          q.add_ld = blk_ld(k.n), q.add_bs = blk_size(k.n, k.n);
          reads.insert(reads.end(), epi.begin(), epi.end());
        }
        q.deps = reads;
        q.c_dep = (q.C != nullptr && p != 0 && it - 1 >= i) ? 0 : -1;
        q.sig = ctr(slots[ci]);
        done[ci].push_back(slots[ci]++);
        chain.push_back(q);
      }
    }
    // dynamic schedule state: the first class's area (zeroed with its counters)
    msign_status st = launch_grouped(chain, ns_op_dt(cls.front()), stream, /*ordered=*/true, cls.front().w.cnt);
    if (st != MSIGN_OK) return st;
    if (improved && j == 2)
      for (const NsClass& k : cls)
        if (k.improved) {
          st = launch_improved_init(k, sch, stream);
          if (st != MSIGN_OK) return st;
        }
    i = j;
  }
  return MSIGN_OK;
}

// ---------------------------------------------------------------- gram_ns plan

struct GramBuffers {
  float* partials;
  float* scale;
  void* P[2];  // fp16 X (n x ldm)
  void* R;     // fp16 n x ldn
  void* Z;
  void* Q[2];
  void* RZ;
  int* cnt;  // zeroed before each chained launch: kSchedBytes of schedule state, then the
             // row-block counters of up to kMaxClasses classes [class][batch][tiles]
  float* part[kMaxAddends];  // split-K partials of n x n products (blocked fp32)
};

// K parts of a Gram-NS symmetric product of inner dimension K (see
// Chain::add_split): only where the triangle tiles leave CTA pairs idle, each
// part at least 2048 of K (measured: with shorter parts the extra
// partial-store epilogue costs more than the mainloop saves; 2048 x 16384
// gains 6%, the n x n products of K = n <= 2048 stay whole).  Planned from
// the shape alone, like syrk_parts, so the workspace query stays host-only.
inline int gram_parts(int64_t batch, int64_t n, int64_t K) {
  const int64_t want = std::min<int64_t>({kMaxAddends + 1,
                                          std::max<int64_t>(1, kPlanPairs / std::max<int64_t>(1, triangle_tiles(n) * batch)),
                                          std::max<int64_t>(1, K / 2048)});
  const int64_t len = round_up(ceil_div(K, want), kBM);
  return static_cast<int>(std::min<int64_t>(ceil_div(K, len), kMaxAddends + 1));
}

void carve_gram(Carver& cv, int64_t batch, int64_t n, int64_t m, GramBuffers* b) {
  const int64_t ldm = round_up(m, 8), ldn = round_up(n, 8);
  b->partials = static_cast<float*>(cv.take(sizeof(float) * kNormParts * batch));
  b->scale = static_cast<float*>(cv.take(sizeof(float) * batch));
  b->P[0] = cv.take(2ull * batch * n * ldm);
  b->P[1] = cv.take(2ull * batch * n * ldm);
  b->R = cv.take(2ull * batch * n * ldn);
  b->Z = cv.take(2ull * batch * n * ldn);
  b->Q[0] = cv.take(2ull * batch * n * ldn);
  b->Q[1] = cv.take(2ull * batch * n * ldn);
  b->RZ = cv.take(2ull * batch * n * ldn);
  b->cnt = static_cast<int*>(cv.take(kSchedBytes + sizeof(int) * kMaxClasses * batch * ceil_div(n, kBM)));
  // fp32 partials for the split products: K is m (X X^T) or n (n x n)
  const int parts = std::max(gram_parts(batch, n, m), gram_parts(batch, n, n));
  for (int q = 0; q < kMaxAddends; ++q)
    b->part[q] = q + 1 < parts ? static_cast<float*>(cv.take(4ull * batch * blk_size(n, n))) : nullptr;
}

// Classes of one chained launch whose dependencies are derived from the
// buffers they read and write, by 256-row block (see RowDep):
//   read after write  -- the producer's rows the consumer tile reads: row tm
//                        of an A operand, row tn of a K-major B operand, all
//                        rows of an MN-major one (X in Q X), row tm for C;
//   write after read  -- every earlier reader of the buffer being
//                        overwritten, on the rows of the written tile (tm,
//                        and tn for a symmetric output), or on all its rows
//                        when that reader read the buffer MN-major;
//   write after write -- the buffer's previous writer, on the same rows.
// A class waits only for classes before it, so the launch cannot deadlock.
// When a launch would exceed kMaxClasses, the chain is launched and
// restarted: stream order covers everything across launches.
struct Chain {
  struct Use {
    int cls, mode;
  };
  struct Buf {
    int writer = -1;
    std::vector<Use> readers;
  };
  int* state;  // kSchedBytes + counters
  int64_t batch, rows;
  int ab_dt;
  cudaStream_t stream;
  std::vector<ClassSpec> cls;
  std::vector<int> target;  // per class: 8 x tiles touching a row block
  std::vector<std::pair<const void*, Buf>> bufs;

  Buf& buf(const void* p) {
    for (auto& b : bufs)
      if (b.first == p) return b.second;
    bufs.push_back({p, Buf{}});
    return bufs.back().second;
  }
  int* counters(int c) { return state + kSchedBytes / sizeof(int) + static_cast<int64_t>(c) * batch * rows; }

  msign_status flush() {
    if (cls.empty()) return MSIGN_OK;
    const size_t bytes = kSchedBytes + sizeof(int) * cls.size() * batch * rows;
    if (cudaMemsetAsync(state, 0, bytes, stream) != cudaSuccess) return MSIGN_ERR_CUDA;
    msign_status st = launch_grouped(cls, ab_dt, stream, /*ordered=*/true, state);
    cls.clear();
    target.clear();
    bufs.clear();
    return st;
  }

  // reads: (buffer, DEP_TM / DEP_TN / DEP_ALL, plus DEP_EPI when only the
  // epilogue reads it); c_buf: the buffer read as C.  Reads are waited for
  // before the mainloop; write-after-read and write-after-write orders only
  // before the epilogue stores (DEP_EPI), so the mainloop starts early.
  msign_status add(ClassSpec s, const std::vector<std::pair<const void*, int>>& reads, const void* c_buf,
                   const std::vector<const void*>& writes) {
    if (cls.size() == static_cast<size_t>(kMaxClasses)) {
      msign_status st = flush();
      if (st != MSIGN_OK) return st;
    }
    const int me = static_cast<int>(cls.size());
    std::vector<std::pair<int, int>> need;  // (class, mode): one entry per class and DEP_EPI kind
    auto want = [&](int c, int mode) {
      for (auto& n : need)
        if (n.first == c && (n.second & DEP_EPI) == (mode & DEP_EPI)) {
          n.second |= mode;
          return;
        }
      need.push_back({c, mode});
    };
    const int out_rows = s.symmetric ? (DEP_TM | DEP_TN) : DEP_TM;
    for (const auto& r : reads) {
      const Buf& b = buf(r.first);
      if (b.writer >= 0) want(b.writer, r.second);
    }
    if (c_buf != nullptr && buf(c_buf).writer >= 0) want(buf(c_buf).writer, DEP_TM);  // C tile (tm, tn)
    for (const void* w : writes) {
      const Buf& b = buf(w);
      for (const Use& u : b.readers) want(u.cls, DEP_EPI | ((u.mode & DEP_ALL) ? DEP_ALL : out_rows));
      if (b.writer >= 0) want(b.writer, DEP_EPI | out_rows);
    }
    s.deps.clear();
    s.c_dep = -1;
    for (const auto& n : need) {
      int mode = (n.second & DEP_ALL) ? (DEP_ALL | (n.second & DEP_EPI)) : n.second;
      if (mode & DEP_EPI) {
        // already covered by a wait on the same class before the mainloop?
        bool covered = false;
        for (const auto& o : need)
          if (o.first == n.first && !(o.second & DEP_EPI) &&
              ((o.second & DEP_ALL) || ((mode & ~o.second & (DEP_TM | DEP_TN | DEP_ALL)) == 0)))
            covered = true;
        if (covered) continue;
      }
      s.deps.push_back(RowDep{counters(n.first), static_cast<int>(rows), target[n.first], mode});
      if (c_buf != nullptr && buf(c_buf).writer == n.first && !(mode & DEP_EPI))
        s.c_dep = static_cast<int>(s.deps.size()) - 1;
    }
    if (s.deps.size() > static_cast<size_t>(kMaxDeps)) return MSIGN_ERR_UNSUPPORTED;
    s.sig = counters(me);
    const int64_t tiles_n = ceil_div(s.N, s.bn);
    // tiles touching a row block: a row of tiles, or for a symmetric output
    // (tiles of both 256-wide halves of a row block count) the same number
    target.push_back(static_cast<int>(kTileSignals * tiles_n));
    cls.push_back(s);
    for (const void* w : writes) {
      Buf& b = buf(w);
      b.writer = me;
      b.readers.clear();
    }
    for (const auto& r : reads) buf(r.first).readers.push_back({me, r.second});
    if (c_buf != nullptr) buf(c_buf).readers.push_back({me, DEP_TM});
    return MSIGN_OK;
  }

  // The same product with its inner dimension split into `parts` ranges of
  // whole 256-blocks: every part but the last stores its fp32 partial tiles
  // into part_buf[p] (blocked layout, part_ld wide, part_bs per matrix);
  // the last part adds them, in order, to its own accumulator before the
  // product's real epilogue, waiting for them in its epilogue only.  All
  // parts run their mainloops side by side: a product of few tiles and a
  // long K fills more of the GPU.  The sum is taken in a fixed order.
  msign_status add_split(const ClassSpec& s, int parts, const std::vector<std::pair<const void*, int>>& reads,
                         const void* c_buf, const std::vector<const void*>& writes, float* const* part_buf,
                         int64_t part_ld, int64_t part_bs) {
    const int64_t K = s.K, len = round_up(ceil_div(K, std::max(parts, 1)), kBM);
    parts = static_cast<int>(std::min<int64_t>(ceil_div(K, len), kMaxAddends + 1));
    if (parts <= 1) return add(s, reads, c_buf, writes);
    const int out_rows = s.symmetric ? (DEP_TM | DEP_TN) : DEP_TM;
    std::vector<std::pair<const void*, int>> last_reads = reads;
    for (int q = 0; q + 1 < parts; ++q) {
      ClassSpec c;
      c.A = s.A, c.B = s.B, c.b_mn = s.b_mn, c.symmetric = s.symmetric, c.mirror = s.mirror, c.bn = s.bn;
      c.a_sym = s.a_sym, c.b_sym = s.b_sym, c.split = s.split;
      c.M = s.M, c.N = s.N, c.batch = s.batch;
      c.K = len, c.k_begin = q * len, c.k_total = K;
      c.outs = {out_blocked(part_buf[q], part_ld, part_bs)};
      msign_status st = add(c, reads, nullptr, {part_buf[q]});
      if (st != MSIGN_OK) return st;
      last_reads.push_back({part_buf[q], DEP_EPI | out_rows});
    }
    ClassSpec c = s;
    c.k_begin = (parts - 1) * len, c.K = K - c.k_begin, c.k_total = K;
    for (int q = 0; q + 1 < parts; ++q) c.addends.push_back(part_buf[q]);
    c.add_ld = part_ld, c.add_bs = part_bs;
    return add(c, last_reads, c_buf, writes);
  }
};

// Restart schedule -> segment bounds [0, r1, r2, ..., T].
msign_status gram_segments(int T, const int* restart_after, int n_restart, std::vector<int>* bounds) {
  std::vector<int> cuts;
  if (restart_after == nullptr && n_restart < 0) {
    if (T > 2) cuts.push_back(2);  // [P3] section 3.2: restart after the second step
  } else {
    if (n_restart < 0 || (n_restart > 0 && restart_after == nullptr)) return MSIGN_ERR_INVALID_ARG;
    for (int i = 0; i < n_restart; ++i) {
      if (restart_after[i] < 1 || restart_after[i] > T - 1) return MSIGN_ERR_INVALID_ARG;
      cuts.push_back(restart_after[i]);
    }
    std::sort(cuts.begin(), cuts.end());
    cuts.erase(std::unique(cuts.begin(), cuts.end()), cuts.end());
  }
  bounds->clear();
  bounds->push_back(0);
  for (int c : cuts) bounds->push_back(c);
  bounds->push_back(T);
  return MSIGN_OK;
}

}  // namespace msb

using namespace msb;


// ================================================================ C ABI

// Standard NS on validated arguments: batch matrices of rows x cols, input
// `in` (in_dt; rows in_ld apart, matrices in_bs apart) -> output `out`
// (out_dt; out_ld, out_bs), compute dtype `compute`, the schedule `sch`, a
// workspace of at least msign_ns_workspace_size() bytes.  [P2] eq. 4-7.
msign_status ns_run(const void* in, int in_dt, int64_t in_ld, int64_t in_bs, void* out, int out_dt, int64_t out_ld,
                    int64_t out_bs, msign_dtype compute_dtype, int64_t batch, int64_t rows, int64_t cols,
                    const Schedule& sch, void* workspace, cudaStream_t stream) {
  msign_status st = MSIGN_OK;
  const bool tr = rows > cols;  // iterate on the side with the smaller Gram matrix
  const int64_t n = tr ? cols : rows, m = tr ? rows : cols;
  const int64_t ldm = round_up(m, 8);
  const bool fp32 = compute_dtype == MSIGN_FP32;
  const int cd = to_dt(compute_dtype);  // the input is cast to the compute dtype first
  Carver cv(workspace);
  NsBuffers w;
  carve_ns(cv, batch, n, m, &w, fp32);

  // bf16 and fp32-accurate operands: one fused pass writes the unscaled x and
  // the factor s, applied by the first step.  fp16 operands must be scaled
  // before the cast (fp16 range), so that path normalises first.
  const bool fused = cd != DT_FP16;
  if (fused) {
    if (cudaMemsetAsync(w.cnt, 0, state_bytes(batch, n, kMaxClasses), stream) != cudaSuccess) return MSIGN_ERR_CUDA;
    IngestArgs a = ingest_args(in, in_dt, rows, cols, tr, cd, w.P[0], fp32 ? DT_TF32_HI : DT_BF16, ldm,
                               fp32 ? 2 * n * ldm : n * ldm);
    a.op_plane = n * ldm;
    a.in_bs = in_bs, a.ld_in = in_ld;
    if (fp32) a.master = w.master, a.ld_m = blk_ld(m), a.m_bs = blk_size(n, m);  // else see NsClass::c0_op
    a.partials = w.partials, a.ticket = ns_ticket_ptr(w), a.s_out = w.scale, a.s2_out = w.scale + batch;
    a.eps = sch.eps;
    st = launch_ingest(a, batch, stream);
  } else {
    if (in_ld != cols) return MSIGN_ERR_INVALID_ARG;  // the norm pass reads whole matrices
    st = launch_norm(in, in_dt, rows * cols, in_bs, batch, cd, sch.eps, 0, w.partials, w.scale, stream);
    if (st != MSIGN_OK) return st;
    IngestArgs a = ingest_args(in, in_dt, rows, cols, tr, cd, w.P[0], cd, ldm, n * ldm);
    a.pre_scale = w.scale;
    a.in_bs = in_bs, a.ld_in = in_ld;
    a.master = w.master, a.ld_m = blk_ld(m), a.m_bs = blk_size(n, m);
    st = launch_ingest(a, batch, stream);
  }
  if (st != MSIGN_OK) return st;
  std::vector<NsClass> cls(1);
  cls[0].w = w;
  cls[0].batch = batch, cls[0].n = n, cls[0].m = m;
  cls[0].fp32 = fp32;
  cls[0].op_dt = fp32 ? DT_BF16 : cd;
  cls[0].final_outs = {out_to(out, out_dt, out_ld, out_bs, tr)};
  if (fused) cls[0].s = w.scale, cls[0].s2 = w.scale + batch;
  cls[0].c0_op = fused && !fp32;
  cls[0].improved = sch.init == 1;
  return ns_iterate(cls, sch, stream, fused);
}

// msign_ns's automatic route (msign_coeffs.method = 1): Gram NS where it is
// expected to beat standard NS.  Gram NS saves FLOPs in proportion to m - n
// (it touches the n x m operand only in its first and last products), while
// its chain of n x n products costs latency that only larger problems hide;
// at n = 4096 the n x n products fill under two waves of CTA pairs, so the
// saving must be larger there.  Measured on a B200 (default schedules, L2
// flushed, median of 20; time of Gram NS over standard NS):
//   m - n >= 3072:        0.93 at 512 x 3584, 0.91 at 1024 x 4096, 0.87 at
//                         2048 x 5120, 0.96 at 3072 x 6144, 0.98 at
//                         4096 x 7168, 0.87 at 6144 x 9216, 0.86 at
//                         4096 x 8192, 0.71 at 4096 x 14336;
//   m - n = 2048, n <= 2048: 0.98 at 512 x 2560, 0.94 at 1024 x 3072, 0.95 at
//                         2048 x 4096 (0.94 for a batch of 4);
//   below the rule:       1.04 at 4096 x 6144, 1.13 at 4096 x 5120, 0.99 at
//                         2048 x 3072, 1.09 at 1024 x 2048, 1.08 at
//                         512 x 1536, 0.99 at 256 x 4096, 1.13 at 256 x 2048.
// Only shapes whose Gram-NS workspace fits in msign_ns's qualify, so the
// workspace query stays the same for both routes (2048 x 4096 alone does
// not fit).
constexpr int64_t kGramMinRows = 512;          // n
constexpr int64_t kGramMinExcess = 3072;       // m - n, any n
constexpr int64_t kGramMinExcessSmall = 2048;  // m - n, n <= kGramSmallRows
constexpr int64_t kGramSmallRows = 2048;
// muon_step runs its Gram-NS matrices after the grouped standard-route launch
// instead of inside it, where a small matrix shares the launch with the large
// ones: there a matrix takes Gram NS only from m - n >= 4096 (a Llama layer's
// 1024 x 4096 k and v stay in the group).
constexpr int64_t kGramMuonMinExcess = 4096;

bool gram_route(int64_t batch, int64_t rows, int64_t cols, msign_dtype compute, const Schedule& sch,
                int64_t min_excess = 0) {
  if (sch.method != 1 || compute == MSIGN_FP32 || sch.init != 0) return false;
  if (batch <= 0 || rows <= 0 || cols <= 0) return false;
  const int64_t n = std::min(rows, cols), m = std::max(rows, cols);
  const int64_t need = std::max(n <= kGramSmallRows ? kGramMinExcessSmall : kGramMinExcess, min_excess);
  if (n < kGramMinRows || m - n < need) return false;
  return gram_ns_workspace_size(batch, rows, cols) <= msign_ns_workspace_size(batch, rows, cols, compute);
}

extern "C" {

int msign_abi_version(void) { return 106; }

int msign_set_chaining(int enable) { return msb::g_chaining.exchange(enable != 0 ? 1 : 0); }

const char* msign_status_string(msign_status s) {
  switch (s) {
    case MSIGN_OK: return "ok";
    case MSIGN_ERR_INVALID_ARG: return "invalid argument";
    case MSIGN_ERR_UNSUPPORTED: return "unsupported configuration";
    case MSIGN_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MSIGN_ERR_CUDA: return "CUDA error";
    case MSIGN_ERR_TIMEOUT: return "a bounded device wait timed out";
  }
  return "unknown status";
}

msign_status msign_selftest_timeout(uint64_t limit_ns, msign_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return MSIGN_ERR_INVALID_ARG;
  DeviceState* dev = nullptr;
  msign_status st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  selftest_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(dev->err, limit_ns);
  return launch_ok();
}

msign_status msign_sync_status(msign_stream_t stream) {
  DeviceState* dev = nullptr;
  msign_status st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return MSIGN_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, dev->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MSIGN_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpy(dev->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return MSIGN_ERR_CUDA;
    return MSIGN_ERR_TIMEOUT;
  }
  return MSIGN_OK;
}

msign_status msign_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof = enable != 0;
  return MSIGN_OK;
}

msign_status msign_profile_read(int kind, int* launches, double* total_ms, double* flops, double* bytes) {
  if (launches == nullptr || total_ms == nullptr || flops == nullptr || bytes == nullptr) return MSIGN_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  *launches = 0;
  *total_ms = 0.0;
  *flops = 0.0;
  *bytes = 0.0;
  for (const ProfRec& r : g_prof_recs) {
    if (r.kind != kind) continue;
    if (cudaEventSynchronize(r.e1) != cudaSuccess) return MSIGN_ERR_CUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, r.e0, r.e1) != cudaSuccess) return MSIGN_ERR_CUDA;
    *launches += 1;
    *total_ms += ms;
    *flops += r.flops;
    *bytes += r.bytes;
  }
  return MSIGN_OK;
}

msign_status msign_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (const ProfRec& r : g_prof_recs) {
    cudaEventSynchronize(r.e1);
    g_event_pool.push_back(r.e0);
    g_event_pool.push_back(r.e1);
  }
  g_prof_recs.clear();
  return MSIGN_OK;
}

size_t msign_ns_workspace_size(int64_t batch, int64_t rows, int64_t cols, msign_dtype compute_dtype) {
  if (batch <= 0 || rows <= 0 || cols <= 0) return 0;
  const int64_t n = std::min(rows, cols), m = std::max(rows, cols);
  Carver cv(nullptr);
  NsBuffers b;
  carve_ns(cv, batch, n, m, &b, compute_dtype == MSIGN_FP32);
  return cv.off + 1024;
}

int msign_ns_route(int64_t batch, int64_t rows, int64_t cols, msign_dtype compute_dtype, const msign_coeffs* coeffs) {
  if (!valid_dtype(compute_dtype) || batch < 0 || rows < 0 || cols < 0) return -MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  const msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return -static_cast<int>(st);
  if (sch.init != 0 && compute_dtype == MSIGN_FP32) return -MSIGN_ERR_UNSUPPORTED;
  return gram_route(batch, rows, cols, compute_dtype, sch) ? 1 : 0;
}

msign_status msign_ns(const void* in, void* out, msign_dtype io_dtype, msign_dtype compute_dtype, int64_t batch,
                      int64_t rows, int64_t cols, int64_t in_stride, int64_t out_stride, const msign_coeffs* coeffs,
                      void* workspace, size_t workspace_bytes, msign_stream_t stream_) {
  if (!valid_dtype(io_dtype) || !valid_dtype(compute_dtype)) return MSIGN_ERR_INVALID_ARG;
  if (batch < 0 || rows < 0 || cols < 0) return MSIGN_ERR_INVALID_ARG;
  if (!valid_strides(rows, cols, in_stride, out_stride)) return MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return st;
  if (sch.init != 0 && compute_dtype == MSIGN_FP32) return MSIGN_ERR_UNSUPPORTED;
  if (batch == 0 || rows == 0 || cols == 0) return MSIGN_OK;
  if (in == nullptr || out == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (batch > 65535 || rows > (1 << 30) || cols > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
  const size_t need = msign_ns_workspace_size(batch, rows, cols, compute_dtype);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  if (gram_route(batch, rows, cols, compute_dtype, sch)) {
    // Gram NS with the same schedule, Gram NS's eps unless one was given,
    // and the page's restart after step 2 where the schedule has one
    msign_coeffs g = {};
    g.steps = sch.steps();
    g.abc = sch.abc.data();
    g.eps = (coeffs != nullptr && coeffs->eps >= 0.0f) ? coeffs->eps : -1.0f;
    return gram_ns(in, out, io_dtype, batch, rows, cols, in_stride, out_stride, &g, nullptr, sch.steps() >= 3 ? -1 : 0,
                   workspace, workspace_bytes, stream_);
  }
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  const int io = to_dt(io_dtype);
  return ns_run(in, io, cols, in_stride > 0 ? in_stride : rows * cols, out, io, cols,
                out_stride > 0 ? out_stride : rows * cols, compute_dtype, batch, rows, cols, sch, workspace,
                reinterpret_cast<cudaStream_t>(stream_));
}

size_t gram_xxt_workspace_size(int64_t batch, int64_t n, int64_t m, msign_dtype x_dtype, const void* X) {
  if (batch <= 0 || n <= 0 || m <= 0) return 0;
  const int es = x_dtype == MSIGN_FP32 ? 4 : 2;
  if ((reinterpret_cast<uintptr_t>(X) % 16) == 0 && (m * es) % 16 == 0) return 0;
  return 2ull * batch * n * round_up(m, 8) + 2048;
}

msign_status gram_xxt(const void* X, msign_dtype x_dtype, void* A, msign_dtype a_dtype, int64_t batch, int64_t n,
                      int64_t m, void* workspace, size_t workspace_bytes, msign_stream_t stream_) {
  if (!valid_dtype(x_dtype) || !valid_dtype(a_dtype)) return MSIGN_ERR_INVALID_ARG;
  if (batch < 0 || n < 0 || m < 0) return MSIGN_ERR_INVALID_ARG;
  if (batch == 0 || n == 0) return MSIGN_OK;
  if (X == nullptr && m > 0) return MSIGN_ERR_INVALID_ARG;
  if (A == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (x_dtype == MSIGN_FP32) return MSIGN_ERR_UNSUPPORTED;
  if (batch > 65535 || n > (1 << 30) || m > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (m == 0) {  // empty inner dimension: A = 0
    const size_t bytes = static_cast<size_t>(batch) * n * n * (a_dtype == MSIGN_FP32 ? 4 : 2);
    return cudaMemsetAsync(A, 0, bytes, stream) == cudaSuccess ? MSIGN_OK : MSIGN_ERR_CUDA;
  }
  const int xd = to_dt(x_dtype);
  Mat Xm{X, xd, n, m, m, n * m};
  const size_t need = gram_xxt_workspace_size(batch, n, m, x_dtype, X);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
      return MSIGN_ERR_WORKSPACE;
    const int64_t ldm = round_up(m, 8);
    msign_status st = launch_ingest(ingest_args(X, xd, n, m, false, DT_FP32, workspace, xd, ldm, n * ldm), batch, stream);
    if (st != MSIGN_OK) return st;
    Xm = Mat{workspace, xd, n, m, ldm, n * ldm};
  }
  ClassSpec s;
  s.A = Xm;
  s.B = Xm;
  s.symmetric = true;
  s.mirror = true;  // the user gets the full, exactly symmetric matrix
  s.M = n, s.N = n, s.K = m, s.batch = batch;
  s.bn = pick_bn(n, n, batch, true);
  const int ad = to_dt(a_dtype);
  s.outs = {out_to(A, ad, n, n * n, false)};
  return launch_grouped({s}, xd, stream);
}


size_t gram_ns_workspace_size(int64_t batch, int64_t rows, int64_t cols) {
  if (batch <= 0 || rows <= 0 || cols <= 0) return 0;
  const int64_t n = std::min(rows, cols), m = std::max(rows, cols);
  Carver cv(nullptr);
  GramBuffers b;
  carve_gram(cv, batch, n, m, &b);
  return cv.off + 1024;
}

}  // extern "C"

// Gram NS on validated arguments: `in` (in_dt) -> `out` (out_dt), the
// segment bounds of the restart schedule, a workspace of at least
// gram_ns_workspace_size() bytes.  [P3] Algorithm 2.
//   in_list: optional HOST array of `batch` device pointers, one input matrix
//            each (then `in` and in_bs are unused);
//   out == nullptr: the result goes into a dead X buffer of the workspace
//            (rows x cols with leading dimension cols, matrix b at
//            b * n * round_up(m, 8) elements, out_dt), returned in *o_ws.
msign_status gram_run(const void* in, int in_dt, void* out, int out_dt, int64_t batch, int64_t rows, int64_t cols,
                      int64_t in_bs, int64_t out_bs, const Schedule& sch, const std::vector<int>& bounds,
                      void* workspace, cudaStream_t stream, const void* const* in_list = nullptr,
                      void** o_ws = nullptr) {
  msign_status st = MSIGN_OK;
  const bool tr = rows > cols;
  const int64_t n = tr ? cols : rows, m = tr ? rows : cols;
  const int64_t ldm = round_up(m, 8), ldn = round_up(n, 8);
  Carver cv(workspace);
  GramBuffers w;
  carve_gram(cv, batch, n, m, &w);
  const int64_t sq = n * ldn, rect = n * ldm;
  // every n x n intermediate is symmetric and kept as its upper 256-blocks
  auto sym_out = [&](void* p, float gamma) { return std::vector<EpiOut>{out_to(p, DT_FP16, ldn, sq, false, gamma)}; };
  auto sqm = [&](void* p) { return Mat{p, DT_FP16, n, n, ldn, sq}; };

  // [P3] Algorithm 2 steps 1-2: X <- X / (||X||_F + eps); X <- float16(X)
  if (in_list == nullptr) {
    st = launch_norm(in, in_dt, rows * cols, in_bs, batch, DT_FP32, sch.eps, 1, w.partials, w.scale, stream);
    if (st != MSIGN_OK) return st;
    IngestArgs a = ingest_args(in, in_dt, rows, cols, tr, DT_FP32, w.P[0], DT_FP16, ldm, rect);
    a.pre_scale = w.scale;
    a.in_bs = in_bs;
    st = launch_ingest(a, batch, stream);
    if (st != MSIGN_OK) return st;
  } else {
    for (int64_t b = 0; b < batch; ++b) {
      st = launch_norm(in_list[b], in_dt, rows * cols, rows * cols, 1, DT_FP32, sch.eps, 1, w.partials + b * kNormParts,
                       w.scale + b, stream);
      if (st != MSIGN_OK) return st;
      IngestArgs a = ingest_args(in_list[b], in_dt, rows, cols, tr, DT_FP32, static_cast<char*>(w.P[0]) + 2 * b * rect,
                                 DT_FP16, ldm, rect);
      a.pre_scale = w.scale + b;
      st = launch_ingest(a, 1, stream);
      if (st != MSIGN_OK) return st;
    }
  }

  // every product of the iteration, chained (see Chain); a tile of a later
  // product starts as soon as the row blocks it touches are final
  Chain ch;
  ch.state = w.cnt, ch.batch = batch, ch.rows = ceil_div(n, kBM), ch.ab_dt = DT_FP16, ch.stream = stream;
  const int DEP_TMN = DEP_TM | DEP_TN;
  // split K for the symmetric products with few tiles and a long K
  auto parts_for = [&](int64_t K) { return gram_parts(batch, n, K); };
  // (products split in K keep 256-wide tiles; the others take pick_bn's width)
  auto add_sym = [&](ClassSpec s, const std::vector<std::pair<const void*, int>>& reads, const void* c_buf,
                     const std::vector<const void*>& writes) {
    const int parts = parts_for(s.K);
    s.bn = parts > 1 ? kBN : pick_bn(n, n, batch, true);
    return ch.add_split(s, parts, reads, c_buf, writes, w.part, blk_ld(n), blk_size(n, n));
  };
  int cur = 0;
  for (size_t seg = 0; seg + 1 < bounds.size(); ++seg) {
    const int s0 = bounds[seg], s1 = bounds[seg + 1];
    const Mat X{w.P[cur], DT_FP16, n, m, ldm, rect};
    {  // R = X X^T
      ClassSpec s;
      s.A = X, s.B = X, s.symmetric = true;
      s.M = n, s.N = n, s.K = m, s.batch = batch;
      s.outs = sym_out(w.R, 0.0f);
      st = add_sym(s, {{w.P[cur], DEP_TMN}}, nullptr, {w.R});
      if (st != MSIGN_OK) return st;
    }
    int q = -1;  // Q = I until the first step of the segment sets it
    for (int t = s0; t < s1; ++t) {
      const float a = sch.abc[3 * t], b = sch.abc[3 * t + 1], c = sch.abc[3 * t + 2];
      const bool first = (t == s0), last = (t == s1 - 1);
      {  // Z = b R + c R^2; on the first step also Q = Z + a I (Q Z with Q = I)
        ClassSpec s;
        s.A = sqm(w.R), s.B = sqm(w.R), s.symmetric = true, s.a_sym = true, s.b_sym = true;
        s.M = n, s.N = n, s.K = n, s.batch = batch;
        s.alpha = c, s.beta = b;
        s.C = w.R, s.c_dt = DT_FP16, s.ldc = ldn, s.c_bs = sq;
        s.outs = sym_out(w.Z, 0.0f);
        std::vector<const void*> writes{w.Z};
        if (first) {
          std::vector<EpiOut> qo = sym_out(w.Q[0], a);
          s.outs.insert(s.outs.end(), qo.begin(), qo.end());
          writes.push_back(w.Q[0]);
        }
        st = add_sym(s, {{w.R, DEP_TMN}}, w.R, writes);
        if (st != MSIGN_OK) return st;
        if (first) q = 0;
      }
      if (!first) {  // Q <- Q Z + a Q
        ClassSpec s;
        s.A = sqm(w.Q[q]), s.B = sqm(w.Z), s.symmetric = true, s.a_sym = true, s.b_sym = true;
        s.M = n, s.N = n, s.K = n, s.batch = batch;
        s.alpha = 1.0f, s.beta = a;
        s.C = w.Q[q], s.c_dt = DT_FP16, s.ldc = ldn, s.c_bs = sq;
        s.outs = sym_out(w.Q[q ^ 1], 0.0f);
        st = add_sym(s, {{w.Q[q], DEP_TM}, {w.Z, DEP_TN}}, w.Q[q], {w.Q[q ^ 1]});
        if (st != MSIGN_OK) return st;
      }
      if (!last) {  // RZ <- R Z + a R
        ClassSpec s;
        s.A = sqm(w.R), s.B = sqm(w.Z), s.symmetric = true, s.a_sym = true, s.b_sym = true;
        s.M = n, s.N = n, s.K = n, s.batch = batch;
        s.alpha = 1.0f, s.beta = a;
        s.C = w.R, s.c_dt = DT_FP16, s.ldc = ldn, s.c_bs = sq;
        s.outs = sym_out(w.RZ, 0.0f);
        st = add_sym(s, {{w.R, DEP_TM}, {w.Z, DEP_TN}}, w.R, {w.RZ});
        if (st != MSIGN_OK) return st;
      }
      if (!first) q ^= 1;
      if (!last) {  // R <- Z RZ + a RZ
        ClassSpec s;
        s.A = sqm(w.Z), s.B = sqm(w.RZ), s.symmetric = true, s.a_sym = true, s.b_sym = true;
        s.M = n, s.N = n, s.K = n, s.batch = batch;
        s.alpha = 1.0f, s.beta = a;
        s.C = w.RZ, s.c_dt = DT_FP16, s.ldc = ldn, s.c_bs = sq;
        s.outs = sym_out(w.R, 0.0f);
        st = add_sym(s, {{w.Z, DEP_TM}, {w.RZ, DEP_TN}}, w.RZ, {w.R});
        if (st != MSIGN_OK) return st;
      }
    }
    {  // X <- Q X (the restart), or the output after the last segment
      ClassSpec s;
      s.A = sqm(w.Q[q]), s.a_sym = true, s.B = X, s.b_mn = true;
      s.M = n, s.N = m, s.K = n, s.batch = batch;
      s.bn = pick_bn(n, m, batch, false);
      const bool final = seg + 2 == bounds.size();
      if (final && out == nullptr) {
        // the previous X copy is dead: the result takes its place
        out = w.P[cur ^ 1], out_bs = rect;
        if (o_ws != nullptr) *o_ws = out;
      }
      void* dst = final ? out : w.P[cur ^ 1];
      if (final)
        s.outs = {out_to(out, out_dt, cols, out_bs, tr)};
      else
        s.outs = {out_to(w.P[cur ^ 1], DT_FP16, ldm, rect, false)};
      st = ch.add(s, {{w.Q[q], DEP_TM}, {w.P[cur], DEP_ALL}}, nullptr, {dst});
      if (st != MSIGN_OK) return st;
    }
    cur ^= 1;
  }
  return ch.flush();
}

extern "C" {

msign_status gram_ns(const void* in, void* out, msign_dtype io_dtype, int64_t batch, int64_t rows, int64_t cols,
                     int64_t in_stride, int64_t out_stride, const msign_coeffs* coeffs, const int* restart_after,
                     int n_restart, void* workspace, size_t workspace_bytes, msign_stream_t stream_) {
  if (!valid_dtype(io_dtype)) return MSIGN_ERR_INVALID_ARG;
  if (batch < 0 || rows < 0 || cols < 0) return MSIGN_ERR_INVALID_ARG;
  if (!valid_strides(rows, cols, in_stride, out_stride)) return MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  msign_status st = read_schedule(coeffs, kGramEps, &sch);
  if (st != MSIGN_OK) return st;
  if (sch.init != 0) return MSIGN_ERR_UNSUPPORTED;  // the sharper normalisation is a standard-NS option
  if (sch.method != 0) return MSIGN_ERR_INVALID_ARG;  // a route choice is msign_ns's
  const int T = sch.steps();
  std::vector<int> bounds;
  st = gram_segments(T, restart_after, n_restart, &bounds);
  if (st != MSIGN_OK) return st;
  if (batch == 0 || rows == 0 || cols == 0) return MSIGN_OK;
  if (in == nullptr || out == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (batch > 65535 || rows > (1 << 30) || cols > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
  const size_t need = gram_ns_workspace_size(batch, rows, cols);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != MSIGN_OK) return st;

  const int io = to_dt(io_dtype);
  return gram_run(in, io, out, io, batch, rows, cols, in_stride > 0 ? in_stride : rows * cols,
                  out_stride > 0 ? out_stride : rows * cols, sch, bounds, workspace,
                  reinterpret_cast<cudaStream_t>(stream_));
}

// Workspace of one group of Muon matrices: one NsBuffers set per distinct
// oriented shape, in first-seen order.
static size_t muon_group_bytes(const std::vector<std::pair<int64_t, int64_t>>& shapes,
                               const std::vector<int64_t>& counts) {
  Carver cv(nullptr);
  for (size_t i = 0; i < shapes.size(); ++i) {
    NsBuffers b;
    carve_ns(cv, counts[i], shapes[i].first, shapes[i].second, &b);
  }
  return cv.off + 1024;
}

// The standard-NS classes of matrices begin .. end - 1: one per distinct
// oriented shape; empty matrices and those marked in `gram` (the Gram-NS
// route) belong to none.
static void muon_group_shapes(const int64_t* rows, const int64_t* cols, int begin, int end,
                              std::vector<std::pair<int64_t, int64_t>>* shapes, std::vector<int64_t>* counts,
                              std::vector<int>* cls_of, std::vector<int64_t>* slot_of,
                              const std::vector<char>* gram = nullptr) {
  shapes->clear();
  counts->clear();
  cls_of->assign(end - begin, -1);
  slot_of->assign(end - begin, -1);
  for (int i = begin; i < end; ++i) {
    if (rows[i] == 0 || cols[i] == 0) continue;
    if (gram != nullptr && (*gram)[i]) continue;
    const std::pair<int64_t, int64_t> sh{std::min(rows[i], cols[i]), std::max(rows[i], cols[i])};
    size_t c = 0;
    while (c < shapes->size() && (*shapes)[c] != sh) ++c;
    if (c == shapes->size()) {
      shapes->push_back(sh);
      counts->push_back(0);
    }
    (*cls_of)[i - begin] = static_cast<int>(c);
    (*slot_of)[i - begin] = (*counts)[c]++;
  }
}

// Workspace of a batch of Muon matrices on the Gram-NS route: Gram NS's own
// (O, the bf16 result, takes the place of Gram NS's dead X copy).
static size_t muon_gram_bytes(int64_t batch, int64_t rows, int64_t cols) {
  return gram_ns_workspace_size(batch, rows, cols);
}

// muon_step's per-matrix route (msign_coeffs.method = 1): Gram NS for a
// matrix that msign_ns's route gives to it and whose m - n is at least
// kGramMuonMinExcess, when Gram NS's workspace (O in bf16 over its dead copy
// of X) fits in the matrix's standard-route workspace.
static bool muon_gram_route(int64_t rows, int64_t cols, const Schedule& sch) {
  if (rows <= 0 || cols <= 0 || !gram_route(1, rows, cols, MSIGN_BF16, sch, kGramMuonMinExcess)) return false;
  const std::pair<int64_t, int64_t> sh{std::min(rows, cols), std::max(rows, cols)};
  return muon_gram_bytes(1, rows, cols) <= muon_group_bytes({sh}, {1});
}

int muon_step_route(int64_t rows, int64_t cols, const msign_coeffs* coeffs) {
  if (rows < 0 || cols < 0) return -MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  const msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return -static_cast<int>(st);
  return muon_gram_route(rows, cols, sch) ? 1 : 0;
}

size_t muon_step_workspace_size(int num, const int64_t* rows, const int64_t* cols) {
  if (num <= 0 || rows == nullptr || cols == nullptr) return 0;
  std::vector<std::pair<int64_t, int64_t>> shapes;
  std::vector<int64_t> counts, slots;
  std::vector<int> cls;
  muon_group_shapes(rows, cols, 0, num, &shapes, &counts, &cls, &slots);
  if (shapes.empty()) return 0;
  return muon_group_bytes(shapes, counts);
}

msign_status muon_step(int num, void* const* W, float* const* M, const void* const* G, const int64_t* rows,
                       const int64_t* cols, msign_dtype w_dtype, msign_dtype g_dtype, float momentum, float lr,
                       const msign_coeffs* coeffs, void* workspace, size_t workspace_bytes,
                       msign_stream_t stream_) {
  if (num < 0) return MSIGN_ERR_INVALID_ARG;
  if (num == 0) return MSIGN_OK;
  if (W == nullptr || M == nullptr || G == nullptr || rows == nullptr || cols == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (!valid_dtype(w_dtype) || !valid_dtype(g_dtype)) return MSIGN_ERR_INVALID_ARG;
  if (w_dtype == MSIGN_FP16 || g_dtype == MSIGN_FP16) return MSIGN_ERR_UNSUPPORTED;
  if (!std::isfinite(momentum) || !std::isfinite(lr)) return MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return st;
  size_t largest = 0;
  for (int i = 0; i < num; ++i) {
    if (rows[i] < 0 || cols[i] < 0) return MSIGN_ERR_INVALID_ARG;
    if (rows[i] == 0 || cols[i] == 0) continue;
    if (W[i] == nullptr || M[i] == nullptr || G[i] == nullptr) return MSIGN_ERR_INVALID_ARG;
    if (rows[i] > (1 << 30) || cols[i] > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
    largest = std::max(largest, muon_step_workspace_size(1, rows + i, cols + i));
  }
  if (largest == 0) return MSIGN_OK;
  if (workspace == nullptr || workspace_bytes < largest || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int wd = to_dt(w_dtype), gd = to_dt(g_dtype);

  // msign_coeffs.method = 1: the matrices muon_step_route gives to Gram NS
  // (the workspace query stays the same for both routes)
  std::vector<char> gram(num, 0);
  Schedule gsch;
  std::vector<int> gbounds;
  if (sch.method == 1) {
    for (int i = 0; i < num; ++i) {
      gram[i] = muon_gram_route(rows[i], cols[i], sch) ? 1 : 0;
    }
    gsch.abc = sch.abc;
    gsch.eps = (coeffs != nullptr && coeffs->eps >= 0.0f) ? coeffs->eps : kGramEps;
    st = gram_segments(gsch.steps(), nullptr, gsch.steps() >= 3 ? -1 : 0, &gbounds);
    if (st != MSIGN_OK) return st;
  }
  const unsigned ew_grid = static_cast<unsigned>(std::max(1, dev->sms) * 8);

  int begin = 0;
  while (begin < num) {
    // the longest prefix of the remaining list whose workspace fits
    int end = begin + 1;
    std::vector<std::pair<int64_t, int64_t>> shapes;
    std::vector<int64_t> counts, slots;
    std::vector<int> cls;
    while (end < num) {
      muon_group_shapes(rows, cols, begin, end + 1, &shapes, &counts, &cls, &slots, &gram);
      if (muon_group_bytes(shapes, counts) > workspace_bytes) break;
      ++end;
    }
    muon_group_shapes(rows, cols, begin, end, &shapes, &counts, &cls, &slots, &gram);
    // the Gram-NS matrices of this range, after the group: those of equal
    // shape (rows, cols) share one batched Gram-NS chain, as many at a time
    // as the workspace holds
    auto run_gram = [&]() -> msign_status {
      std::vector<char> done(end - begin, 0);
      for (int i = begin; i < end; ++i) {
        if (!gram[i] || done[i - begin]) continue;
        std::vector<int> same;
        for (int j = i; j < end; ++j)
          if (gram[j] && !done[j - begin] && rows[j] == rows[i] && cols[j] == cols[i]) same.push_back(j);
        const int64_t r = rows[i], c = cols[i], ne = r * c;
        const unsigned g = static_cast<unsigned>(std::min<int64_t>(ceil_div(ne, 8 * 256), ew_grid));
        size_t at = 0;
        while (at < same.size()) {
          int64_t nb = static_cast<int64_t>(same.size() - at);
          while (nb > 1 && muon_gram_bytes(nb, r, c) > workspace_bytes) --nb;
          std::vector<const void*> ins;
          for (int64_t b = 0; b < nb; ++b) {
            const int k = same[at + b];
            done[k - begin] = 1;
            prof_begin(stream);
            momentum_kernel<<<g, 256, 0, stream>>>(M[k], G[k], gd, momentum, ne);
            prof_end(3, stream, 0.0, static_cast<double>(ne) * (8 + dtype_size(gd)));
            msign_status e = launch_ok();
            if (e != MSIGN_OK) return e;
            ins.push_back(M[k]);
          }
          void* o = nullptr;
          msign_status e = gram_run(nullptr, DT_FP32, nullptr, DT_BF16, nb, r, c, 0, 0, gsch, gbounds, workspace, stream,
                                    ins.data(), &o);
          if (e != MSIGN_OK) return e;
          const int64_t ostride = std::min(r, c) * round_up(std::max(r, c), 8);  // Gram NS's X copy per matrix
          const float coef = lr * std::sqrt(std::max(1.0f, static_cast<float>(r) / static_cast<float>(c)));
          for (int64_t b = 0; b < nb; ++b) {
            const int k = same[at + b];
            prof_begin(stream);
            update_rows_kernel<<<g, 256, 0, stream>>>(W[k], wd, static_cast<char*>(o) + 2 * b * ostride, DT_BF16, coef,
                                                      ne);
            prof_end(3, stream, 0.0, static_cast<double>(ne) * (2 + 2 * dtype_size(wd)));
            e = launch_ok();
            if (e != MSIGN_OK) return e;
          }
          at += static_cast<size_t>(nb);
        }
      }
      return MSIGN_OK;
    };
    if (shapes.empty()) {
      st = run_gram();
      if (st != MSIGN_OK) return st;
      begin = end;
      continue;
    }
    Carver cv(workspace);
    std::vector<NsClass> ns(shapes.size());
    for (size_t c = 0; c < shapes.size(); ++c) {
      carve_ns(cv, counts[c], shapes[c].first, shapes[c].second, &ns[c].w);
      ns[c].batch = counts[c];
      ns[c].n = shapes[c].first;
      ns[c].m = shapes[c].second;
      ns[c].final_outs = {out_blocked(ns[c].w.master, blk_ld(ns[c].m), blk_size(ns[c].n, ns[c].m))};
      ns[c].s = ns[c].w.scale;
      ns[c].s2 = ns[c].w.scale + counts[c];
      ns[c].improved = sch.init == 1;
      ns[c].c0_op = true;  // the ingest below writes no master
      if (cudaMemsetAsync(ns[c].w.cnt, 0, state_bytes(counts[c], ns[c].n, kMaxClasses), stream) != cudaSuccess)
        return MSIGN_ERR_CUDA;
    }
    // one fused pass per matrix: M <- mu M + G in place, x = bf16(M) (unscaled)
    // into the class slot, s = 1/||x||_F for the first step
    for (int i = begin; i < end; ++i) {
      const int c = cls[i - begin];
      if (c < 0) continue;
      const int64_t slot = slots[i - begin];
      const NsClass& k = ns[c];
      const bool tr = rows[i] > cols[i];
      const int64_t ldm = round_up(k.m, 8), per = k.n * ldm;
      IngestArgs a = ingest_args(M[i], DT_FP32, rows[i], cols[i], tr, DT_BF16,
                                 static_cast<char*>(k.w.P[0]) + 2 * slot * per, DT_BF16, ldm, per);
      a.partials = k.w.partials + slot * kNormParts, a.ticket = ns_ticket_ptr(k.w) + slot;
      a.s_out = k.w.scale + slot, a.s2_out = k.w.scale + k.batch + slot, a.eps = sch.eps;
      a.G = G[i], a.g_dt = gd, a.mu = momentum;
      st = launch_ingest(a, 1, stream);
      if (st != MSIGN_OK) return st;
    }
    st = ns_iterate(ns, sch, stream, /*zeroed=*/true);
    if (st != MSIGN_OK) return st;
    // W <- W - lr * sqrt(max(1, rows/cols)) * O
    for (int i = begin; i < end; ++i) {
      const int c = cls[i - begin];
      if (c < 0) continue;
      const NsClass& k = ns[c];
      const int64_t mb = blk_size(k.n, k.m);
      const float coef = lr * std::sqrt(std::max(1.0f, static_cast<float>(rows[i]) / static_cast<float>(cols[i])));
      dim3 g(static_cast<unsigned>((cols[i] + 31) / 32), static_cast<unsigned>((rows[i] + 31) / 32));
      prof_begin(stream);
      apply_update_kernel<<<g, dim3(32, 8), 0, stream>>>(W[i], wd, static_cast<int>(rows[i]),
                                                         static_cast<int>(cols[i]), k.w.master + slots[i - begin] * mb,
                                                         blk_ld(k.m), rows[i] > cols[i] ? 1 : 0, coef);
      prof_end(3, stream, 0.0, static_cast<double>(rows[i]) * cols[i] * (4 + 2 * dtype_size(wd)));
      st = launch_ok();
      if (st != MSIGN_OK) return st;
    }
    st = run_gram();
    if (st != MSIGN_OK) return st;
    begin = end;
  }
  return MSIGN_OK;
}


}  // extern "C"

// ---------------------------------------------------------------- Mousse
//
// The Mousse post (anti-entrophic.github.io/posts/10054, section "Mousse")
// preconditions msign with Shampoo-style Kronecker factors L and R:
// Delta W = -L^(-1/4) msign(L^(-1/4) G R^(-1/4)) R^(-1/4).  Two entry points
// cover it: mousse_inv_root forms the inverse fourth roots of the damped
// factors, and mousse_direction applies the two-sided projection, msign and
// the back-projection.

namespace msb {

constexpr int kRootDefaultIters = 20;
constexpr int kRootMaxIters = 1000;

struct RootBuffers {
  float* partials;
  float* scale;  // s = 1 / (||A||_F + eps) per matrix
  float* X[2];   // iterates X_j, tf32 plane pairs (upper 256-blocks read)
  float* M[2];   // M_j = X_j^4 (A + eps I), plane pairs
  float* T2;     // ((5 I - M) / 4)^2
  float* T4;     // its square
  int* cnt;      // chained-launch state (see Chain)
};

void carve_root(Carver& cv, int64_t batch, int64_t n, RootBuffers* b) {
  const uint64_t mat = 8ull * batch * n * round_up(n, 8);  // two fp32 planes per matrix
  b->partials = static_cast<float*>(cv.take(sizeof(float) * kNormParts * batch));
  b->scale = static_cast<float*>(cv.take(sizeof(float) * batch));
  for (int i = 0; i < 2; ++i) b->X[i] = static_cast<float*>(cv.take(mat));
  for (int i = 0; i < 2; ++i) b->M[i] = static_cast<float*>(cv.take(mat));
  b->T2 = static_cast<float*>(cv.take(mat));
  b->T4 = static_cast<float*>(cv.take(mat));
  b->cnt = static_cast<int*>(cv.take(kSchedBytes + sizeof(int) * kMaxClasses * batch * ceil_div(n, kBM)));
}

// (A + eps I)^(-1/4) by the coupled Newton iteration for inverse p-th roots
// (p = 4): with T_j = (5 I - M_j) / 4,
//   X_{j+1} = X_j T_j,   M_{j+1} = T_j^4 M_j,
// from X_0 = s^(1/4) I and M_0 = s (A + eps I), which keeps M_j = X_j^4 (A + eps I)
// and drives M_j to I and X_j to (A + eps I)^(-1/4).  Every matrix is a
// polynomial in A, so every product is symmetric and runs on the triangle
// schedule, in fp32-accurate arithmetic (3xTF32 on hi/lo planes).  Per step
// four products: M M (T^2 in the epilogue: (25 I - 10 M + M M) / 16), T^2 T^2,
// T^4 M, and X M (X T in the epilogue: 5/4 X - 1/4 X M); X_1 comes from the
// start kernel, and the last X M writes the user's output with exact mirrors.
msign_status root_run(const float* A, float* out, int64_t batch, int64_t n, float eps, int iters, void* workspace,
                      cudaStream_t stream) {
  const int64_t ldn = round_up(n, 8), pl = n * ldn;
  Carver cv(workspace);
  RootBuffers w;
  carve_root(cv, batch, n, &w);
  msign_status st = launch_norm(A, DT_FP32, n * n, n * n, batch, DT_FP32, eps, 1, w.partials, w.scale, stream);
  if (st != MSIGN_OK) return st;
  {
    const int64_t blocks = std::min<int64_t>(ceil_div(n * n, 256), 1024);
    dim3 g(static_cast<unsigned>(blocks), static_cast<unsigned>(batch));
    prof_begin(stream);
    inv_root_start_kernel<<<g, 256, 0, stream>>>(A, static_cast<int>(n), n * n, w.scale, eps, w.M[0], w.X[0], ldn,
                                                 pl);
    prof_end(3, stream, 0.0, static_cast<double>(batch) * n * n * 20.0);
    st = launch_ok();
    if (st != MSIGN_OK) return st;
  }
  Chain ch;
  ch.state = w.cnt, ch.batch = batch, ch.rows = ceil_div(n, kBM), ch.ab_dt = DT_FP32, ch.stream = stream;
  const int DEP_TMN = DEP_TM | DEP_TN;
  auto planes = [&](float* p, float gamma) {
    std::vector<EpiOut> v = split_out(p, ldn, pl);
    for (EpiOut& e : v) e.gamma = gamma;
    return v;
  };
  auto product = [&](float* a, float* b, float alpha, float beta, float* c, std::vector<EpiOut> outs) {
    ClassSpec s;
    s.A = Mat{a, DT_FP32, n, n, ldn, pl}, s.B = Mat{b, DT_FP32, n, n, ldn, pl};
    s.symmetric = true, s.a_sym = true, s.b_sym = true, s.split = true;
    s.M = n, s.N = n, s.K = n, s.batch = batch;
    s.bn = pick_bn(n, n, batch, true);
    s.alpha = alpha, s.beta = beta;
    if (c != nullptr) s.C = c, s.c_dt = DT_FP32, s.ldc = ldn, s.c_bs = 2 * pl, s.c_plane = pl;
    s.outs = std::move(outs);
    return s;
  };
  int cm = 0, cx = 0;  // M_{j-1} in M[cm], X_j in X[cx]
  for (int j = 1; j < iters; ++j) {
    st = ch.add(product(w.M[cm], w.M[cm], 1.0f / 16, -10.0f / 16, w.M[cm], planes(w.T2, 25.0f / 16)),
                {{w.M[cm], DEP_TMN}}, w.M[cm], {w.T2});
    if (st != MSIGN_OK) return st;
    st = ch.add(product(w.T2, w.T2, 1.0f, 0.0f, nullptr, planes(w.T4, 0.0f)), {{w.T2, DEP_TMN}}, nullptr, {w.T4});
    if (st != MSIGN_OK) return st;
    st = ch.add(product(w.T4, w.M[cm], 1.0f, 0.0f, nullptr, planes(w.M[cm ^ 1], 0.0f)),
                {{w.T4, DEP_TM}, {w.M[cm], DEP_TN}}, nullptr, {w.M[cm ^ 1]});
    if (st != MSIGN_OK) return st;
    cm ^= 1;
    const bool last = j + 1 == iters;
    ClassSpec x = product(w.X[cx], w.M[cm], -0.25f, 1.25f, w.X[cx],
                          last ? std::vector<EpiOut>{out_to(out, DT_FP32, n, n * n, false)} : planes(w.X[cx ^ 1], 0.0f));
    x.mirror = last;  // the user gets the full, exactly symmetric matrix
    st = ch.add(x, {{w.X[cx], DEP_TM}, {w.M[cm], DEP_TN}}, w.X[cx],
                {last ? static_cast<const void*>(out) : static_cast<const void*>(w.X[cx ^ 1])});
    if (st != MSIGN_OK) return st;
    cx ^= 1;
  }
  return ch.flush();
}

struct MousseBuffers {
  void* Lb;  // bf16 L^(-1/4), rows x ldr
  void* Rb;  // bf16 R^(-1/4), cols x ldc
  void* B1;  // bf16 rows x ldc: G, then G~, then L^(-1/4) O
  void* B2;  // bf16 rows x ldc: L^(-1/4) G, then O = msign(G~)
  void* ns;  // msign workspace
};

void carve_mousse(Carver& cv, int64_t batch, int64_t rows, int64_t cols, MousseBuffers* b) {
  const int64_t ldr = round_up(rows, 8), ldc = round_up(cols, 8);
  b->Lb = cv.take(2ull * batch * rows * ldr);
  b->Rb = cv.take(2ull * batch * cols * ldc);
  b->B1 = cv.take(2ull * batch * rows * ldc);
  b->B2 = cv.take(2ull * batch * rows * ldc);
  b->ns = cv.take(msign_ns_workspace_size(batch, rows, cols, MSIGN_BF16));
}

}  // namespace msb

extern "C" {

size_t mousse_inv_root_workspace_size(int64_t batch, int64_t n) {
  if (batch <= 0 || n <= 0) return 0;
  Carver cv(nullptr);
  RootBuffers b;
  carve_root(cv, batch, n, &b);
  return cv.off + 1024;
}

msign_status mousse_inv_root(const float* A, float* out, int64_t batch, int64_t n, float eps, int iters,
                             void* workspace, size_t workspace_bytes, msign_stream_t stream) {
  if (batch < 0 || n < 0 || !std::isfinite(eps) || eps < 0.0f) return MSIGN_ERR_INVALID_ARG;
  if (iters <= 0) iters = kRootDefaultIters;
  if (iters < 2 || iters > kRootMaxIters) return MSIGN_ERR_INVALID_ARG;
  if (batch == 0 || n == 0) return MSIGN_OK;
  if (A == nullptr || out == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (batch > 65535 || n > (1 << 20)) return MSIGN_ERR_UNSUPPORTED;
  const size_t need = mousse_inv_root_workspace_size(batch, n);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  msign_status st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  return root_run(A, out, batch, n, eps, iters, workspace, reinterpret_cast<cudaStream_t>(stream));
}

size_t mousse_direction_workspace_size(int64_t batch, int64_t rows, int64_t cols) {
  if (batch <= 0 || rows <= 0 || cols <= 0) return 0;
  Carver cv(nullptr);
  MousseBuffers b;
  carve_mousse(cv, batch, rows, cols, &b);
  return cv.off + 1024;
}

msign_status mousse_direction(const void* G, void* out, msign_dtype io_dtype, int64_t batch, int64_t rows,
                              int64_t cols, const float* L_root, const float* R_root, const msign_coeffs* coeffs,
                              void* workspace, size_t workspace_bytes, msign_stream_t stream_) {
  if (!valid_dtype(io_dtype) || batch < 0 || rows < 0 || cols < 0) return MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return st;
  if (sch.method != 0) return MSIGN_ERR_INVALID_ARG;  // standard NS inside the whitened space
  if (batch == 0 || rows == 0 || cols == 0) return MSIGN_OK;
  if (G == nullptr || out == nullptr || L_root == nullptr || R_root == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (batch > 65535 || rows > (1 << 30) || cols > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
  const size_t need = mousse_direction_workspace_size(batch, rows, cols);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  const int io = to_dt(io_dtype);
  const int64_t ldr = round_up(rows, 8), ldc = round_up(cols, 8);
  const int64_t rect = rows * ldc;
  Carver cv(workspace);
  MousseBuffers w;
  carve_mousse(cv, batch, rows, cols, &w);
  // bf16 operand copies of G and of the two roots
  st = launch_ingest(ingest_args(G, io, rows, cols, false, DT_BF16, w.B1, DT_BF16, ldc, rect), batch, stream);
  if (st != MSIGN_OK) return st;
  st = launch_ingest(ingest_args(L_root, DT_FP32, rows, rows, false, DT_BF16, w.Lb, DT_BF16, ldr, rows * ldr), batch,
                     stream);
  if (st != MSIGN_OK) return st;
  st = launch_ingest(ingest_args(R_root, DT_FP32, cols, cols, false, DT_BF16, w.Rb, DT_BF16, ldc, cols * ldc), batch,
                     stream);
  if (st != MSIGN_OK) return st;
  const Mat Lm{w.Lb, DT_BF16, rows, rows, ldr, rows * ldr};
  const Mat Rm{w.Rb, DT_BF16, cols, cols, ldc, cols * ldc};
  // L^(-1/4) Y: Y (rows x cols) is the MN-major B operand
  auto left = [&](void* y, std::vector<EpiOut> outs) {
    ClassSpec s;
    s.A = Lm, s.B = Mat{y, DT_BF16, rows, cols, ldc, rect}, s.b_mn = true;
    s.M = rows, s.N = cols, s.K = rows, s.batch = batch;
    s.bn = pick_bn(rows, cols, batch, false);
    s.outs = std::move(outs);
    return launch_grouped({s}, DT_BF16, stream);
  };
  // Y R^(-1/4): R^(-1/4) is symmetric, so its rows are the K-major B operand
  auto right = [&](void* y, std::vector<EpiOut> outs) {
    ClassSpec s;
    s.A = Mat{y, DT_BF16, rows, cols, ldc, rect}, s.B = Rm;
    s.M = rows, s.N = cols, s.K = cols, s.batch = batch;
    s.bn = pick_bn(rows, cols, batch, false);
    s.outs = std::move(outs);
    return launch_grouped({s}, DT_BF16, stream);
  };
  st = left(w.B1, {out_to(w.B2, DT_BF16, ldc, rect, false)});  // L^(-1/4) G
  if (st != MSIGN_OK) return st;
  st = right(w.B2, {out_to(w.B1, DT_BF16, ldc, rect, false)});  // G~ = L^(-1/4) G R^(-1/4)
  if (st != MSIGN_OK) return st;
  st = ns_run(w.B1, DT_BF16, ldc, rect, w.B2, DT_BF16, ldc, rect, MSIGN_BF16, batch, rows, cols, sch, w.ns,
              stream);  // O = msign(G~)
  if (st != MSIGN_OK) return st;
  st = left(w.B2, {out_to(w.B1, DT_BF16, ldc, rect, false)});  // L^(-1/4) O
  if (st != MSIGN_OK) return st;
  return right(w.B1, {out_to(out, io, cols, rows * cols, false)});  // ... R^(-1/4)
}

}  // extern "C"

// ---------------------------------------------------------------- no-allocation variant
//
// Some callers cannot allocate device memory at the point where they need
// msign: plugins hosted by a framework that owns all of the GPU's memory
// through its own pool, or real-time loops that forbid any allocation after
// start-up (cudaMalloc may synchronise the device).  msign_ns_noalloc()
// serves them from a fixed scratch array that lives in the library's own
// device image.

namespace msb {

// Built-in scratch for msign_ns_noalloc: 32 MiB, resident on every GPU that
// loads this library until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

}  // namespace msb

extern "C" {

size_t msign_ns_host_workspace_size(int64_t batch, int64_t rows, int64_t cols, msign_dtype io_dtype,
                                    msign_dtype compute_dtype) {
  if (batch <= 0 || rows <= 0 || cols <= 0 || !valid_dtype(io_dtype)) return 0;
  const uint64_t xb = static_cast<uint64_t>(batch) * rows * cols * (io_dtype == MSIGN_FP32 ? 4 : 2);
  return round_up(xb, 256) + msign_ns_workspace_size(batch, rows, cols, compute_dtype);
}

msign_status msign_ns_host(const void* in_host, void* out_host, msign_dtype io_dtype, msign_dtype compute_dtype,
                           int64_t batch, int64_t rows, int64_t cols, const msign_coeffs* coeffs, void* workspace,
                           size_t workspace_bytes, msign_stream_t stream_) {
  // msign_ns's checks first: nothing is enqueued on an argument error
  if (!valid_dtype(io_dtype) || !valid_dtype(compute_dtype)) return MSIGN_ERR_INVALID_ARG;
  if (batch < 0 || rows < 0 || cols < 0) return MSIGN_ERR_INVALID_ARG;
  Schedule sch;
  msign_status st = read_schedule(coeffs, kNsEps, &sch);
  if (st != MSIGN_OK) return st;
  if (sch.init != 0 && compute_dtype == MSIGN_FP32) return MSIGN_ERR_UNSUPPORTED;
  if (batch == 0 || rows == 0 || cols == 0) return MSIGN_OK;
  if (in_host == nullptr || out_host == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (batch > 65535 || rows > (1 << 30) || cols > (1 << 30)) return MSIGN_ERR_UNSUPPORTED;
  const size_t need = msign_ns_host_workspace_size(batch, rows, cols, io_dtype, compute_dtype);
  if (workspace == nullptr || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) % 256) != 0)
    return MSIGN_ERR_WORKSPACE;
  DeviceState* dev = nullptr;
  st = device_state(&dev);
  if (st != MSIGN_OK) return st;
  const size_t xb = static_cast<size_t>(batch) * rows * cols * (io_dtype == MSIGN_FP32 ? 4 : 2);
  const size_t xr = round_up(xb, 256);
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  void* dx = workspace;
  if (cudaMemcpyAsync(dx, in_host, xb, cudaMemcpyHostToDevice, stream) != cudaSuccess) return MSIGN_ERR_CUDA;
  st = msign_ns(dx, dx, io_dtype, compute_dtype, batch, rows, cols, 0, 0, coeffs, static_cast<char*>(workspace) + xr,
                workspace_bytes - xr, stream_);
  if (st != MSIGN_OK) return st;
  if (cudaMemcpyAsync(out_host, dx, xb, cudaMemcpyDeviceToHost, stream) != cudaSuccess) return MSIGN_ERR_CUDA;
  return MSIGN_OK;
}

size_t msign_ns_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

msign_status msign_ns_noalloc(const void* in, void* out, msign_dtype io_dtype, int64_t batch, int64_t rows,
                              int64_t cols, const msign_coeffs* coeffs, msign_stream_t stream) {
  if (!valid_dtype(io_dtype) || batch < 0 || rows < 0 || cols < 0) return MSIGN_ERR_INVALID_ARG;
  if (batch == 0 || rows == 0 || cols == 0) return MSIGN_OK;
  if (in == nullptr || out == nullptr) return MSIGN_ERR_INVALID_ARG;
  if (msign_ns_workspace_size(batch, rows, cols, MSIGN_BF16) > kNoAllocScratchBytes) return MSIGN_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MSIGN_ERR_CUDA;
  void* scratch = nullptr;
  {
    // The array's host-side name is only a stand-in; the device address of
    // this device's copy comes from cudaGetSymbolAddress, once per device.
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MSIGN_ERR_CUDA;
      g_noalloc_ptr[dev] = p;
    }
    scratch = g_noalloc_ptr[dev];
  }
  // msign_ns clears the state it needs at zero (tile claims, ingest tickets,
  // row-block counters) with a cudaMemsetAsync on `stream` before use, and
  // writes every other buffer it carves before reading it, so what an
  // earlier call left in the array does not matter.
  return msign_ns(in, out, io_dtype, MSIGN_BF16, batch, rows, cols, 0, 0, coeffs, scratch, kNoAllocScratchBytes,
                  stream);
}

}  // extern "C"
