// C ABI of libqlora.so: argument validation, workspace planning and the
// launch order of the quantizer, the dequantizer and the LoRA linear.
#include <cmath>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"

namespace qlora {

// ----------------------------------------------------------------- NF4 table
namespace {

// Standard normal quantile by Newton's method on the complementary error
// function, in extended precision.
long double normal_quantile(long double p) {
  long double x = 0.0L;
  const long double rt2 = sqrtl(2.0L);
  const long double inv_sqrt_2pi = 0.398942280401432677939946059934381868L;
  for (int it = 0; it < 200; ++it) {
    const long double f = 0.5L * erfcl(-x / rt2) - p;
    const long double d = inv_sqrt_2pi * expl(-0.5L * x * x);
    const long double step = f / d;
    x -= step;
    if (fabsl(step) < 1e-19L * (1.0L + fabsl(x))) break;
  }
  return x;
}

Nf4Table build_nf4_table() {
  // 8 positive quantiles at p = d + (1/2 - d) i / 8 and 7 negative ones at
  // p = d + (1/2 - d) i / 7 (i from 0), an exact zero, scaled so the
  // extreme levels are -1 and +1.
  const long double d = 1.0L - (1.0L / 32.0L + 1.0L / 30.0L) / 2.0L;
  long double v[16];
  int k = 0;
  for (int i = 0; i < 7; ++i) v[k++] = -normal_quantile(d + (0.5L - d) * i / 7.0L);
  v[k++] = 0.0L;
  for (int i = 7; i >= 0; --i) v[k++] = normal_quantile(d + (0.5L - d) * i / 8.0L);
  long double top = 0.0L;
  for (int i = 0; i < 16; ++i) top = fmaxl(top, fabsl(v[i]));
  Nf4Table t{};
  for (int i = 0; i < 16; ++i) t.level[i] = static_cast<float>(v[i] / top);
  return t;
}

// Decision thresholds of an ascending table: code = #{ i : n > thresh[i] } is the
// nearest level with ties to the lower index.  thresh[i] = exact midpoint of
// level[i] and level[i+1] (representable in double) rounded toward -inf to fp32;
// between two equal levels the upper one is never nearer, so the threshold is
// the next one (code i+1 is skipped).
void set_thresholds(Nf4Table &t) {
  for (int i = 14; i >= 0; --i) {
    if (t.level[i] == t.level[i + 1] && i < 14) {
      t.thresh[i] = t.thresh[i + 1];
      continue;
    }
    const double mid = (static_cast<double>(t.level[i]) + static_cast<double>(t.level[i + 1])) * 0.5;
    float f = static_cast<float>(mid);
    if (static_cast<double>(f) > mid) f = nextafterf(f, -INFINITY);
    t.thresh[i] = f;
  }
}

Nf4Table build_table(int format) {
  Nf4Table t{};
  if (format == QLORA_FORMAT_NF4) {
    t = build_nf4_table();
  } else if (format == QLORA_FORMAT_FP4) {
    // e2m1: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (scaled by 1/6 so the largest is 1);
    // codes 0..7 carry the negative values from -1 up to -0, codes 8..15 +0 up to +1
    const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    for (int i = 0; i < 8; ++i) {
      t.level[7 - i] = -mag[i] / 6.0f;
      t.level[8 + i] = mag[i] / 6.0f;
    }
  } else {   // QLORA_FORMAT_INT4
    for (int c = 0; c < 16; ++c) t.level[c] = static_cast<float>(c - 8) / 7.0f;
  }
  set_thresholds(t);
  return t;
}

std::atomic<uint64_t> g_wait_limit{2000000000ull};

__global__ void selftest_wait_kernel(uint64_t limit, int *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must give up.
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit)) latch_status(status, QLORA_ERR_DEVICE_TIMEOUT);
}

}  // namespace

const Nf4Table &format_table(int format) {
  static const Nf4Table t[3] = {build_table(QLORA_FORMAT_NF4), build_table(QLORA_FORMAT_FP4),
                                build_table(QLORA_FORMAT_INT4)};
  return t[format == QLORA_FORMAT_FP4 ? 1 : (format == QLORA_FORMAT_INT4 ? 2 : 0)];
}

const Nf4Table &nf4_table() { return format_table(QLORA_FORMAT_NF4); }

Nf4Table weight_table(const qlora_nf4_weight *w) {
  Nf4Table t = format_table(w->format);
  if (w->dq == QLORA_DQ_SIGNED) {
    const int64_t nb = ceil_div(w->rows * w->cols, kBlock);
    t.qx = 128u;
    t.offset = w->group_scale + ceil_div(nb, kGroup);
  }
  return t;
}

uint64_t wait_limit() { return g_wait_limit.load(); }

std::atomic<int> g_stream_k{QLORA_STREAM_K_AUTO};
int stream_k_mode() { return g_stream_k.load(); }

// ----------------------------------------------------------------- device status word
__device__ int g_device_status;

int *device_status_ptr() {
  static int *ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int *>(p);
  }
  return ptrs[dev];
}

// ----------------------------------------------------------------- side stream
// A low-priority stream per (host thread, device) on which the backward runs
// the dB and dA products while the dgrad GEMM occupies the main stream: the
// GEMM's CTAs are dispatched first, the adapter products fill the SMs its
// last, partial wave leaves idle.  Fork and join are event record / wait, so
// the pattern is also legal inside stream capture.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

SideStream *side_stream() {
  thread_local SideStream per_dev[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  SideStream &ss = per_dev[dev];
  if (!ss.s) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithPriority(&ss.s, cudaStreamNonBlocking, lo) != cudaSuccess) {
      ss.s = nullptr;
      return nullptr;
    }
    if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess)
      return nullptr;
  }
  return &ss;
}

// ----------------------------------------------------------------- kernel timing hook
namespace {
struct Prof {
  bool on = false;
  std::vector<cudaEvent_t> pool;                 // reused across enable() calls
  size_t next = 0;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pairs[kProfKinds];
  cudaEvent_t open[kProfKinds] = {};
  int64_t launches[kProfKinds] = {};
};
Prof &prof() {
  static Prof p;
  return p;
}
cudaEvent_t prof_event() {
  Prof &P = prof();
  if (P.next == P.pool.size()) {
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    P.pool.push_back(e);
  }
  return P.pool[P.next++];
}
}  // namespace

bool prof_on() { return prof().on; }

void prof_mark(int kind, bool begin, cudaStream_t st) {
  Prof &P = prof();
  if (!P.on || kind <= 0 || kind >= kProfKinds) return;
  cudaEvent_t e = prof_event();
  if (!e) return;
  if (cudaEventRecord(e, st) != cudaSuccess) {   // no timing for this launch (the error is left for the next check)
    if (!begin) P.open[kind] = nullptr;
    return;
  }
  if (begin) {
    P.open[kind] = e;
  } else if (P.open[kind]) {
    P.pairs[kind].emplace_back(P.open[kind], e);
    P.open[kind] = nullptr;
    ++P.launches[kind];
    ++P.launches[kProfAll];
  }
}

// ----------------------------------------------------------------- tensor maps
namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}
}  // namespace

bool make_tmap_2d(CUtensorMap *tm, const void *base, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(tm, dtype, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ----------------------------------------------------------------- workspace plan
namespace {

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
  // byte offsets into the workspace
  size_t part = 0, H = 0, sH = 0, Hs = 0, Gb = 0, Gs = 0, sk = 0, total = 0;
  bool has_sk = false;   // the fused GEMMs run on CTA pairs: room for their stream-K tail
  size_t min_total = 0;  // without the stream-K tail (the last region, optional)
  // the stream-K region when the caller's workspace holds it, else null
  void *sk_region(void *ws, size_t ws_bytes) const {
    return has_sk && ws_bytes >= total ? static_cast<char *>(ws) + sk : nullptr;
  }
  int spH = 1, spG = 1, spB = 1, spA = 1;
  int64_t kpsH = 0, kpsG = 0, kpsB = 0, kpsA = 0;
  bool gemv = false;
};

// `packed`: the base weight is a packed NF4 weight (the few-token and
// one-CTA kernels may run); a dense W' always takes the pair kernel.
Plan make_plan(int op, int64_t M, int64_t N, int64_t K, int r, bool packed = true) {
  Plan p;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up(bytes);
    return o;
  };
  const size_t Mr = static_cast<size_t>(M) * r;
  if (op == QLORA_OP_FWD && packed && M <= kGemvMaxTokens && gemv_enabled()) {
    p.gemv = true;
    p.part = take(gemv_workspace_bytes(M, N, K, r));
    p.total = p.min_total = off;
    return p;
  }
  skinny_plan(M, r, K, &p.spH, &p.kpsH);
  size_t part = skinny_part_floats(M, r, p.spH);
  if (op == QLORA_OP_BWD) {
    skinny_plan(M, r, N, &p.spG, &p.kpsG);
    // dB and dA share one launch (one split count over their tiles together)
    skinny_plan_pair(N, 2 * r, 2 * r, K, M, &p.spB, &p.kpsB);
    p.spA = p.spB;
    p.kpsA = p.kpsB;
    part = std::max(part, skinny_part_floats(M, r, p.spG));
    part = std::max(part, skinny_part_floats(N, 2 * r, p.spB) + skinny_part_floats(2 * r, K, p.spA));
  }
  p.part = take(part * 4);
  p.H = take(Mr * 4);
  if (op == QLORA_OP_FWD) {
    p.sH = take(Mr * 2);
  } else {
    p.Hs = take(Mr * 2 * 2);
    p.Gb = take(Mr * 2);
    p.Gs = take(Mr * 2 * 2);
  }
  p.min_total = off;
  if (!packed || M > kPairMinRows) {
    p.has_sk = true;
    p.sk = take(pair_sk_workspace_bytes(M));
  }
  p.total = off;
  return p;
}

template <typename T>
T *at(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

qlora_status check_weight(const qlora_nf4_weight *w) {
  if (!w || !w->codes || !w->absmax_q || !w->group_scale) return QLORA_ERR_INVALID_ARG;
  if (w->rows < 1 || w->cols < 1) return QLORA_ERR_INVALID_ARG;
  if (w->format < QLORA_FORMAT_NF4 || w->format > QLORA_FORMAT_INT4) return QLORA_ERR_INVALID_ARG;
  if (w->dq != QLORA_DQ_PLAIN && w->dq != QLORA_DQ_SIGNED) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(w->codes) || !aligned16(w->absmax_q) || !aligned16(w->group_scale)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// Shape, pointer and alignment checks shared by the linear calls (no workspace).
qlora_status check_linear_shape(int64_t N, int64_t K, int64_t M, int r, float s, const void *X, const void *A,
                                const void *B, const void *out) {
  if (!X || !A || !B || !out) return QLORA_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || M < 1 || r < 8 || r > 256 || !std::isfinite(s)) return QLORA_ERR_INVALID_ARG;
  if (r % 8 != 0 || K % 64 != 0 || N % 8 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 1)
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(out)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

qlora_status check_linear(const qlora_nf4_weight *w, int64_t M, int r, float s, const void *X, const void *A,
                          const void *B, const void *out) {
  qlora_status st = check_weight(w);
  if (st != QLORA_OK) return st;
  return check_linear_shape(w->rows, w->cols, M, r, s, X, A, B, out);
}

// Where the fused GEMMs take the base weight from: a packed NF4 weight, or a
// dense bf16 W' [N, K] the caller materialized (any quantizer's output).
struct WeightSrc {
  const qlora_nf4_weight *w;
  const uint16_t *dense;
  int64_t N, K;
};

QGemmArgs gemm_args(const WeightSrc &src, bool dgrad, int64_t M, const uint16_t *act, const uint16_t *lora_act,
                    const uint16_t *lora_w, int r, uint16_t *out) {
  QGemmArgs g{};
  g.dgrad = dgrad;
  g.M = M;
  g.wN = src.N;
  g.wK = src.K;
  g.act = act;
  g.lora_act = lora_act;
  g.lora_w = lora_w;
  g.r = r;
  g.out = out;
  if (src.w) {
    g.codes = src.w->codes;
    g.absmax_q = src.w->absmax_q;
    g.group_scale = src.w->group_scale;
    g.tab = weight_table(src.w);
  } else {
    g.tab = format_table(QLORA_FORMAT_NF4);
    g.wdense = src.dense;
  }
  return g;
}

qlora_status check_ws(const void *ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

#define QL_CUDA(expr)                                 \
  do {                                                \
    if ((expr) != cudaSuccess) return QLORA_ERR_CUDA; \
  } while (0)
#define QL_TRY(expr)                          \
  do {                                        \
    const qlora_status _s = (expr);           \
    if (_s != QLORA_OK) return _s;            \
  } while (0)

// H = X A^T into H (fp32) and bf16(s*H) into sH; optional hi/lo copy into Hs.
qlora_status run_h(const Plan &p, void *ws, const uint16_t *X, const uint16_t *A, int64_t M, int64_t K, int r,
                   float s, float *H, uint16_t *sH, uint16_t *Hs, cudaStream_t st) {
  SkinnyArgs a{X, K, true, A, K, true, M, r, K, p.spH, p.kpsH, at<float>(ws, p.part)};
  a.ep.kind = kSkinnyH;
  a.ep.s = s;
  a.ep.out_f = H;
  a.ep.out_b = sH;
  a.ep.out_hl = Hs;
  if (skinny_fused_ok(a)) {
    QL_CUDA(launch_skinny(a, st));
    return QLORA_OK;
  }
  a.ep = SkinnyEpilogue{};
  QL_CUDA(launch_skinny(a, st));
  QL_CUDA(launch_finalize_h(at<float>(ws, p.part), p.spH, M, r, s, H, sH, Hs, st));
  return QLORA_OK;
}

}  // namespace

qlora_status validate_weight(const qlora_nf4_weight *w) { return check_weight(w); }

}  // namespace qlora

using namespace qlora;

extern "C" {

size_t qlora_codes_bytes(int64_t rows, int64_t cols) {
  return rows < 1 || cols < 1 ? 0 : static_cast<size_t>((rows * cols + 1) / 2);
}
size_t qlora_absmax_bytes(int64_t rows, int64_t cols) {
  return rows < 1 || cols < 1 ? 0 : static_cast<size_t>((rows * cols + kBlock - 1) / kBlock);
}
size_t qlora_group_scale_bytes(int64_t rows, int64_t cols) {
  const int64_t nb = (rows * cols + kBlock - 1) / kBlock;
  return rows < 1 || cols < 1 ? 0 : static_cast<size_t>((nb + kGroup - 1) / kGroup) * 4;
}
size_t qlora_group_scale_bytes_dq(int64_t rows, int64_t cols, int dq) {
  if (dq != QLORA_DQ_PLAIN && dq != QLORA_DQ_SIGNED) return 0;
  const size_t b = qlora_group_scale_bytes(rows, cols);
  return b == 0 ? 0 : b + (dq == QLORA_DQ_SIGNED ? 4 : 0);
}
size_t qlora_quantize_workspace_bytes(int64_t rows, int64_t cols, int dq) {
  if (rows < 1 || cols < 1 || dq != QLORA_DQ_SIGNED) return 0;
  return quantize_workspace_bytes(rows * cols);
}

const char *qlora_status_string(qlora_status st) {
  switch (st) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_INVALID_ARG: return "QLORA_ERR_INVALID_ARG";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "QLORA_ERR_UNSUPPORTED_SHAPE";
    case QLORA_ERR_MISALIGNED: return "QLORA_ERR_MISALIGNED";
    case QLORA_ERR_NONFINITE: return "QLORA_ERR_NONFINITE";
    case QLORA_ERR_DEVICE_TIMEOUT: return "QLORA_ERR_DEVICE_TIMEOUT";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE";
    case QLORA_ERR_BOUNDS: return "QLORA_ERR_BOUNDS";
  }
  return "QLORA_ERR_UNKNOWN";
}

qlora_status qlora_nf4_codebook(float *out) {
  if (!out) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out, nf4_table().level, sizeof(float) * 16);
  return QLORA_OK;
}

qlora_status qlora_format_codebook(int format, float *levels, float *thresh) {
  if (!levels || format < QLORA_FORMAT_NF4 || format > QLORA_FORMAT_INT4) return QLORA_ERR_INVALID_ARG;
  const Nf4Table &t = format_table(format);
  std::memcpy(levels, t.level, sizeof(float) * 16);
  if (thresh) std::memcpy(thresh, t.thresh, sizeof(float) * 15);
  return QLORA_OK;
}

uint64_t qlora_set_wait_limit(uint64_t cycles) { return g_wait_limit.exchange(cycles); }

int qlora_set_stream_k(int mode) {
  if (mode < QLORA_STREAM_K_OFF || mode > QLORA_STREAM_K_ALWAYS) return -1;
  return g_stream_k.exchange(mode);
}

void qlora_profile_enable(int on) {
  Prof &P = prof();
  P.on = on != 0;
  P.next = 0;
  for (int k = 0; k < kProfKinds; ++k) {
    P.pairs[k].clear();
    P.open[k] = nullptr;
    P.launches[k] = 0;
  }
}

qlora_status qlora_profile_read(int kind, double *ms_total, int64_t *launches) {
  if (kind < 0 || kind >= kProfKinds || !ms_total || !launches) return QLORA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return QLORA_ERR_CUDA;
  Prof &P = prof();
  double tot = 0.0;
  for (int k = (kind == kProfAll ? 1 : kind); k <= (kind == kProfAll ? kProfKinds - 1 : kind); ++k)
    for (auto &pr : P.pairs[k]) {
      float ms = 0.0f;
      if (cudaEventElapsedTime(&ms, pr.first, pr.second) != cudaSuccess) return QLORA_ERR_CUDA;
      tot += ms;
    }
  *ms_total = tot;
  *launches = P.launches[kind];
  return QLORA_OK;
}

qlora_status qlora_selftest_wait_timeout(uint64_t cycles, void *stream) {
  int *status = device_status_ptr();
  if (!status) return QLORA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(cycles, status);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_device_status(void *stream) {
  int *p = device_status_ptr();
  if (!p) return QLORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QLORA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return QLORA_ERR_CUDA;
  }
  return static_cast<qlora_status>(v);
}

size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r) {
  if (op < QLORA_OP_FWD || op > QLORA_OP_BWD_DENSE || M < 1 || N < 1 || K < 1 || r < 1) return 0;
  const bool dense = op == QLORA_OP_FWD_DENSE || op == QLORA_OP_BWD_DENSE;
  const int base = dense ? op - QLORA_OP_FWD_DENSE : op;
  return make_plan(base, M, N, K, r, !dense).total;
}

size_t qlora_workspace_min_bytes(int op, int64_t M, int64_t N, int64_t K, int r) {
  if (op < QLORA_OP_FWD || op > QLORA_OP_BWD_DENSE || M < 1 || N < 1 || K < 1 || r < 1) return 0;
  const bool dense = op == QLORA_OP_FWD_DENSE || op == QLORA_OP_BWD_DENSE;
  const int base = dense ? op - QLORA_OP_FWD_DENSE : op;
  return make_plan(base, M, N, K, r, !dense).min_total;
}

qlora_status qlora_quantize_nf4_ws(const void *W, int dtype, const qlora_nf4_weight *out, void *ws,
                                   size_t ws_bytes, void *stream) {
  if (!W || (dtype != QLORA_DTYPE_F32 && dtype != QLORA_DTYPE_BF16)) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_weight(out));
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  const int64_t numel = out->rows * out->cols;
  if (out->dq == QLORA_DQ_SIGNED) {
    if (numel >= (int64_t(1) << 38)) return QLORA_ERR_UNSUPPORTED_SHAPE;
    if (!ws || ws_bytes < quantize_workspace_bytes(numel)) return QLORA_ERR_WORKSPACE;
    if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  }
  int *status = device_status_ptr();
  if (!status) return QLORA_ERR_CUDA;
  QL_CUDA(launch_quantize(W, dtype, numel, out->codes, out->absmax_q, out->group_scale, weight_table(out),
                          out->dq == QLORA_DQ_SIGNED ? ws : nullptr, status, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

qlora_status qlora_quantize_nf4(const void *W, int dtype, const qlora_nf4_weight *out, void *stream) {
  return qlora_quantize_nf4_ws(W, dtype, out, nullptr, 0, stream);
}

qlora_status qlora_dequantize(const qlora_nf4_weight *w, uint16_t *W_out, void *stream) {
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_weight(w));
  if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
  QL_CUDA(launch_dequantize(w->codes, w->absmax_q, w->group_scale, w->rows * w->cols, weight_table(w),
                            W_out, static_cast<cudaStream_t>(stream)));
  return QLORA_OK;
}

}  // extern "C"

namespace {

qlora_status linear_fwd_impl(const WeightSrc &src, const uint16_t *X, int64_t M, const uint16_t *A,
                             const uint16_t *B, int r, float s, uint16_t *Y, float *H_out, void *ws, size_t ws_bytes,
                             void *stream) {
  const int64_t N = src.N, K = src.K;
  const Plan p = make_plan(QLORA_OP_FWD, M, N, K, r, src.w != nullptr);
  QL_TRY(check_ws(ws, ws_bytes, p.min_total));
  if (H_out && !aligned16(H_out)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float *H = H_out ? H_out : at<float>(ws, p.H);
  if (p.gemv) {
    const qlora_nf4_weight *w = src.w;
    GemvArgs g{M, N, K, X, w->codes, w->absmax_q, w->group_scale, A, B, r, s, Y, H_out, at<void>(ws, p.part),
               weight_table(w)};
    return launch_gemv(g, st);
  }
  QGemmArgs g = gemm_args(src, false, M, X, at<uint16_t>(ws, p.sH), B, r, Y);
  g.sk_ws = p.sk_region(ws, ws_bytes);
  // the GEMM's stream-K counters are cleared before H, so the GEMM follows H directly
  QL_TRY(qgemm_prepare_split(g, st, &g.sk_zeroed));
  QL_TRY(run_h(p, ws, X, A, M, K, r, s, H, at<uint16_t>(ws, p.sH), nullptr, st));
  return launch_qgemm(g, st);
}

qlora_status linear_bwd_impl(const WeightSrc &src, const uint16_t *X, const uint16_t *dY, int64_t M,
                             const uint16_t *A, const uint16_t *B, int r, float s, const float *H_saved,
                             uint16_t *dX, float *dA, float *dB, void *ws, size_t ws_bytes, void *stream) {
  const int64_t N = src.N, K = src.K;
  const Plan p = make_plan(QLORA_OP_BWD, M, N, K, r, src.w != nullptr);
  QL_TRY(check_ws(ws, ws_bytes, p.min_total));
  if (!aligned16(dY) || !aligned16(dA) || !aligned16(dB)) return QLORA_ERR_MISALIGNED;
  QGemmArgs dgrad = gemm_args(src, true, M, dY, at<uint16_t>(ws, p.Gb), A, r, dX);
  dgrad.sk_ws = p.sk_region(ws, ws_bytes);
  if (H_saved && !aligned16(H_saved)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the dgrad GEMM's stream-K counters are cleared before the products it depends on
  QL_TRY(qgemm_prepare_split(dgrad, st, &dgrad.sk_zeroed));
  float *part = at<float>(ws, p.part);
  uint16_t *Hs = at<uint16_t>(ws, p.Hs);
  uint16_t *Gb = at<uint16_t>(ws, p.Gb);
  uint16_t *Gs = at<uint16_t>(ws, p.Gs);

  // H (recomputed when not saved) as a hi/lo bf16 pair for dB.  With a saved H
  // the split is done by the G product's epilogue (fused path) or a small kernel.
  bool hs_pending = false;
  if (H_saved) {
    hs_pending = true;
  } else {
    QL_TRY(run_h(p, ws, X, A, M, K, r, s, at<float>(ws, p.H), Gb /* scratch for s*H, overwritten below */, Hs,
                 st));
  }
  // G = s dY B  -> Gb (dgrad operand) and Gs (hi/lo, for dA)
  {
    SkinnyArgs a{dY, N, true, B, r, false, M, r, N, p.spG, p.kpsG, part};
    a.ep.kind = kSkinnyG;
    a.ep.s = s;
    a.ep.out_b = Gb;
    a.ep.out_hl = Gs;
    if (hs_pending) {
      a.ep.aux = H_saved;
      a.ep.aux_hl = Hs;
    }
    if (skinny_fused_ok(a)) {
      QL_CUDA(launch_skinny(a, st));
      hs_pending = false;
    } else {
      a.ep = SkinnyEpilogue{};
      QL_CUDA(launch_skinny(a, st));
      QL_CUDA(launch_finalize_g(part, p.spG, M, r, s, Gb, Gs, st));
    }
  }
  if (hs_pending) QL_CUDA(launch_split_hilo(H_saved, M, r, Hs, st));
  // dB = s dY^T H  and  dA = G^T X
  SkinnyArgs aB{dY, N, false, Hs, 2 * static_cast<int64_t>(r), false, N, 2 * static_cast<int64_t>(r), M, p.spB,
                p.kpsB, part};
  aB.ep.kind = kSkinnyCols;
  aB.ep.s = s;
  aB.ep.out_f = dB;
  SkinnyArgs aA{Gs, 2 * static_cast<int64_t>(r), false, X, K, false, 2 * static_cast<int64_t>(r), K, M, p.spA,
                p.kpsA, part};
  aA.ep.kind = kSkinnyRows;
  aA.ep.out_f = dA;
  // Both finishing in-kernel (no shared partial buffer): one launch of the two,
  // on the side stream beside the dgrad GEMM.
  // (Off while the timing hook records, so that every kernel's events time it alone.)
  const bool paired = skinny_pair_ok(aB, aA);
  SideStream *side = (paired && !prof_on()) ? side_stream() : nullptr;
  if (side) {
    QL_CUDA(cudaEventRecord(side->fork, st));
    QL_CUDA(cudaStreamWaitEvent(side->s, side->fork, 0));
    // dX = dY W' + Gb A first, so that its CTAs are dispatched ahead of the products'
    const qlora_status gst = launch_qgemm(dgrad, st);
    QL_CUDA(launch_skinny_pair(aB, aA, side->s));
    QL_CUDA(cudaEventRecord(side->join, side->s));
    QL_CUDA(cudaStreamWaitEvent(st, side->join, 0));
    return gst;
  }
  if (paired) {
    QL_CUDA(launch_skinny_pair(aB, aA, st));
    return launch_qgemm(dgrad, st);
  }
  if (skinny_fused_ok(aB)) {
    QL_CUDA(launch_skinny(aB, st));
  } else {
    aB.ep = SkinnyEpilogue{};
    QL_CUDA(launch_skinny(aB, st));
    QL_CUDA(launch_finalize_cols(part, p.spB, N, r, s, dB, st));
  }
  if (skinny_fused_ok(aA)) {
    QL_CUDA(launch_skinny(aA, st));
  } else {
    aA.ep = SkinnyEpilogue{};
    QL_CUDA(launch_skinny(aA, st));
    QL_CUDA(launch_finalize_rows(part, p.spA, r, K, dA, st));
  }
  // dX = dY W' + Gb A
  return launch_qgemm(dgrad, st);
}

}  // namespace

extern "C" {

qlora_status qlora_linear_fwd(const qlora_nf4_weight *w, const uint16_t *X, int64_t M, const uint16_t *A,
                              const uint16_t *B, int r, float s, uint16_t *Y, float *H_out, void *ws,
                              size_t ws_bytes, void *stream) {
  if (!w) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear(w, M, r, s, X, A, B, Y));
  return linear_fwd_impl(WeightSrc{w, nullptr, w->rows, w->cols}, X, M, A, B, r, s, Y, H_out, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd(const qlora_nf4_weight *w, const uint16_t *X, const uint16_t *dY, int64_t M,
                              const uint16_t *A, const uint16_t *B, int r, float s, const float *H_saved,
                              uint16_t *dX, float *dA, float *dB, void *ws, size_t ws_bytes, void *stream) {
  if (!w || !dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear(w, M, r, s, X, A, B, dX));
  return linear_bwd_impl(WeightSrc{w, nullptr, w->rows, w->cols}, X, dY, M, A, B, r, s, H_saved, dX, dA, dB, ws,
                         ws_bytes, stream);
}

qlora_status qlora_linear_fwd_dense(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X, int64_t M,
                                    const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y, float *H_out,
                                    void *ws, size_t ws_bytes, void *stream) {
  if (!W) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear_shape(N, K, M, r, s, X, A, B, Y));
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  return linear_fwd_impl(WeightSrc{nullptr, W, N, K}, X, M, A, B, r, s, Y, H_out, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_dense(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X, const uint16_t *dY,
                                    int64_t M, const uint16_t *A, const uint16_t *B, int r, float s,
                                    const float *H_saved, uint16_t *dX, float *dA, float *dB, void *ws,
                                    size_t ws_bytes, void *stream) {
  if (!W || !dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear_shape(N, K, M, r, s, X, A, B, dX));
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  return linear_bwd_impl(WeightSrc{nullptr, W, N, K}, X, dY, M, A, B, r, s, H_saved, dX, dA, dB, ws, ws_bytes,
                         stream);
}

qlora_status qlora_linear_fwd_materialized(qlora_materialize_fn materialize, void *ctx, uint16_t *W_scratch,
                                           int64_t N, int64_t K, const uint16_t *X, int64_t M, const uint16_t *A,
                                           const uint16_t *B, int r, float s, uint16_t *Y, float *H_out, void *ws,
                                           size_t ws_bytes, void *stream) {
  if (!materialize || !W_scratch) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear_shape(N, K, M, r, s, X, A, B, Y));
  if (!aligned16(W_scratch)) return QLORA_ERR_MISALIGNED;
  QL_TRY(check_ws(ws, ws_bytes, make_plan(QLORA_OP_FWD, M, N, K, r, false).min_total));
  QL_TRY(materialize(ctx, W_scratch, N, K, stream));
  return qlora_linear_fwd_dense(W_scratch, N, K, X, M, A, B, r, s, Y, H_out, ws, ws_bytes, stream);
}

qlora_status qlora_linear_bwd_materialized(qlora_materialize_fn materialize, void *ctx, uint16_t *W_scratch,
                                           int64_t N, int64_t K, const uint16_t *X, const uint16_t *dY, int64_t M,
                                           const uint16_t *A, const uint16_t *B, int r, float s,
                                           const float *H_saved, uint16_t *dX, float *dA, float *dB, void *ws,
                                           size_t ws_bytes, void *stream) {
  if (!materialize || !W_scratch || !dY || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  QL_TRY(check_linear_shape(N, K, M, r, s, X, A, B, dX));
  if (!aligned16(W_scratch)) return QLORA_ERR_MISALIGNED;
  QL_TRY(check_ws(ws, ws_bytes, make_plan(QLORA_OP_BWD, M, N, K, r, false).min_total));
  QL_TRY(materialize(ctx, W_scratch, N, K, stream));
  return qlora_linear_bwd_dense(W_scratch, N, K, X, dY, M, A, B, r, s, H_saved, dX, dA, dB, ws, ws_bytes, stream);
}

}  // extern "C"
