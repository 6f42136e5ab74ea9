// Low-rank plus quantized decomposition of a frozen weight, W ~ Q + L1 L2.
//
// "LQ-LoRA: Low-rank Plus Quantized Matrix Decomposition for Efficient
// Language Model Finetuning", abstract: each pretrained matrix is split by an
// iterative algorithm into a high-precision low-rank part and a quantized
// part; finetuning keeps the quantized part fixed and trains the low-rank one.
// The alternation run here starts from the principal rank-r part of W and
// then repeats
//     Q = quantize(W - L1 L2);   L1 L2 = rank-r approximation of W - W'(Q)
// with the library's own quantizer.  The rank-r step is randomized subspace
// iteration (range finder with power iterations on a caller-given Gaussian
// test matrix, then the eigen-decomposition of the small l x l matrix B B^T).
//
// Every pass over the N x K residual R = W - W' reads W (fp32) and the packed
// weight and forms R on the fly; R is never stored.  The small l x l steps
// (Gram sums, Cholesky, triangular inverse, Jacobi eigen-decomposition) run in
// fp64 in one CTA each.  Reductions are split over CTAs with partial results
// summed in a fixed order, so a run is bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int kLqMaxL = 96;       // widest test matrix (l); keeps the l x l work in one CTA
constexpr int kLqThreads = 256;

// The quantized part as the kernels see it (absent for the first rank-r step,
// which factors W itself).
struct LqQuant {
  const uint8_t *codes;      // nullptr: no quantized part, R = W
  const uint8_t *absmax_q;
  const float *group_scale;
  Nf4Table tab;
};

// W'[e] (the bf16 value of the dequantized weight, as fp32) for flat index e;
// `lv` holds the 16 levels in shared memory.
__device__ __forceinline__ float lq_wq(const LqQuant &q, const float *lv, int64_t e, float mu) {
  const uint32_t code = (__ldg(q.codes + (e >> 1)) >> ((e & 1) * 4)) & 15u;
  const int64_t blk = e >> 6;
  const float ap = block_constant(__ldg(q.absmax_q + blk), __ldg(q.group_scale + (blk >> 8)), q.tab.qx, mu);
  return __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[code], ap)));
}

__device__ __forceinline__ void lq_load_levels(const LqQuant &q, float *lv, float *mu_s) {
  if (threadIdx.x < 16) lv[threadIdx.x] = q.tab.level[threadIdx.x];
  if (threadIdx.x == 0) *mu_s = q.codes ? dq_offset(q.tab) : 0.0f;
}

// Fixed-order block sum of one fp64 value per thread (256 threads).
__device__ double block_sum_f64(double v, double *red) {
  red[threadIdx.x] = v;
  __syncthreads();
  for (int s = kLqThreads / 2; s > 0; s >>= 1) {
    if (static_cast<int>(threadIdx.x) < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const double out = red[0];
  __syncthreads();
  return out;
}

// ---- low-rank residual -------------------------------------------------------
// Tile of 32 rows x 128 columns, thread (tx, ty) owns rows ty + 8 i and
// columns tx + 32 c.  P = sum_j L1[n, j] L2[j, k] is accumulated in fp64 in
// the order j = 0 .. r-1 (each product of two fp32 values is exact in fp64, so
// an FMA gives the same sum as a product then an add).  Outputs, each optional:
//   E[n, k] = fl32(fl64(W) - P)                       (quantizer input)
//   part[cta] = sum over the tile of (fl64(W - W') - P)^2, fl64(W) - P without
//   a quantized part (no L1: P = 0).
constexpr int kResRows = 32, kResCols = 128, kResJ = 32;

__global__ void __launch_bounds__(kLqThreads) lq_residual_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                                 const float *__restrict__ L1,
                                                                 const float *__restrict__ L2, int r, LqQuant q,
                                                                 float *__restrict__ E, double *__restrict__ part) {
  __shared__ float l1s[kResRows][kResJ + 1];
  __shared__ float l2s[kResJ][kResCols];
  __shared__ float lv[16];
  __shared__ float mu_s;
  __shared__ double red[kLqThreads];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kResRows, k0 = static_cast<int64_t>(blockIdx.x) * kResCols;
  lq_load_levels(q, lv, &mu_s);
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[i][c] = 0.0;
  if (L1 != nullptr) {
    for (int j0 = 0; j0 < r; j0 += kResJ) {
      for (int idx = threadIdx.x; idx < kResRows * kResJ; idx += kLqThreads) {
        const int rr = idx / kResJ, jj = idx % kResJ;
        const int64_t n = n0 + rr;
        l1s[rr][jj] = (n < N && j0 + jj < r) ? __ldg(L1 + n * r + j0 + jj) : 0.0f;
      }
      for (int idx = threadIdx.x; idx < kResJ * kResCols; idx += kLqThreads) {
        const int jj = idx / kResCols, cc = idx % kResCols;
        const int64_t k = k0 + cc;
        l2s[jj][cc] = (k < K && j0 + jj < r) ? __ldg(L2 + static_cast<int64_t>(j0 + jj) * K + k) : 0.0f;
      }
      __syncthreads();
      const int jn = min(kResJ, r - j0);
      for (int jj = 0; jj < jn; ++jj) {
        double a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = static_cast<double>(l1s[ty + 8 * i][jj]);
#pragma unroll
        for (int c = 0; c < 4; ++c) b[c] = static_cast<double>(l2s[jj][tx + 32 * c]);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[i][c] = __fma_rn(a[i], b[c], acc[i][c]);
      }
      __syncthreads();
    }
  } else {
    __syncthreads();   // levels and mu are visible
  }
  const float mu = mu_s;
  double sq = 0.0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = n0 + ty + 8 * i;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t k = k0 + tx + 32 * c;
      if (n < N && k < K) {
        const int64_t e = n * K + k;
        const float w = __ldg(W + e);
        if (E) E[e] = __double2float_rn(__dsub_rn(static_cast<double>(w), acc[i][c]));
        if (part) {
          double d = static_cast<double>(w);
          if (q.codes) d = __dsub_rn(d, static_cast<double>(lq_wq(q, lv, e, mu)));
          d = __dsub_rn(d, acc[i][c]);
          sq = __fma_rn(d, d, sq);
        }
      }
    }
  }
  if (part) {
    const double s = block_sum_f64(sq, red);
    if (threadIdx.x == 0) part[static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x] = s;
  }
}

// out[0] = sum of part[0 .. n) in index order (sum mode), or
// out[0] = sqrt(sum / *norm2) (relative error mode, norm2 != nullptr).
__global__ void lq_sum_kernel(const double *__restrict__ part, int64_t n, const double *__restrict__ norm2,
                              double *__restrict__ out) {
  __shared__ double red[kLqThreads];
  // thread t sums a contiguous stretch, then the stretches are added in order
  const int64_t per = (n + kLqThreads - 1) / kLqThreads;
  const int64_t a = static_cast<int64_t>(threadIdx.x) * per, b = min(n, a + per);
  double s = 0.0;
  for (int64_t i = a; i < b; ++i) s = __dadd_rn(s, part[i]);
  const double tot = block_sum_f64(s, red);
  if (threadIdx.x == 0) *out = norm2 ? (*norm2 > 0.0 ? sqrt(tot / *norm2) : 0.0) : tot;
}

// ---- Y = R M and Z = R^T Y on tensor cores ------------------------------------
// One CTA per SM: a 128-row tile of the output (rows n of R for Y = R M,
// columns k of R for Z = R^T Y) over one split of the reduction, walked 32
// deep per step.
//   warp 1   loader: lane 0 brings the step's 128 x 32 tile of W (128B-
//            swizzled), its codes and the small operand's two 32-deep tiles
//            (below) by TMA into a 3- or 4-stage ring (as shared memory
//            allows); all lanes fetch the block
//            constants (8-bit code, group scale) three steps ahead into
//            registers and store them beside the tile (their row stride,
//            K / 64 bytes, is not TMA-able in general).
//   warps 2-17 form R = fl32(W - W') from the ring (one run of 8 elements per
//            thread and step) and split it exactly as
//            R = Rh + Rl (Rh: R with the low 13 mantissa bits cleared, a tf32
//            value; Rl = R - Rh, exact in fp32), and write it K-major and
//            128-byte-swizzled into a 2-stage operand ring (transposed for Z's
//            R^T tile, lane = reduction index, so a warp's 4-byte stores hit
//            32 banks).  Elements outside the matrix or the split are zero (a
//            zero-filled code would decode as a level).
// The small operand (M or Y, [reduction, l]) is split the same way once per
// product by lq_tc_split_kernel into the layout the MMA reads: per 32-deep
// block, an hi and a lo tile of nl rows (l rounded up to 16; the extra rows
// zero) x 32 fp32, which the loader's TMA swizzles as it lands.
//   warp 0   one thread issues tcgen05.mma kind::tf32 (M = 128, N = l rounded
//            up to 16, K = 8) for Rh Bh + Rh Bl + Rl Bh into an fp32 TMEM
//            accumulator: the dropped Rl Bl term and the tensor core's
//            truncation of the low parts to tf32 leave about 2^-20 of |R| |B|
//            per product term, the level of an fp32 multiply-add.
// Warps 2-5 then write the tile's rows to part[split][row][c], and
// lq_sum_splits_kernel adds the splits in order.
// Operand-ring depth (compile-time tunable; three stages measured slightly slower than two).
#ifndef QLORA_LQ_OP_STAGES
#define QLORA_LQ_OP_STAGES 2
#endif
constexpr int kTcRows = 128, kTcRed = 32, kTcMaxRawStages = 4, kTcOpStages = QLORA_LQ_OP_STAGES, kTcProducers = 512;
constexpr int kTcThreads = 64 + kTcProducers;
constexpr int kTcATile = kTcRows * kTcRed * 4;          // 16 KB: one component of the R tile (and W's raw tile)
// raw stage: W tile (16 KB), codes (2 KB), the small operand's hi and lo tiles (nl x 128 B each, 1024-
// aligned for the swizzle), 8-bit constants, group scales
constexpr int kTcRawCodes = kTcATile, kTcRawB = kTcRawCodes + 2048;
__host__ __device__ constexpr int lq_tc_raw_q(int nl) { return kTcRawB + 2 * nl * kTcRed * 4; }
__host__ __device__ constexpr int lq_tc_raw_s(int nl) { return lq_tc_raw_q(nl) + 128; }
__host__ __device__ constexpr int lq_tc_raw_bytes(int nl) { return (lq_tc_raw_s(nl) + 128 * 4 + 1023) / 1024 * 1024; }
// raw stages that fit beside the operand ring in 227 KB
__host__ __device__ constexpr int lq_tc_raw_stages(int nl) {
  return (232448 - kTcOpStages * 2 * kTcATile - 1024 - 160) / lq_tc_raw_bytes(nl) >= kTcMaxRawStages
             ? kTcMaxRawStages
             : 3;
}
__host__ __device__ constexpr int lq_tc_smem(int nl) {
  return lq_tc_raw_stages(nl) * lq_tc_raw_bytes(nl) + kTcOpStages * 2 * kTcATile + 1024 + 160;
}
constexpr uint64_t kTcDrain = 4000000000ull;

// Byte offset of element (row, c), c < 32, in a K-major 128-byte-swizzled tile of 32-bit elements.
__device__ __forceinline__ uint32_t tc_off(int row, int c) {
  return static_cast<uint32_t>(row * 128 + ((((c >> 2) ^ row) & 7) << 4) + (c & 3) * 4);
}
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

__device__ __forceinline__ bool lq_wait(uint64_t *bar, uint32_t parity, uint64_t limit, volatile int *abort_flag,
                                        int *status) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > limit) {
      *abort_flag = 1;
      latch_status(status, QLORA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// The small operand [red, l] split for the products: Bt[(b * 2 + h) * nl + j][c]
// = component h (0: tf32-exact high part, 1: remainder) of B[32 b + c][j], zero
// for j >= l or 32 b + c >= red.  One thread per four consecutive c (16-byte
// stores of both components); the reads hit L2 (B is a few MB at most).
__global__ void __launch_bounds__(256) lq_tc_split_kernel(const float *__restrict__ B, int64_t red, int l, int nl,
                                                          int nblk, float *__restrict__ Bt) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nblk * nl * (kTcRed / 4)) return;
  const int c4 = e & 7, bj = e >> 3;
  const int b = bj / nl, j = bj - b * nl;
  float x[4], hv[4], lo[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int64_t r = static_cast<int64_t>(b) * kTcRed + 4 * c4 + t;
    x[t] = (j < l && r < red) ? __ldg(B + r * l + j) : 0.0f;
    hv[t] = tf32_hi(x[t]);
    lo[t] = __fsub_rn(x[t], hv[t]);
  }
  float *hi_row = Bt + (static_cast<int64_t>(b * 2) * nl + j) * kTcRed + 4 * c4;
  *reinterpret_cast<float4 *>(hi_row) = make_float4(hv[0], hv[1], hv[2], hv[3]);
  *reinterpret_cast<float4 *>(hi_row + static_cast<int64_t>(nl) * kTcRed) = make_float4(lo[0], lo[1], lo[2], lo[3]);
}

// The block constants a loader lane fetches for one step: rows lane + 32 j
// (Y = R M, one 64-block per row) or row lane, blocks 0 and 1 (Z = R^T Y).
struct TcConst {
  uint32_t q[4];
  float S[4];
};

template <bool TRANS>
__device__ __forceinline__ TcConst tc_const_load(const LqQuant &q, int64_t N, int64_t K, int64_t o0, int64_t r0,
                                                 int64_t rb, int lane) {
  TcConst c{};
  if (!q.codes) return c;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int64_t n, k;
    bool ok;
    if (!TRANS) {
      n = o0 + lane + 32 * j;
      k = r0;
      ok = n < N && r0 < rb;
    } else {
      n = r0 + lane;
      k = o0 + 64 * j;
      ok = j < 2 && n < rb && k < K;
    }
    if (ok) {
      const int64_t blk = (n * K + k) >> 6;
      c.q[j] = __ldg(q.absmax_q + blk);
      c.S[j] = __ldg(q.group_scale + (blk >> 8));
    }
  }
  return c;
}

template <bool TRANS>
__global__ void __launch_bounds__(kTcThreads, 1)
    lq_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmC,
                 const __grid_constant__ CUtensorMap tmB, int64_t N, int64_t K, LqQuant q, int l, int nl,
                 int64_t red_per, float *__restrict__ part, int *status, uint64_t wait_limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int op_bytes = 2 * kTcATile;
  const int raw_bytes = lq_tc_raw_bytes(nl), raw_q = lq_tc_raw_q(nl), raw_s = lq_tc_raw_s(nl);
  const int RS = lq_tc_raw_stages(nl);
  uint8_t *raw_ring = smem;
  uint8_t *op_ring = smem + RS * raw_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(op_ring + kTcOpStages * op_bytes);
  uint64_t *raw_full = bars, *raw_empty = bars + kTcMaxRawStages;
  uint64_t *op_full = bars + 2 * kTcMaxRawStages, *op_empty = op_full + kTcOpStages, *acc_full = op_empty + kTcOpStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  __shared__ float lv[16];
  __shared__ float mu_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t rows_total = TRANS ? K : N;   // output rows
  const int64_t o0 = static_cast<int64_t>(blockIdx.x) * kTcRows;
  const int64_t ra = static_cast<int64_t>(blockIdx.y) * red_per;
  const int64_t rb = min(TRANS ? N : K, ra + red_per);
  const int nsteps = rb > ra ? static_cast<int>((rb - ra + kTcRed - 1) / kTcRed) : 0;
  const bool quant = q.codes != nullptr;
  lq_load_levels(q, lv, &mu_s);
  if (threadIdx.x == 0) {
    for (int s = 0; s < RS; ++s) {
      mbar_init(&raw_full[s], 1 + 32);           // the TMA lane's expect-tx arrival + every loader lane's constants
      mbar_init(&raw_empty[s], kTcProducers + 1);   // + the MMAs' commit (they read the small tiles there)
    }
    for (int s = 0; s < kTcOpStages; ++s) {
      mbar_init(&op_full[s], kTcProducers);
      mbar_init(&op_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmB);
    if (quant) tma_prefetch_desc(&tmC);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const float mu = mu_s;

  if (warp == 0) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32_f32(kTcRows, nl);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % kTcOpStages, sr = i % RS;
        if (!lq_wait(&op_full[s], (i / kTcOpStages) & 1, wait_limit, abort_flag, status) ||
            !lq_wait(&raw_full[sr], (i / RS) & 1, wait_limit, abort_flag, status))
          break;
        tc_fence_after();
        const uint32_t ah = smem_addr(op_ring + s * op_bytes), al = ah + kTcATile;
        const uint32_t bh = smem_addr(raw_ring + sr * raw_bytes + kTcRawB), bl = bh + nl * kTcRed * 4;
        for (int kk = 0; kk < kTcRed / 8; ++kk) {   // K = 8 tf32 = 32 bytes per MMA
          const uint64_t dah = sdesc_sw128(ah + kk * 32, 16, 1024), dal = sdesc_sw128(al + kk * 32, 16, 1024);
          const uint64_t dbh = sdesc_sw128(bh + kk * 32, 16, 1024), dbl = sdesc_sw128(bl + kk * 32, 16, 1024);
          tc_mma_tf32(tmem, dah, dbh, idesc, (i | kk) != 0 ? 1u : 0u);
          tc_mma_tf32(tmem, dah, dbl, idesc, 1u);
          tc_mma_tf32(tmem, dal, dbh, idesc, 1u);
        }
        tc_commit(&op_empty[s]);
        tc_commit(&raw_empty[sr]);
      }
      tc_commit(acc_full);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- loader
    const uint32_t bytes = static_cast<uint32_t>(kTcATile + (quant ? 2048 : 0) + 2 * nl * kTcRed * 4);
    // three register slots used in place (slot u of step i is reloaded for step i + 3 right after it
    // is stored), so no instruction ever waits on a constant load still in flight
    TcConst c[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) c[u] = tc_const_load<TRANS>(q, N, K, o0, ra + u * kTcRed, rb, lane);
    bool stop = false;
#pragma unroll 1
    for (int i0 = 0; i0 < nsteps && !stop; i0 += 3) {
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int i = i0 + u;
        if (i >= nsteps || stop) break;
        const int s = i % RS;
        const int64_t r0 = ra + static_cast<int64_t>(i) * kTcRed;
        if (i >= RS && !lq_wait(&raw_empty[s], ((i / RS) & 1) ^ 1, wait_limit, abort_flag, status)) {
          stop = true;
          break;
        }
        uint8_t *st = raw_ring + s * raw_bytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&raw_full[s], bytes);
          if (!TRANS) {
            tma_load_2d(st, &tmW, &raw_full[s], static_cast<int>(r0), static_cast<int>(o0));
            if (quant)
              tma_load_2d(st + kTcRawCodes, &tmC, &raw_full[s], static_cast<int>(r0 / 2), static_cast<int>(o0));
          } else {
            for (int b = 0; b < 4; ++b)
              tma_load_2d(st + 4096 * b, &tmW, &raw_full[s], static_cast<int>(o0) + 32 * b, static_cast<int>(r0));
            if (quant)
              tma_load_2d(st + kTcRawCodes, &tmC, &raw_full[s], static_cast<int>(o0 / 2), static_cast<int>(r0));
          }
          const int blk = static_cast<int>(r0 / kTcRed);   // the small operand's hi and lo tiles of this block
          tma_load_2d(st + kTcRawB, &tmB, &raw_full[s], 0, 2 * blk * nl);
          tma_load_2d(st + kTcRawB + nl * kTcRed * 4, &tmB, &raw_full[s], 0, (2 * blk + 1) * nl);
        }
        uint8_t *qs = st + raw_q;
        float *ss = reinterpret_cast<float *>(st + raw_s);
#pragma unroll
        for (int j = 0; j < (TRANS ? 2 : 4); ++j) {
          const int idx = TRANS ? lane * 2 + j : lane + 32 * j;
          qs[idx] = static_cast<uint8_t>(c[u].q[j]);
          ss[idx] = c[u].S[j];
        }
        mbar_arrive(&raw_full[s]);
        c[u] = tc_const_load<TRANS>(q, N, K, o0, r0 + 3 * kTcRed, rb, lane);
      }
    }
  } else {
    // ---------------------------------------------------------------- producers
    const int pt = threadIdx.x - 64, pw = pt >> 5;
    for (int i = 0; i < nsteps; ++i) {
      const int sr = i % RS, so = i % kTcOpStages;
      const int64_t r0 = ra + static_cast<int64_t>(i) * kTcRed;
      if (!lq_wait(&raw_full[sr], (i / RS) & 1, wait_limit, abort_flag, status)) break;
      if (i >= kTcOpStages && !lq_wait(&op_empty[so], ((i / kTcOpStages) & 1) ^ 1, wait_limit, abort_flag, status))
        break;
      const uint8_t *st = raw_ring + sr * raw_bytes;
      const uint8_t *qs = st + raw_q;
      const float *ss = reinterpret_cast<const float *>(st + raw_s);
      uint8_t *ah = op_ring + so * op_bytes, *al = ah + kTcATile;
      {
        // this thread's run of 8 elements: (tile row, reduction offset) for Y = R M,
        // (reduction row = lane, tile column 8 g) for Z = R^T Y
        int row, col, ci;
        uint32_t w_off, c_off;
        bool ok;
        if (!TRANS) {
          row = pt >> 2;                         // 8 rows x 4 runs per warp
          col = 8 * (pt & 3);
          w_off = static_cast<uint32_t>(row * 128);
          c_off = static_cast<uint32_t>(row * 16 + (pt & 3) * 4);
          ci = row;
          ok = o0 + row < N && r0 + col < rb;
        } else {
          const int g = pw;                      // 16 groups of 8 tile columns, lane = reduction row
          row = lane;
          col = 8 * g;
          w_off = static_cast<uint32_t>(4096 * (g >> 2) + lane * 128);
          c_off = static_cast<uint32_t>(lane * 64 + g * 4);
          ci = lane * 2 + (g >> 3);
          ok = r0 + lane < rb && o0 + col < K;
        }
        const int cc = TRANS ? 8 * ((col >> 3) & 3) : col;   // column within the 32-wide swizzled raw tile
        const float4 wa = *reinterpret_cast<const float4 *>(st + w_off + ((((cc >> 2) ^ row) & 7) << 4));
        const float4 wb = *reinterpret_cast<const float4 *>(st + w_off + (((((cc >> 2) + 1) ^ row) & 7) << 4));
        const float w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
        float rv[8];
        if (!ok) {
#pragma unroll
          for (int t = 0; t < 8; ++t) rv[t] = 0.0f;
        } else if (!quant) {
#pragma unroll
          for (int t = 0; t < 8; ++t) rv[t] = w[t];
        } else {
          const uint32_t codes = *reinterpret_cast<const uint32_t *>(st + kTcRawCodes + c_off);
          const float ap = block_constant(qs[ci], ss[ci], q.tab.qx, mu);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float wq = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[(codes >> (4 * t)) & 15u], ap)));
            rv[t] = __fsub_rn(w[t], wq);
          }
        }
        float hv[8], lo[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          hv[t] = tf32_hi(rv[t]);
          lo[t] = __fsub_rn(rv[t], hv[t]);
        }
        if (!TRANS) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t off = tc_off(row, col + 4 * h);
            *reinterpret_cast<float4 *>(ah + off) = make_float4(hv[4 * h], hv[4 * h + 1], hv[4 * h + 2], hv[4 * h + 3]);
            *reinterpret_cast<float4 *>(al + off) = make_float4(lo[4 * h], lo[4 * h + 1], lo[4 * h + 2], lo[4 * h + 3]);
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint32_t off = tc_off(col + t, lane);
            *reinterpret_cast<float *>(ah + off) = hv[t];
            *reinterpret_cast<float *>(al + off) = lo[t];
          }
        }
      }
      fence_proxy_async_smem();   // generic-proxy writes visible to the tensor core
      mbar_arrive(&op_full[so]);
      mbar_arrive(&raw_empty[sr]);
    }
    // epilogue: warps 2..5 hold TMEM lanes 32 (warp % 4) .. + 31 = output rows of the tile
    if (warp <= 5) {
      const bool ok = mbar_wait(acc_full, 0, kTcDrain);
      tc_fence_after();
      const bool live = __all_sync(0xffffffffu, ok && *abort_flag == 0 && nsteps > 0);
      const int quarter = warp & 3;
      const int64_t orow = o0 + quarter * 32 + lane;
      float *out = part + static_cast<int64_t>(blockIdx.y) * rows_total * l + orow * l;
      if (!ok) latch_status(status, QLORA_ERR_DEVICE_TIMEOUT);
      for (int c0 = 0; c0 < nl; c0 += 16) {
        uint32_t v[16];
        if (live) {
          tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + c0, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;   // empty or aborted split: zero
        }
        if (orow < rows_total) {
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (c0 + e < l) out[c0 + e] = __uint_as_float(v[e]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// Z[e] = sum over splits s = 0 .. ns-1 (in order) of part[s][e].
__global__ void lq_sum_splits_kernel(const float *__restrict__ part, int ns, int64_t n, float *__restrict__ Z) {
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = part[e];
    for (int i = 1; i < ns; ++i) s = __fadd_rn(s, part[static_cast<int64_t>(i) * n + e]);
    Z[e] = s;
  }
}

// ---- Gram matrices of tall fp32 matrices, in fp64 -----------------------------
// CTA (g, part): entries g * per_group + t + 256 m (t the thread) of the l x l
// matrix X^T X over the part's rows; each product of two fp32 values is exact
// in fp64.  part[p][e] holds the part sums; lq_gram_sum_kernel adds the parts
// in part order.
constexpr int kGramRows = 32;
constexpr int kGramGroups = 4;
constexpr int kGramMaxParts = 64;
constexpr int kGramPer = (kLqMaxL * kLqMaxL / kGramGroups + kLqThreads - 1) / kLqThreads;   // 9

__global__ void __launch_bounds__(kLqThreads) lq_gram_kernel(const float *__restrict__ X, int64_t rows, int l,
                                                             int64_t rows_per, double *__restrict__ part) {
  __shared__ float Xs[kGramRows][kLqMaxL];
  const int64_t na = static_cast<int64_t>(blockIdx.y) * rows_per, nb = min(rows, na + rows_per);
  const int ll = l * l;
  const int per_group = (ll + kGramGroups - 1) / kGramGroups;
  const int e0 = blockIdx.x * per_group, e1 = min(ll, e0 + per_group);
  double acc[kGramPer];
  int ea[kGramPer], eb[kGramPer];
#pragma unroll
  for (int m = 0; m < kGramPer; ++m) {
    const int e = e0 + threadIdx.x + kLqThreads * m;
    acc[m] = 0.0;
    ea[m] = e < e1 ? e / l : 0;
    eb[m] = e < e1 ? e % l : 0;
  }
  for (int64_t n0 = na; n0 < nb; n0 += kGramRows) {
    for (int idx = threadIdx.x; idx < kGramRows * l; idx += kLqThreads) {
      const int rr = idx / l, c = idx % l;
      Xs[rr][c] = (n0 + rr < nb) ? __ldg(X + (n0 + rr) * l + c) : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int rr = 0; rr < kGramRows; ++rr) {
#pragma unroll
      for (int m = 0; m < kGramPer; ++m)
        acc[m] = __fma_rn(static_cast<double>(Xs[rr][ea[m]]), static_cast<double>(Xs[rr][eb[m]]), acc[m]);
    }
    __syncthreads();
  }
  double *out = part + static_cast<int64_t>(blockIdx.y) * ll;
#pragma unroll
  for (int m = 0; m < kGramPer; ++m) {
    const int e = e0 + threadIdx.x + kLqThreads * m;
    if (e < e1) out[e] = acc[m];
  }
}

__global__ void lq_gram_sum_kernel(const double *__restrict__ part, int nparts, int ll, double *__restrict__ G) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= ll) return;
  double s = 0.0;
  for (int p = 0; p < nparts; ++p) s = __dadd_rn(s, part[static_cast<int64_t>(p) * ll + e]);
  G[e] = s;
}

// Row pitch of l x l fp64 matrices in shared memory: odd, so that a warp
// walking down a column touches every bank pair once.
__host__ __device__ __forceinline__ int lq_pitch(int l) { return l | 1; }

// G (global, l x l, dense) into shared memory with row pitch lp.
__device__ void lq_load_gram(const double *__restrict__ Gg, int l, int lp, double *G) {
  for (int e = threadIdx.x; e < l * l; e += blockDim.x) G[(e / l) * lp + e % l] = Gg[e];
  __syncthreads();
}

// ---- Cholesky and triangular inverse (one CTA) ---------------------------------
// G = L L^T (right-looking, column by column); a column whose pivot is not
// above 1e-24 of the largest diagonal entry is numerically dependent and is
// dropped (zero in L and in the inverse).  T = L^-T, so that X T has
// orthonormal columns when G = X^T X.
__global__ void __launch_bounds__(kLqThreads) lq_chol_inv_kernel(const double *__restrict__ Gg, int l,
                                                                 double *__restrict__ T) {
  extern __shared__ __align__(16) double lq_smem[];
  const int lp = lq_pitch(l);
  double *G = lq_smem;               // [l][lp]: lower triangle becomes L
  double *Xi = lq_smem + l * lp;     // [l][lp]: L^-1 (lower)
  __shared__ double dmax;
  __shared__ int dead[kLqMaxL];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  lq_load_gram(Gg, l, lp, G);
  if (threadIdx.x == 0) {
    double m = 0.0;
    for (int a = 0; a < l; ++a) m = fmax(m, G[a * lp + a]);
    dmax = m;
  }
  __syncthreads();
  const double tol = 1e-24 * dmax;
  // Right-looking elimination on the unscaled columns (one barrier per column):
  // G[a][b] -= G[a][j] G[b][j] / G[j][j] for j < b <= a; column j and the pivot
  // are not written in step j, so every thread reads them after the previous
  // step's barrier.  Afterwards L[a][j] = G[a][j] / sqrt(G[j][j]).
  for (int j = 0; j < l; ++j) {
    const double piv = G[j * lp + j];
    const double inv = piv > tol ? 1.0 / piv : 0.0;   // a dependent column is dropped
    for (int a = j + 1 + warp; a < l; a += nwarps) {
      const double gaj = G[a * lp + j] * inv;
      for (int b = j + 1 + lane; b <= a; b += 32) G[a * lp + b] = __fma_rn(-gaj, G[b * lp + j], G[a * lp + b]);
    }
    __syncthreads();
  }
  __shared__ double rinv[kLqMaxL];
  for (int j = threadIdx.x; j < l; j += blockDim.x) {
    const double piv = G[j * lp + j];
    dead[j] = !(piv > tol);
    const double d = dead[j] ? 0.0 : sqrt(piv);
    rinv[j] = dead[j] ? 0.0 : 1.0 / d;
    G[j * lp + j] = d;
  }
  __syncthreads();
  for (int a = warp; a < l; a += nwarps)
    for (int j = lane; j < a; j += 32) G[a * lp + j] *= rinv[j];
  __syncthreads();
  // L^-1 by forward substitution, one column per thread (four partial sums per dot product)
  for (int c = threadIdx.x; c < l; c += blockDim.x) {
    for (int j = 0; j < l; ++j) {
      double v = 0.0;
      if (j >= c && !dead[j]) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        int i = c;
        for (; i + 3 < j; i += 4) {
          s0 = __fma_rn(G[j * lp + i], Xi[i * lp + c], s0);
          s1 = __fma_rn(G[j * lp + i + 1], Xi[(i + 1) * lp + c], s1);
          s2 = __fma_rn(G[j * lp + i + 2], Xi[(i + 2) * lp + c], s2);
          s3 = __fma_rn(G[j * lp + i + 3], Xi[(i + 3) * lp + c], s3);
        }
        for (; i < j; ++i) s0 = __fma_rn(G[j * lp + i], Xi[i * lp + c], s0);
        v = ((j == c ? 1.0 : 0.0) - ((s0 + s1) + (s2 + s3))) / G[j * lp + j];
      }
      Xi[j * lp + c] = v;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < l * l; e += blockDim.x) {
    const int a = e / l, b = e % l;
    T[e] = Xi[b * lp + a];
  }
}

// ---- small right factor: out = X S (X fp32 [rows, l], S fp64 [l, cols]) -------
// fp64 accumulation, fp32 result; `transposed` stores out[c][n] ([cols, rows]).
constexpr int kSgRows = 32;

__global__ void __launch_bounds__(kLqThreads) lq_small_gemm_kernel(const float *__restrict__ X, int64_t rows, int l,
                                                                   const double *__restrict__ S, int cols,
                                                                   float *__restrict__ out, int transposed) {
  extern __shared__ __align__(16) double lq_smem[];
  double *Ss = lq_smem;                                        // [l][cols]
  float *Xs = reinterpret_cast<float *>(lq_smem + l * cols);   // [kSgRows][l]
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * kSgRows;
  for (int e = threadIdx.x; e < l * cols; e += blockDim.x) Ss[e] = S[e];
  for (int idx = threadIdx.x; idx < kSgRows * l; idx += blockDim.x) {
    const int rr = idx / l, c = idx % l;
    Xs[idx] = (n0 + rr < rows) ? __ldg(X + (n0 + rr) * l + c) : 0.0f;
  }
  __syncthreads();
  for (int c = tx; c < cols; c += 32) {
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int j = 0; j < l; ++j) {
      const double s = Ss[j * cols + c];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = __fma_rn(static_cast<double>(Xs[(4 * ty + i) * l + j]), s, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t n = n0 + 4 * ty + i;
      if (n < rows) {
        if (transposed)
          out[static_cast<int64_t>(c) * rows + n] = __double2float_rn(acc[i]);
        else
          out[n * cols + c] = __double2float_rn(acc[i]);
      }
    }
  }
}

// ---- symmetric eigen-decomposition (one CTA), parallel cyclic Jacobi ------------
// C = sum of Gram parts (l x l, l even).  Each sweep pairs all indices in l - 1
// rounds (circle method: index l-1 stays, the others rotate), the l/2 disjoint
// rotations of a round are applied together: A <- J^T A J, V <- V J, with
// c, s from the symmetric 2x2 Schur step (t = sign(tau) / (|tau| + sqrt(1 +
// tau^2)), tau = (a_qq - a_pp) / (2 a_pq)).  Sweeps stop when the off-diagonal
// mass is below 1e-24 of the total (entries about 1e-12 of the matrix; fp64
// rounding alone leaves about l^2 1e-32), at most kJacobiSweeps.  Then the r largest
// eigenvalues lam (ties to the lower index), s = sqrt(lam), and
//   M1[:, i] = v_i sqrt(s_i),  M2[:, i] = v_i / sqrt(s_i)
// (zero for s_i <= 1e-12 s_0), so that with C = B B^T and B = Q^T R:
// L1 = Q M1, L2^T = B^T M2.
constexpr int kJacobiSweeps = 30;

__global__ void __launch_bounds__(kLqThreads) lq_jacobi_kernel(const double *__restrict__ Gg, int l, int r,
                                                               double *__restrict__ M1, double *__restrict__ M2,
                                                               double *__restrict__ sv) {
  extern __shared__ __align__(16) double lq_smem[];
  const int lp = lq_pitch(l);
  double *A = lq_smem;               // [l][lp]
  double *V = lq_smem + l * lp;      // [l][lp]
  __shared__ double cs[kLqMaxL / 2][2];
  __shared__ int pr[kLqMaxL / 2][2];
  __shared__ double red[kLqThreads];
  __shared__ int order[kLqMaxL];
  __shared__ int taken[kLqMaxL];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  lq_load_gram(Gg, l, lp, A);
  for (int e = threadIdx.x; e < l * l; e += blockDim.x) V[(e / l) * lp + e % l] = (e / l == e % l) ? 1.0 : 0.0;
  __syncthreads();
  const int h = l / 2;
  for (int sweep = 0; sweep < kJacobiSweeps; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int a = warp; a < l; a += nwarps)
      for (int b = lane; b < l; b += 32) {
        const double v = A[a * lp + b] * A[a * lp + b];
        tot += v;
        if (a != b) off += v;
      }
    off = block_sum_f64(off, red);
    tot = block_sum_f64(tot, red);
    if (!(off > 1e-24 * tot)) break;
    for (int round = 0; round < l - 1; ++round) {
      if (static_cast<int>(threadIdx.x) < h) {
        const int i = threadIdx.x;
        int p, q;
        if (i == 0) {
          p = round;
          q = l - 1;
        } else {
          p = (round + i) % (l - 1);
          q = (round - i + (l - 1)) % (l - 1);
        }
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        const double apq = A[p * lp + q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (A[q * lp + q] - A[p * lp + p]) / (2.0 * apq);
          const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = 1.0 / sqrt(1.0 + t * t);
          s = t * c;
        }
        pr[i][0] = p;
        pr[i][1] = q;
        cs[i][0] = c;
        cs[i][1] = s;
      }
      __syncthreads();
      // rows: A <- J^T A (a pair per warp, its columns over the lanes)
      for (int i = warp; i < h; i += nwarps) {
        const int p = pr[i][0], q = pr[i][1];
        const double c = cs[i][0], s = cs[i][1];
        for (int j = lane; j < l; j += 32) {
          const double ap = A[p * lp + j], aq = A[q * lp + j];
          A[p * lp + j] = c * ap - s * aq;
          A[q * lp + j] = s * ap + c * aq;
        }
      }
      __syncthreads();
      // columns: A <- A J, V <- V J
      for (int i = warp; i < h; i += nwarps) {
        const int p = pr[i][0], q = pr[i][1];
        const double c = cs[i][0], s = cs[i][1];
        for (int j = lane; j < l; j += 32) {
          const double ap = A[j * lp + p], aq = A[j * lp + q];
          A[j * lp + p] = c * ap - s * aq;
          A[j * lp + q] = s * ap + c * aq;
          const double vp = V[j * lp + p], vq = V[j * lp + q];
          V[j * lp + p] = c * vp - s * vq;
          V[j * lp + q] = s * vp + c * vq;
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    // the r largest eigenvalues, ties to the lower index
    for (int a = 0; a < l; ++a) taken[a] = 0;
    for (int i = 0; i < r; ++i) {
      int best = -1;
      for (int a = 0; a < l; ++a)
        if (!taken[a] && (best < 0 || A[a * lp + a] > A[best * lp + best])) best = a;
      taken[best] = 1;
      order[i] = best;
    }
  }
  __syncthreads();
  const double s0 = sqrt(fmax(A[order[0] * lp + order[0]], 0.0));
  for (int e = threadIdx.x; e < l * r; e += blockDim.x) {
    const int a = e / r, i = e % r;
    const double si = sqrt(fmax(A[order[i] * lp + order[i]], 0.0));
    const bool keep = s0 > 0.0 && si > 1e-12 * s0;
    const double hh = keep ? sqrt(si) : 0.0;
    const double v = V[a * lp + order[i]];
    M1[e] = keep ? v * hh : 0.0;
    M2[e] = keep ? v / hh : 0.0;
    if (sv && a == 0) sv[i] = si;
  }
}

}  // namespace

// ---- host side ------------------------------------------------------------------
namespace {

struct LqPlan {
  int64_t N, K;
  int r, l;
  int64_t rt_rows, rt_splits;      // row range per split and number of splits of R^T Y
  int64_t rm_cols, rm_splits;      // K range per split and number of splits of R M
  int64_t res_ctas;                // CTAs of the residual kernel (error parts)
  int64_t gram_parts_max;
  size_t E, qws, Ya, Yb, Za, Zb, Zpart, Bt, Gpart, G, T, M1, M2, sv, errpart, norm2, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// at most kGramMaxParts parts of a multiple of kGramRows rows each
void gram_split(int64_t rows, int64_t *parts, int64_t *per) {
  const int64_t q = ceil_div(ceil_div(rows, kGramMaxParts), kGramRows) * kGramRows;
  *per = q;
  *parts = ceil_div(rows, q);
}

LqPlan lq_plan(int64_t N, int64_t K, int r, int l, int dq) {
  LqPlan p{};
  p.N = N;
  p.K = K;
  p.r = r;
  p.l = l;
  // both products: one CTA per SM in one wave, splits of the reduction at least four steps deep
  const int64_t col_tiles = ceil_div(K, kTcRows);
  int64_t splits = std::max<int64_t>(1, std::min<int64_t>(148 / col_tiles, ceil_div(N, 4 * kTcRed)));
  p.rt_rows = ceil_div(ceil_div(N, splits), kTcRed) * kTcRed;
  p.rt_splits = ceil_div(N, p.rt_rows);
  const int64_t row_tiles = ceil_div(N, kTcRows);
  splits = std::max<int64_t>(1, std::min<int64_t>(148 / row_tiles, ceil_div(K, 4 * kTcRed)));
  p.rm_cols = ceil_div(ceil_div(K, splits), kTcRed) * kTcRed;
  p.rm_splits = ceil_div(K, p.rm_cols);
  p.res_ctas = ceil_div(K, kResCols) * ceil_div(N, kResRows);
  p.gram_parts_max = kGramMaxParts;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  p.E = take(4 * static_cast<size_t>(N * K));
  p.qws = take(dq == QLORA_DQ_SIGNED ? quantize_workspace_bytes(N * K) : 0);
  p.Ya = take(4 * static_cast<size_t>(N) * l);
  p.Yb = take(4 * static_cast<size_t>(N) * l);
  p.Za = take(4 * static_cast<size_t>(K) * l);
  p.Zb = take(4 * static_cast<size_t>(K) * l);
  p.Zpart = take(4 * std::max(static_cast<size_t>(p.rt_splits) * K, static_cast<size_t>(p.rm_splits) * N) * l);
  // the products' split small operand: hi and lo tiles of (l rounded up to 16) x 32 per 32-deep block
  p.Bt = take(4 * 2 * static_cast<size_t>(ceil_div(std::max(N, K), kTcRed)) * kTcRed * ceil_div(l, 16) * 16);
  p.Gpart = take(8 * static_cast<size_t>(p.gram_parts_max) * l * l);
  p.G = take(8 * static_cast<size_t>(l) * l);
  p.T = take(8 * static_cast<size_t>(l) * l);
  p.M1 = take(8 * static_cast<size_t>(l) * r);
  p.M2 = take(8 * static_cast<size_t>(l) * r);
  p.sv = take(8 * static_cast<size_t>(r));
  p.errpart = take(8 * static_cast<size_t>(p.res_ctas));
  p.norm2 = take(8);
  p.total = off;
  return p;
}

template <typename T>
T *wsp(void *ws, size_t off) {
  return reinterpret_cast<T *>(static_cast<char *>(ws) + off);
}

struct LqRun {
  const LqPlan &p;
  void *ws;
  const float *W;
  cudaStream_t st;
  cudaError_t err = cudaSuccess;

  void check() {
    if (err == cudaSuccess) err = cudaGetLastError();
  }

  // part[] = squared-error parts of W - W'(q) - L1 L2 (and E when given)
  void residual(const float *L1, const float *L2, const LqQuant &q, float *E, double *part) {
    const dim3 grid(static_cast<unsigned>(ceil_div(p.K, kResCols)), static_cast<unsigned>(ceil_div(p.N, kResRows)));
    prof_mark(kProfLqResidual, true, st);
    lq_residual_kernel<<<grid, kLqThreads, 0, st>>>(W, p.N, p.K, L1, L2, p.r, q, E, part);
    prof_mark(kProfLqResidual, false, st);
    check();
  }
  void sum(const double *part, int64_t n, const double *norm2, double *out) {
    lq_sum_kernel<<<1, kLqThreads, 0, st>>>(part, n, norm2, out);
    check();
  }
  // one tensor-core product launch: out-rows tiles x splits CTAs
  template <bool TRANS>
  void tc_product(const LqQuant &q, const float *B, int64_t red_per, int64_t splits, float *part) {
    const int nl = static_cast<int>(ceil_div(p.l, 16) * 16);
    const int smem = lq_tc_smem(nl);
    if (err == cudaSuccess) err = cudaFuncSetAttribute(lq_tc_kernel<TRANS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int *status = device_status_ptr();
    if (err == cudaSuccess && !status) err = cudaErrorInvalidValue;
    if (err != cudaSuccess) return;
    CUtensorMap tmW, tmC, tmB;
    // W [N, K] fp32: 32 x 128 (Y) or four 32 x 32 (Z) boxes, 128B-swizzled; codes [N, K/2] bytes:
    // 16 x 128 (Y) or 64 x 32 (Z) boxes; the small operand [reduction, l] fp32: l x 32 boxes
    bool ok = make_tmap_2d(&tmW, W, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.K, p.N, static_cast<uint64_t>(p.K) * 4, 32,
                           TRANS ? 32 : kTcRows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (q.codes)
      ok = ok && make_tmap_2d(&tmC, q.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, p.K / 2, p.N, static_cast<uint64_t>(p.K) / 2,
                              TRANS ? 64 : 16, TRANS ? 32 : kTcRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    else
      tmC = tmW;
    // the small operand, split into hi / lo tiles of nl x 32 per 32-deep block
    const int64_t red = TRANS ? p.N : p.K, nblk = ceil_div(red, kTcRed);
    if (nblk * nl * (kTcRed / 4) >= (int64_t(1) << 31)) ok = false;   // the split kernel indexes with 32 bits
    float *Bt = wsp<float>(ws, p.Bt);
    ok = ok && make_tmap_2d(&tmB, Bt, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, kTcRed, static_cast<uint64_t>(2 * nblk * nl),
                            kTcRed * 4, kTcRed, static_cast<uint32_t>(nl), CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) {
      err = cudaErrorInvalidValue;
      return;
    }
    const dim3 grid(static_cast<unsigned>(ceil_div(TRANS ? p.K : p.N, kTcRows)), static_cast<unsigned>(splits));
    prof_mark(kProfLqProduct, true, st);
    lq_tc_split_kernel<<<static_cast<unsigned>(ceil_div(nblk * nl * (kTcRed / 4), 256)), 256, 0, st>>>(
        B, red, p.l, nl, static_cast<int>(nblk), Bt);
    lq_tc_kernel<TRANS><<<grid, kTcThreads, smem, st>>>(tmW, tmC, tmB, p.N, p.K, q, p.l, nl, red_per, part, status,
                                                         wait_limit());
    prof_mark(kProfLqProduct, false, st);
    check();
  }
  void rmul(const LqQuant &q, const float *M, float *Y) {
    float *part = wsp<float>(ws, p.Zpart);
    tc_product<false>(q, M, p.rm_cols, p.rm_splits, part);
    sum_splits(part, static_cast<int>(p.rm_splits), p.N * p.l, Y);
  }
  void sum_splits(const float *part, int ns, int64_t n, float *out) {
    prof_mark(kProfLqSmall, true, st);
    lq_sum_splits_kernel<<<static_cast<unsigned>(std::min<int64_t>(ceil_div(n, 256), 148 * 8)), 256, 0, st>>>(
        part, ns, n, out);
    prof_mark(kProfLqSmall, false, st);
    check();
  }
  void rtmul(const LqQuant &q, const float *Y, float *Z) {
    float *part = wsp<float>(ws, p.Zpart);
    tc_product<true>(q, Y, p.rt_rows, p.rt_splits, part);
    sum_splits(part, static_cast<int>(p.rt_splits), p.K * p.l, Z);
  }
  // G = X^T X (fp64, l x l) of X [rows, l]
  void gram(const float *X, int64_t rows) {
    int64_t parts, per;
    gram_split(rows, &parts, &per);
    prof_mark(kProfLqSmall, true, st);
    const dim3 grid(kGramGroups, static_cast<unsigned>(parts));
    lq_gram_kernel<<<grid, kLqThreads, 0, st>>>(X, rows, p.l, per, wsp<double>(ws, p.Gpart));
    const int ll = p.l * p.l;
    lq_gram_sum_kernel<<<static_cast<unsigned>(ceil_div(ll, 256)), 256, 0, st>>>(
        wsp<double>(ws, p.Gpart), static_cast<int>(parts), ll, wsp<double>(ws, p.G));
    prof_mark(kProfLqSmall, false, st);
    check();
  }
  void small_gemm(const float *X, int64_t rows, const double *S, int cols, float *out, bool transposed) {
    const size_t smem = 8 * static_cast<size_t>(p.l) * cols + 4 * static_cast<size_t>(kSgRows) * p.l;
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(lq_small_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
    if (err != cudaSuccess) return;
    prof_mark(kProfLqSmall, true, st);
    lq_small_gemm_kernel<<<static_cast<unsigned>(ceil_div(rows, kSgRows)), kLqThreads, smem, st>>>(
        X, rows, p.l, S, cols, out, transposed ? 1 : 0);
    prof_mark(kProfLqSmall, false, st);
    check();
  }
  // the columns of *X [rows, l] made orthonormal by Cholesky QR, `passes`
  // times (the span is unchanged; a second pass restores orthogonality to
  // working precision).  The result lands in *X or *tmp; the pointers are
  // swapped so that *X names it.
  void orth(float **X, float **tmp, int64_t rows, int passes) {
    const size_t smem = 16 * static_cast<size_t>(p.l) * lq_pitch(p.l);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(lq_chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
    for (int pass = 0; pass < passes; ++pass) {
      gram(*X, rows);
      if (err != cudaSuccess) return;
      prof_mark(kProfLqChol, true, st);
      lq_chol_inv_kernel<<<1, kLqThreads, smem, st>>>(wsp<double>(ws, p.G), p.l, wsp<double>(ws, p.T));
      prof_mark(kProfLqChol, false, st);
      check();
      small_gemm(*X, rows, wsp<double>(ws, p.T), p.l, *tmp, false);
      std::swap(*X, *tmp);
    }
  }
  // L1 L2 = rank-r approximation of R (randomized subspace iteration)
  void rsvd(const LqQuant &q, const float *Omega, int power, float *L1, float *L2) {
    float *Ya = wsp<float>(ws, p.Ya), *Yb = wsp<float>(ws, p.Yb);
    float *Za = wsp<float>(ws, p.Za), *Zb = wsp<float>(ws, p.Zb);
    // one Cholesky QR pass between power rounds, two for the basis B is formed from
    rmul(q, Omega, Ya);
    orth(&Ya, &Yb, p.N, power == 0 ? 2 : 1);
    for (int i = 0; i < power; ++i) {
      rtmul(q, Ya, Za);
      orth(&Za, &Zb, p.K, 1);
      rmul(q, Za, Ya);
      orth(&Ya, &Yb, p.N, i + 1 == power ? 2 : 1);
    }
    rtmul(q, Ya, Za);   // B^T = R^T Q
    gram(Za, p.K);
    const size_t smem = 16 * static_cast<size_t>(p.l) * lq_pitch(p.l);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(lq_jacobi_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
    if (err != cudaSuccess) return;
    prof_mark(kProfLqJacobi, true, st);
    lq_jacobi_kernel<<<1, kLqThreads, smem, st>>>(wsp<double>(ws, p.G), p.l, p.r, wsp<double>(ws, p.M1),
                                                  wsp<double>(ws, p.M2), wsp<double>(ws, p.sv));
    prof_mark(kProfLqJacobi, false, st);
    check();
    small_gemm(Ya, p.N, wsp<double>(ws, p.M1), p.r, L1, false);
    small_gemm(Za, p.K, wsp<double>(ws, p.M2), p.r, L2, true);
  }
};

}  // namespace

}  // namespace qlora

using namespace qlora;

#define LQ_TRY(expr)                          \
  do {                                        \
    const qlora_status lq_st_ = (expr);       \
    if (lq_st_ != QLORA_OK) return lq_st_;    \
  } while (0)

namespace {

// Shared argument checks; fills the plan.  l = 0 means "no rank-r step" (the
// residual quantizer alone), checked as l = r.
qlora_status lq_args(const float *W, int64_t N, int64_t K, int r, int l, int dq, void *ws, size_t ws_bytes,
                     LqPlan *plan) {
  if (!W || N < 1 || K < 1) return QLORA_ERR_INVALID_ARG;
  const int lc = l == 0 ? r : l;
  // l a multiple of 4: the test matrix's rows are 16-byte runs for the products' tensor maps
  if (r < 1 || lc < r || lc > kLqMaxL || (l != 0 && (l & 3))) return QLORA_ERR_INVALID_ARG;
  if (N < lc || K < lc) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (l != 0 && K % kBlock != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;   // the products walk whole blocks
  if (dq == QLORA_DQ_SIGNED && N * K >= (int64_t(1) << 38)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  *plan = lq_plan(N, K, r, lc, dq);
  if (!ws || ws_bytes < plan->total) return QLORA_ERR_WORKSPACE;
  if (!aligned16(ws)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

}  // namespace

extern "C" {

size_t qlora_lq_workspace_bytes(int64_t rows, int64_t cols, int r, int l, int dq) {
  const int lc = l == 0 ? r : l;
  if (rows < 1 || cols < 1 || r < 1 || lc < r || lc > kLqMaxL || (dq != QLORA_DQ_PLAIN && dq != QLORA_DQ_SIGNED))
    return 0;
  return lq_plan(rows, cols, r, lc, dq).total;
}

qlora_status qlora_lq_quantize_residual(const float *W, const float *L1, const float *L2, int r,
                                        const qlora_nf4_weight *Q, void *ws, size_t ws_bytes, void *stream) {
  if (!Q || !L1 || !L2) return QLORA_ERR_INVALID_ARG;
  LQ_TRY(validate_weight(Q));
  LqPlan p;
  LQ_TRY(lq_args(W, Q->rows, Q->cols, r, 0, Q->dq, ws, ws_bytes, &p));
  if (!aligned16(L1) || !aligned16(L2)) return QLORA_ERR_MISALIGNED;
  int *status = device_status_ptr();
  if (!status) return QLORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LqRun run{p, ws, W, st};
  const Nf4Table tab = weight_table(Q);
  float *E = wsp<float>(ws, p.E);
  run.residual(L1, L2, LqQuant{nullptr, nullptr, nullptr, tab}, E, nullptr);
  if (run.err == cudaSuccess)
    run.err = launch_quantize(E, QLORA_DTYPE_F32, p.N * p.K, Q->codes, Q->absmax_q, Q->group_scale, tab,
                              Q->dq == QLORA_DQ_SIGNED ? wsp<void>(ws, p.qws) : nullptr, status, st);
  return run.err == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_lq_lowrank(const float *W, int64_t rows, int64_t cols, const qlora_nf4_weight *Q,
                              const float *Omega, int l, int power, int r, float *L1, float *L2, void *ws,
                              size_t ws_bytes, void *stream) {
  if (!Omega || !L1 || !L2 || power < 0 || power > 16) return QLORA_ERR_INVALID_ARG;
  if (l < 1) return QLORA_ERR_INVALID_ARG;
  if (Q) {
    LQ_TRY(validate_weight(Q));
    if (Q->rows != rows || Q->cols != cols) return QLORA_ERR_INVALID_ARG;
  }
  LqPlan p;
  LQ_TRY(lq_args(W, rows, cols, r, l, Q ? Q->dq : QLORA_DQ_PLAIN, ws, ws_bytes, &p));
  if (!aligned16(Omega) || !aligned16(L1) || !aligned16(L2)) return QLORA_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LqRun run{p, ws, W, st};
  const Nf4Table tab = Q ? weight_table(Q) : format_table(QLORA_FORMAT_NF4);
  const LqQuant q = Q ? LqQuant{Q->codes, Q->absmax_q, Q->group_scale, tab} : LqQuant{nullptr, nullptr, nullptr, tab};
  run.rsvd(q, Omega, power, L1, L2);
  return run.err == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

qlora_status qlora_lq_decompose(const float *W, const qlora_nf4_weight *Q, float *L1, float *L2, int r,
                                const float *Omega, int l, int power, int iters, double *err, void *ws,
                                size_t ws_bytes, void *stream) {
  if (!Q || !L1 || !L2 || !Omega || !err || l < 1) return QLORA_ERR_INVALID_ARG;
  if (power < 0 || power > 16 || iters < 1 || iters > 1000) return QLORA_ERR_INVALID_ARG;
  LQ_TRY(validate_weight(Q));
  LqPlan p;
  LQ_TRY(lq_args(W, Q->rows, Q->cols, r, l, Q->dq, ws, ws_bytes, &p));
  if (!aligned16(L1) || !aligned16(L2) || !aligned16(Omega) || !aligned16(err)) return QLORA_ERR_MISALIGNED;
  int *status = device_status_ptr();
  if (!status) return QLORA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  LqRun run{p, ws, W, st};
  const Nf4Table tab = weight_table(Q);
  const LqQuant none{nullptr, nullptr, nullptr, tab};
  const LqQuant quant{Q->codes, Q->absmax_q, Q->group_scale, tab};
  double *part = wsp<double>(ws, p.errpart);
  double *norm2 = wsp<double>(ws, p.norm2);
  float *E = wsp<float>(ws, p.E);

  run.residual(nullptr, nullptr, none, nullptr, part);   // ||W||^2
  run.sum(part, p.res_ctas, nullptr, norm2);
  run.rsvd(none, Omega, power, L1, L2);                   // principal rank-r part of W
  for (int t = 0; t < iters && run.err == cudaSuccess; ++t) {
    run.residual(L1, L2, none, E, nullptr);               // E = W - L1 L2
    if (run.err == cudaSuccess)
      run.err = launch_quantize(E, QLORA_DTYPE_F32, p.N * p.K, Q->codes, Q->absmax_q, Q->group_scale, tab,
                                Q->dq == QLORA_DQ_SIGNED ? wsp<void>(ws, p.qws) : nullptr, status, st);
    run.residual(L1, L2, quant, nullptr, part);           // before the rank-r step
    run.sum(part, p.res_ctas, norm2, err + 2 * t);
    run.rsvd(quant, Omega, power, L1, L2);
    run.residual(L1, L2, quant, nullptr, part);           // after it
    run.sum(part, p.res_ctas, norm2, err + 2 * t + 1);
  }
  return run.err == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // extern "C"
