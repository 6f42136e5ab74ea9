// Low-rank adapter products: the tall-skinny contractions around the fused
// dequant-GEMM.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": small trainable low-rank matrices next to the frozen base; only the
// adapters receive gradients.  With X [M,K], dY [M,N], A [r,K], B [N,r]:
//   H  = X A^T          (forward prologue; reduction over K)
//   G  = s dY B         (reduction over N)
//   dB = s dY^T H       (reduction over the M tokens)
//   dA = G^T X          (reduction over the M tokens)
// Each is C[i,j] = sum_k opA(i,k) opB(j,k) on bf16 tensor cores (mma.sync
// m16n8k16, fp32 accumulate) over 64x64 tiles, split over the reduction into
// fp32 partials that a second kernel sums in a fixed order (deterministic).
// fp32 operands (H, G) enter as a bf16 hi/lo pair: x = hi + lo with
// hi = bf16(x), lo = bf16(x - hi), i.e. two stacked operands, which keeps
// about 16 significant bits.
#include "internal.h"

namespace qlora {

namespace {

constexpr int TI = 64, TJ = 64, TK = 32;
constexpr int SK_THREADS = 128;
constexpr int PAD = 8;   // bf16 elements of padding per smem row

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
  const int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory tile of one operand: K-major -> [TI rows][TK + PAD], MN-major -> [TK rows][TI + PAD].
template <bool KMAJ>
struct TileGeom {
  static constexpr int ROW = KMAJ ? (TK + PAD) : (TI + PAD);
  static constexpr int ROWS = KMAJ ? TI : TK;
  static constexpr int ELEMS = ROW * ROWS;
};

// Copy one 64 x 32 (i x k) operand tile into shared memory with 16-byte cp.async,
// zero-filling rows / chunks outside [0, I) x [k0, kend).
template <bool KMAJ>
__device__ __forceinline__ void load_tile(uint16_t *sdst, const uint16_t *src, int64_t ld, int64_t i0, int64_t I,
                                          int64_t k0, int64_t kend) {
  const int t = threadIdx.x;
#pragma unroll
  for (int q0 = 0; q0 < 2; ++q0) {
    const int q = q0 * SK_THREADS + t;   // 256 chunks of 8 elements
    int64_t gi, gk;
    int srow, scol;
    if (KMAJ) {
      srow = q >> 2;
      scol = (q & 3) * 8;
      gi = i0 + srow;
      gk = k0 + scol;
    } else {
      srow = q >> 3;
      scol = (q & 7) * 8;
      gk = k0 + srow;
      gi = i0 + scol;
    }
    const bool valid = gi < I && gk < kend;
    const uint16_t *g = valid ? (KMAJ ? src + gi * ld + gk : src + gk * ld + gi) : src;
    cp_async16(smem_addr(sdst + srow * TileGeom<KMAJ>::ROW + scol), g, valid);
  }
}

template <bool AK, bool BK_>
__global__ void __launch_bounds__(SK_THREADS) skinny_kernel(const uint16_t *__restrict__ A, int64_t lda,
                                                            const uint16_t *__restrict__ B, int64_t ldb, int64_t I,
                                                            int64_t J, int64_t Kred, int64_t kps,
                                                            float *__restrict__ part) {
  __shared__ __align__(128) uint16_t sA[2][TileGeom<AK>::ELEMS];
  __shared__ __align__(128) uint16_t sB[2][TileGeom<BK_>::ELEMS];
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * TI;
  const int64_t j0 = static_cast<int64_t>(blockIdx.y) * TJ;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.z) * kps;
  const int64_t kend = (kbeg + kps < Kred) ? kbeg + kps : Kred;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wi = (warp >> 1) * 32, wj = (warp & 1) * 32;

  float acc[2][4][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.0f;

  const int nk = kend > kbeg ? static_cast<int>((kend - kbeg + TK - 1) / TK) : 0;
  if (nk > 0) {
    load_tile<AK>(sA[0], A, lda, i0, I, kbeg, kend);
    load_tile<BK_>(sB[0], B, ldb, j0, J, kbeg, kend);
  }
  cp_async_commit();
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) {
      load_tile<AK>(sA[cur ^ 1], A, lda, i0, I, kbeg + (kt + 1) * TK, kend);
      load_tile<BK_>(sB[cur ^ 1], B, ldb, j0, J, kbeg + (kt + 1) * TK, kend);
    }
    cp_async_commit();
    cp_async_wait_1();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; kk += 16) {
      uint32_t af[2][4], bf[4][2];
#pragma unroll
      for (int mi = 0; mi < 2; ++mi) {
        const int ib = wi + mi * 16;
        if (AK) {
          const int row = ib + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = kk + (lane >> 4) * 8;
          ldsm_x4(smem_addr(&sA[cur][row * TileGeom<AK>::ROW + col]), af[mi][0], af[mi][1], af[mi][2], af[mi][3]);
        } else {
          const int krow = kk + (lane & 7) + (lane >> 4) * 8;
          const int col = ib + ((lane >> 3) & 1) * 8;
          ldsm_x4_t(smem_addr(&sA[cur][krow * TileGeom<AK>::ROW + col]), af[mi][0], af[mi][1], af[mi][2],
                    af[mi][3]);
        }
      }
#pragma unroll
      for (int nj = 0; nj < 2; ++nj) {
        const int jb = wj + nj * 16;
        uint32_t r0, r1, r2, r3;
        if (BK_) {
          const int row = jb + (lane & 7) + (lane >> 4) * 8;
          const int col = kk + ((lane >> 3) & 1) * 8;
          ldsm_x4(smem_addr(&sB[cur][row * TileGeom<BK_>::ROW + col]), r0, r1, r2, r3);
        } else {
          const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = jb + (lane >> 4) * 8;
          ldsm_x4_t(smem_addr(&sB[cur][krow * TileGeom<BK_>::ROW + col]), r0, r1, r2, r3);
        }
        bf[2 * nj][0] = r0;
        bf[2 * nj][1] = r1;
        bf[2 * nj + 1][0] = r2;
        bf[2 * nj + 1][1] = r3;
      }
#pragma unroll
      for (int mi = 0; mi < 2; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) mma_bf16_16816(acc[mi][ni], af[mi], bf[ni][0], bf[ni][1]);
    }
    __syncthreads();
  }
  cp_async_wait_0();

  float *out = part + static_cast<int64_t>(blockIdx.z) * I * J;
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int64_t gi = i0 + wi + mi * 16 + (lane >> 2);
      const int64_t gj = j0 + wj + ni * 8 + (lane & 3) * 2;
      if (gj < J) {
        if (gi < I) *reinterpret_cast<float2 *>(out + gi * J + gj) = make_float2(acc[mi][ni][0], acc[mi][ni][1]);
        if (gi + 8 < I)
          *reinterpret_cast<float2 *>(out + (gi + 8) * J + gj) = make_float2(acc[mi][ni][2], acc[mi][ni][3]);
      }
    }
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float bf16_val(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }

__global__ void finalize_h_kernel(const float *__restrict__ part, int splits, int64_t M, int r, float s,
                                  float *__restrict__ H, uint16_t *__restrict__ sH, uint16_t *__restrict__ Hs) {
  const int64_t n = M * r;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float h = part[e];
    for (int z = 1; z < splits; ++z) h = __fadd_rn(h, part[static_cast<int64_t>(z) * n + e]);
    H[e] = h;
    sH[e] = bf16_bits(__fmul_rn(s, h));
    if (Hs) {
      const int64_t m = e / r, j = e % r;
      const uint16_t hi = bf16_bits(h);
      Hs[m * 2 * r + j] = hi;
      Hs[m * 2 * r + r + j] = bf16_bits(__fsub_rn(h, bf16_val(hi)));
    }
  }
}

__global__ void split_hilo_kernel(const float *__restrict__ H, int64_t M, int r, uint16_t *__restrict__ Hs) {
  const int64_t n = M * r;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float h = H[e];
    const int64_t m = e / r, j = e % r;
    const uint16_t hi = bf16_bits(h);
    Hs[m * 2 * r + j] = hi;
    Hs[m * 2 * r + r + j] = bf16_bits(__fsub_rn(h, bf16_val(hi)));
  }
}

__global__ void finalize_g_kernel(const float *__restrict__ part, int splits, int64_t M, int r, float s,
                                  uint16_t *__restrict__ Gb, uint16_t *__restrict__ Gs) {
  const int64_t n = M * r;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float g = part[e];
    for (int z = 1; z < splits; ++z) g = __fadd_rn(g, part[static_cast<int64_t>(z) * n + e]);
    g = __fmul_rn(s, g);
    const uint16_t hi = bf16_bits(g);
    Gb[e] = hi;
    const int64_t m = e / r, j = e % r;
    Gs[m * 2 * r + j] = hi;
    Gs[m * 2 * r + r + j] = bf16_bits(__fsub_rn(g, bf16_val(hi)));
  }
}

// part is [splits][I][2*half]; out[i][j] = scale * sum_z (part[z][i][j] + part[z][i][half + j]).
__global__ void finalize_cols_kernel(const float *__restrict__ part, int splits, int64_t I, int64_t half, float scale,
                                     float *__restrict__ out) {
  const int64_t n = I * half;
  const int64_t zs = I * 2 * half;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / half, j = e % half;
    const int64_t b = i * 2 * half + j;
    float v = __fadd_rn(part[b], part[b + half]);
    for (int z = 1; z < splits; ++z) v = __fadd_rn(v, __fadd_rn(part[z * zs + b], part[z * zs + b + half]));
    out[e] = __fmul_rn(scale, v);
  }
}

// part is [splits][2*half][J]; out[i][j] = sum_z (part[z][i][j] + part[z][half + i][j]).
__global__ void finalize_rows_kernel(const float *__restrict__ part, int splits, int64_t half, int64_t J,
                                     float *__restrict__ out) {
  const int64_t n = half * J;
  const int64_t zs = 2 * half * J;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = __fadd_rn(part[e], part[e + n]);
    for (int z = 1; z < splits; ++z) v = __fadd_rn(v, __fadd_rn(part[z * zs + e], part[z * zs + e + n]));
    out[e] = v;
  }
}

unsigned ew_blocks(int64_t n) {
  int64_t b = (n + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  if (b < 1) b = 1;
  return static_cast<unsigned>(b);
}

}  // namespace

void skinny_plan(int64_t I, int64_t J, int64_t Kred, int *splits, int64_t *k_per_split) {
  int64_t tiles = ceil_div(I, TI) * ceil_div(J, TJ);
  if (tiles < 1) tiles = 1;
  if (Kred < 1) Kred = 1;
  int64_t sp = ceil_div(2 * 148, tiles);
  const int64_t max_sp = Kred / (4 * TK) > 0 ? Kred / (4 * TK) : 1;
  if (sp > max_sp) sp = max_sp;
  if (sp > 64) sp = 64;
  if (sp < 1) sp = 1;
  int64_t kps = ceil_div(ceil_div(Kred, sp), TK) * TK;
  sp = ceil_div(Kred, kps);
  *splits = static_cast<int>(sp);
  *k_per_split = kps;
}

cudaError_t launch_skinny(const SkinnyArgs &a, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(ceil_div(a.I, TI)), static_cast<unsigned>(ceil_div(a.J, TJ)),
                  static_cast<unsigned>(a.splits));
  prof_mark(kProfLora, true, st);
  if (a.a_kmajor && a.b_kmajor)
    skinny_kernel<true, true><<<grid, SK_THREADS, 0, st>>>(a.A, a.lda, a.B, a.ldb, a.I, a.J, a.Kred, a.k_per_split,
                                                           a.part);
  else if (a.a_kmajor && !a.b_kmajor)
    skinny_kernel<true, false><<<grid, SK_THREADS, 0, st>>>(a.A, a.lda, a.B, a.ldb, a.I, a.J, a.Kred, a.k_per_split,
                                                            a.part);
  else if (!a.a_kmajor && a.b_kmajor)
    skinny_kernel<false, true><<<grid, SK_THREADS, 0, st>>>(a.A, a.lda, a.B, a.ldb, a.I, a.J, a.Kred, a.k_per_split,
                                                            a.part);
  else
    skinny_kernel<false, false><<<grid, SK_THREADS, 0, st>>>(a.A, a.lda, a.B, a.ldb, a.I, a.J, a.Kred,
                                                             a.k_per_split, a.part);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

cudaError_t launch_finalize_h(const float *part, int splits, int64_t M, int r, float s, float *H, uint16_t *sH,
                              uint16_t *Hs, cudaStream_t st) {
  prof_mark(kProfLora, true, st);
  finalize_h_kernel<<<ew_blocks(M * r), 256, 0, st>>>(part, splits, M, r, s, H, sH, Hs);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

cudaError_t launch_split_hilo(const float *H, int64_t M, int r, uint16_t *Hs, cudaStream_t st) {
  prof_mark(kProfLora, true, st);
  split_hilo_kernel<<<ew_blocks(M * r), 256, 0, st>>>(H, M, r, Hs);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

cudaError_t launch_finalize_g(const float *part, int splits, int64_t M, int r, float s, uint16_t *Gb, uint16_t *Gs,
                              cudaStream_t st) {
  prof_mark(kProfLora, true, st);
  finalize_g_kernel<<<ew_blocks(M * r), 256, 0, st>>>(part, splits, M, r, s, Gb, Gs);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

cudaError_t launch_finalize_cols(const float *part, int splits, int64_t I, int64_t half, float scale, float *out,
                                 cudaStream_t st) {
  prof_mark(kProfLora, true, st);
  finalize_cols_kernel<<<ew_blocks(I * half), 256, 0, st>>>(part, splits, I, half, scale, out);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

cudaError_t launch_finalize_rows(const float *part, int splits, int64_t half, int64_t J, float *out,
                                 cudaStream_t st) {
  prof_mark(kProfLora, true, st);
  finalize_rows_kernel<<<ew_blocks(half * J), 256, 0, st>>>(part, splits, half, J, out);
  prof_mark(kProfLora, false, st);
  return cudaGetLastError();
}

}  // namespace qlora
