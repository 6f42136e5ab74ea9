// Few-token forward (M <= 16): memory-bound dequant-GEMV.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": the 4-bit base is dequantized on the fly to 16-bit for each pass.
// With a handful of tokens the packed weight stream (0.516 B per weight) is the
// whole cost, so the weight is decoded straight into tensor-core register
// fragments and never touches shared memory.
//
//   kernel 1  H = X A^T (fp32 [M, r]); one warp per adapter row.
//   kernel 2  per CTA: 64 weight rows x one 1024-wide K chunk.  mma.sync
//             m16n8k16 with the weight as the 16-row A operand and the tokens
//             as the 8-column B operand (two column tiles for M > 8).  Each
//             thread owns one whole 64-weight block of two rows, builds that
//             block's 16-entry bf16 table once and decodes its codes with
//             byte permutes.  Within a 256-wide macro-step the K index of the
//             fragment slots is permuted so that thread (g, c) covers block c
//             (the same bijection is applied to the tokens).  fp32 partial
//             sums per K chunk go to the workspace.
//   kernel 3  Y = bf16(sum over chunks + (s H) B^T), chunks summed in order.
#include "decode.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int GV_ROWS = 64;          // weight rows per CTA (4 warps x 16)
constexpr int GV_KC = 1024;          // K chunk per CTA
constexpr int GV_THREADS = 128;
constexpr int GV_MACRO = 256;        // K per macro-step (4 blocks)
constexpr int GV_TOK = 16;           // token capacity

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// H[m][j] = sum_k X[m][k] A[j][k]; one warp per j, all M tokens at once.
__global__ void __launch_bounds__(256) gemv_h_kernel(const uint16_t *__restrict__ X, const uint16_t *__restrict__ A,
                                                     int M, int K, int r, float *__restrict__ H) {
  const int j = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= r) return;
  float acc[GV_TOK];
#pragma unroll
  for (int m = 0; m < GV_TOK; ++m) acc[m] = 0.0f;
  for (int k = lane * 8; k < K; k += 256) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(A + static_cast<int64_t>(j) * K + k));
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int m = 0; m < GV_TOK; ++m) {
      if (m < M) {
        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(m) * K + k));
        const uint32_t xv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[m] = fmaf(__uint_as_float(xv[e] << 16), __uint_as_float(av[e] << 16), acc[m]);
          acc[m] = fmaf(__uint_as_float(xv[e] & 0xFFFF0000u), __uint_as_float(av[e] & 0xFFFF0000u), acc[m]);
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < GV_TOK; ++m) {
    float v = acc[m];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0 && m < M) H[static_cast<int64_t>(m) * r + j] = v;
  }
}

template <int NT>   // number of 8-token column tiles (1: M <= 8, 2: M <= 16)
__global__ void __launch_bounds__(GV_THREADS) gemv_main_kernel(const uint16_t *__restrict__ X, int M, int64_t N,
                                                               int64_t K, const uint8_t *__restrict__ codes,
                                                               const uint8_t *__restrict__ absmax_q,
                                                               const float *__restrict__ group_scale,
                                                               float *__restrict__ part, Nf4Table tab) {
  // X chunk, permuted: word (8 B = 4 tokens-values of one token) at
  // [macro][s][c][tok], so that the 32 lanes of a step read 32 distinct words.
  __shared__ __align__(16) uint2 xs[GV_KC / GV_MACRO][16][4][NT * 8];
  const int64_t n_base = static_cast<int64_t>(blockIdx.x) * GV_ROWS;
  const int64_t k_base = static_cast<int64_t>(blockIdx.y) * GV_KC;
  const int64_t kc = (K - k_base) < GV_KC ? (K - k_base) : GV_KC;   // multiple of 64
  const int nmacro = static_cast<int>((kc + GV_MACRO - 1) / GV_MACRO);

  // Stage X[0:M, k_base : k_base+kc] (zero for tokens >= M or k past the chunk).
  for (int w = threadIdx.x; w < (GV_KC / 4) * NT * 8; w += GV_THREADS) {
    const int tok = w % (NT * 8);
    const int kq = w / (NT * 8);              // which 4-element group of the chunk
    const int k = kq * 4;
    const int ms = k / GV_MACRO, in = k % GV_MACRO;
    const int c = in / 64, s = (in % 64) / 4;
    uint2 v = make_uint2(0, 0);
    if (tok < M && k < kc) v = __ldg(reinterpret_cast<const uint2 *>(X + static_cast<int64_t>(tok) * K + k_base + k));
    xs[ms][s][c][tok] = v;
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t row0 = n_base + warp * 16 + g;       // rows row0 and row0 + 8
  const int64_t kblocks = K / kBlock;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;

  for (int ms = 0; ms < nmacro; ++ms) {
    const int64_t kb = (k_base + static_cast<int64_t>(ms) * GV_MACRO) / kBlock + c;
    const bool kvalid = (static_cast<int64_t>(ms) * GV_MACRO + 64 * c) < kc;
    uint4 cw[2][2];
    float ap[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t n = row0 + 8 * h;
      ap[h] = 0.0f;
      cw[h][0] = cw[h][1] = make_uint4(0, 0, 0, 0);
      if (n < N && kvalid) {
        const int64_t bi = n * kblocks + kb;
        const uint4 *src = reinterpret_cast<const uint4 *>(codes + bi * 32);
        cw[h][0] = __ldcs(src);
        cw[h][1] = __ldcs(src + 1);
        ap[h] = __fmul_rn(static_cast<float>(__ldg(absmax_q + bi)), __ldg(group_scale + (bi >> 8)));
      }
    }
    uint32_t LO[2][4], HI[2][4];
    nf4_block_table(ap[0], tab, LO[0], HI[0]);
    nf4_block_table(ap[1], tab, LO[1], HI[1]);
    const uint32_t words[2][8] = {{cw[0][0].x, cw[0][0].y, cw[0][0].z, cw[0][0].w, cw[0][1].x, cw[0][1].y,
                                   cw[0][1].z, cw[0][1].w},
                                  {cw[1][0].x, cw[1][0].y, cw[1][0].z, cw[1][0].w, cw[1][1].x, cw[1][1].y,
                                   cw[1][1].z, cw[1][1].w}};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t o0[4], o1[4];
      nf4_lut8(words[0][w], LO[0], HI[0], o0);
      nf4_lut8(words[1][w], LO[1], HI[1], o1);
#pragma unroll
      for (int hs = 0; hs < 2; ++hs) {
        const int s = 2 * w + hs;                      // k16 step: in-block offsets 4s .. 4s+3
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint2 xv = xs[ms][s][c][t * 8 + g];
          mma16816(acc[t], o0[2 * hs], o1[2 * hs], o0[2 * hs + 1], o1[2 * hs + 1], xv.x, xv.y);
        }
      }
    }
  }

  // partial[chunk][n][ldp], ldp = M rounded up to even (only live tokens are written)
  const int ldp = (M + 1) & ~1;
  float *out = part + static_cast<int64_t>(blockIdx.y) * N * ldp;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tok = t * 8 + 2 * c;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t n = row0 + 8 * h;
      if (n < N && tok < M) *reinterpret_cast<float2 *>(out + n * ldp + tok) = make_float2(acc[t][2 * h], acc[t][2 * h + 1]);
    }
  }
}

// Y[m][n] = bf16( sum_z part[z][n][m] + sum_j fl32(s*H[m][j]) B[n][j] ).
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float *__restrict__ part, int nchunks, int M,
                                                          int64_t N, const float *__restrict__ H,
                                                          const uint16_t *__restrict__ B, int r, float s,
                                                          uint16_t *__restrict__ Y) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * M) return;
  const int64_t n = idx / M;
  const int m = static_cast<int>(idx % M);
  const int ldp = (M + 1) & ~1;
  float v = 0.0f;
  for (int z = 0; z < nchunks; ++z) v += part[(static_cast<int64_t>(z) * N + n) * ldp + m];
  float l = 0.0f;
  for (int j = 0; j < r; ++j)
    l = fmaf(__fmul_rn(s, H[static_cast<int64_t>(m) * r + j]),
             __uint_as_float(static_cast<uint32_t>(B[n * r + j]) << 16), l);
  const __nv_bfloat16 b = __float2bfloat16_rn(v + l);
  Y[static_cast<int64_t>(m) * N + n] = *reinterpret_cast<const uint16_t *>(&b);
}

}  // namespace

bool gemv_enabled() { return true; }

size_t gemv_partial_bytes(int64_t M, int64_t N, int64_t K) {
  return static_cast<size_t>(ceil_div(K, GV_KC) * N * ((M + 1) & ~int64_t(1))) * 4;
}

qlora_status launch_gemv(const GemvArgs &a, cudaStream_t st) {
  if (a.M < 1 || a.M > kGemvMaxTokens) return QLORA_ERR_UNSUPPORTED_SHAPE;
  float *H = a.H_out ? a.H_out : a.h_ws;
  const int64_t nchunks = ceil_div(a.wK, GV_KC);
  prof_mark(kProfGemv, true, st);
  gemv_h_kernel<<<static_cast<unsigned>(ceil_div(a.r, 8)), 256, 0, st>>>(a.X, a.A, static_cast<int>(a.M),
                                                                         static_cast<int>(a.wK), a.r, H);
  prof_mark(kProfGemv, false, st);
  const dim3 grid(static_cast<unsigned>(ceil_div(a.wN, GV_ROWS)), static_cast<unsigned>(nchunks));
  prof_mark(kProfGemv, true, st);
  if (a.M <= 8)
    gemv_main_kernel<1><<<grid, GV_THREADS, 0, st>>>(a.X, static_cast<int>(a.M), a.wN, a.wK, a.codes, a.absmax_q,
                                                     a.group_scale, a.part, nf4_table());
  else
    gemv_main_kernel<2><<<grid, GV_THREADS, 0, st>>>(a.X, static_cast<int>(a.M), a.wN, a.wK, a.codes, a.absmax_q,
                                                     a.group_scale, a.part, nf4_table());
  prof_mark(kProfGemv, false, st);
  prof_mark(kProfGemv, true, st);
  gemv_reduce_kernel<<<static_cast<unsigned>(ceil_div(a.wN * a.M, 256)), 256, 0, st>>>(
      a.part, static_cast<int>(nchunks), static_cast<int>(a.M), a.wN, H, a.B, a.r, a.s, a.Y);
  prof_mark(kProfGemv, false, st);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
