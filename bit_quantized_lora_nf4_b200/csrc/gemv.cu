// Few-token forward (M <= 16): memory-bound dequant-GEMV.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": every pass expands the 4-bit base to 16-bit as it runs.
// With a handful of tokens the packed weight stream (0.516 B per weight) is the
// whole cost, so the weight is decoded straight into tensor-core register
// fragments and never touches shared memory.
//
//   kernel 1  per CTA: 64 weight rows x one 1024-wide K chunk.  mma.sync
//             m16n8k16 with the weight as the 16-row A operand and the tokens
//             as the 8-column B operand (two column tiles for M > 8).  Each
//             thread owns one whole 64-weight block of two rows, builds that
//             block's 16-entry bf16 table once and decodes its codes with
//             byte permutes.  Within a 256-wide macro-step the K index of the
//             fragment slots is permuted so that thread (g, c) covers block c
//             (the same bijection is applied to the tokens).  fp32 partial
//             sums per K chunk go to the workspace.  The same CTAs also form
//             the adapter prologue's partial sums H_z = X_z A^T over their K
//             chunk (adapter rows spread over the CTAs of a chunk).
//   kernel 2  per CTA of 64 output rows: s*H = s * sum_z H_z into shared
//             memory, then Y = bf16(sum_z Y_z + (s H) B^T); all sums in a
//             fixed order (deterministic).
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

template <int NT>   // number of 8-token column tiles (1: M <= 8, 2: M <= 16)
__global__ void __launch_bounds__(GV_THREADS) gemv_main_kernel(const uint16_t *__restrict__ X, int M, int64_t N,
                                                               int64_t K, const uint8_t *__restrict__ codes,
                                                               const uint8_t *__restrict__ absmax_q,
                                                               const float *__restrict__ group_scale,
                                                               const uint16_t *__restrict__ A, int r,
                                                               float *__restrict__ part, float *__restrict__ hpart,
                                                               Nf4Table tab) {
  // X chunk, permuted: the 8-byte word holding X[tok][k .. k+3] for in-chunk
  // k = 256 ms + 64 c + 4 s sits at xs[ms][s][tok][c], so the 32 lanes of one
  // k16 step (token g, block c) read 32 consecutive words: no bank conflicts.
  __shared__ __align__(16) uint2 xs[GV_KC / GV_MACRO][16][NT * 8][4];
  const int64_t n_base = static_cast<int64_t>(blockIdx.x) * GV_ROWS;
  const int64_t k_base = static_cast<int64_t>(blockIdx.y) * GV_KC;
  const int64_t kc = (K - k_base) < GV_KC ? (K - k_base) : GV_KC;   // multiple of 64
  const int nmacro = static_cast<int>((kc + GV_MACRO - 1) / GV_MACRO);

  // Stage X[0:M, k_base : k_base+kc] with 16-byte loads (8 elements = two words);
  // zero for tokens >= M or k past the chunk.
  for (int w = threadIdx.x; w < (GV_KC / 8) * NT * 8; w += GV_THREADS) {
    const int tok = w % (NT * 8);
    const int k = (w / (NT * 8)) * 8;
    const int ms = k / GV_MACRO, in = k % GV_MACRO;
    const int c = in / 64, s = (in % 64) / 4;           // s is even
    uint4 v = make_uint4(0, 0, 0, 0);
    if (tok < M && k < kc) v = __ldg(reinterpret_cast<const uint4 *>(X + static_cast<int64_t>(tok) * K + k_base + k));
    xs[ms][s][tok][c] = make_uint2(v.x, v.y);
    xs[ms][s + 1][tok][c] = make_uint2(v.z, v.w);
  }
  __syncthreads();

  // Adapter prologue partials for this K chunk: hpart[z][m][j] = sum_k X[m][k] A[j][k]
  // for the adapter rows j = blockIdx.x, blockIdx.x + gridDim.x, ...  Thread t
  // covers k = 8t .. 8t+7 of the chunk for every token (one 16-byte load of A),
  // then the 128 partial sums per token are reduced in a fixed order (warp
  // shuffles, then the 4 warps through shared memory).
  {
    __shared__ float hred[GV_THREADS / 32][GV_TOK];
    const int k = threadIdx.x * 8;
    const int ms = k / GV_MACRO, in = k % GV_MACRO;
    const int c8 = in / 64, s8 = (in % 64) / 4;
    for (int j = blockIdx.x; j < r; j += gridDim.x) {
      uint4 av = make_uint4(0, 0, 0, 0);
      if (k < kc) av = __ldg(reinterpret_cast<const uint4 *>(A + static_cast<int64_t>(j) * K + k_base + k));
      const uint32_t a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
      for (int tok = 0; tok < NT * 8; ++tok) {
        float h = 0.0f;
        if (tok < M) {
          const uint2 x0 = xs[ms][s8][tok][c8], x1 = xs[ms][s8 + 1][tok][c8];
          const uint32_t x4[4] = {x0.x, x0.y, x1.x, x1.y};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            h = fmaf(__uint_as_float(x4[e] << 16), __uint_as_float(a4[e] << 16), h);
            h = fmaf(__uint_as_float(x4[e] & 0xFFFF0000u), __uint_as_float(a4[e] & 0xFFFF0000u), h);
          }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) h += __shfl_xor_sync(0xffffffffu, h, off);
        if ((threadIdx.x & 31) == 0) hred[threadIdx.x >> 5][tok] = h;
      }
      __syncthreads();
      if (threadIdx.x < M) {
        float v = 0.0f;
#pragma unroll
        for (int wq = 0; wq < GV_THREADS / 32; ++wq) v += hred[wq][threadIdx.x];
        hpart[(static_cast<int64_t>(blockIdx.y) * M + threadIdx.x) * r + j] = v;
      }
      __syncthreads();
    }
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int64_t row0 = n_base + warp * 16 + g;       // rows row0 and row0 + 8
  const int64_t kblocks = K / kBlock;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;

  // codes / constants of one macro-step for rows row0 and row0 + 8 (zero when out of range)
  auto fetch = [&](int ms, uint4 (&cw)[2][2], float (&ap)[2]) {
    const int64_t kb = (k_base + static_cast<int64_t>(ms) * GV_MACRO) / kBlock + c;
    const bool kvalid = ms < nmacro && (static_cast<int64_t>(ms) * GV_MACRO + 64 * c) < kc;
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
  };
  uint4 cw[2][2], cn[2][2];
  float ap[2], an[2];
  fetch(0, cw, ap);
  for (int ms = 0; ms < nmacro; ++ms) {
    fetch(ms + 1, cn, an);                 // next macro-step's loads in flight while this one decodes
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
          const uint2 xv = xs[ms][s][t * 8 + g][c];
          mma16816(acc[t], o0[2 * hs], o1[2 * hs], o0[2 * hs + 1], o1[2 * hs + 1], xv.x, xv.y);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      cw[h][0] = cn[h][0];
      cw[h][1] = cn[h][1];
      ap[h] = an[h];
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

constexpr int GV_RED_ROWS = 32;      // output rows per reduce CTA (8 warps x 4 rows)

// Per CTA of 32 output rows: sH[m][j] = fl32(s * sum_z hpart[z][m][j]) into
// shared memory (the CTA with blockIdx.x == 0 also writes the unscaled H when
// asked).  Then 8 lanes per output row n: lane l takes the adapter columns
// 8c .. 8c+7 for c = l, l+8, ... (16-byte loads of B), the 8 partial dot
// products are combined with xor shuffles, and lane l finishes tokens l and
// l+8: Y[m][n] = bf16( sum_z part[z][n][m] + sum_j sH[m][j] B[n][j] ).
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float *__restrict__ part,
                                                          const float *__restrict__ hpart, int nchunks, int M,
                                                          int64_t N, const uint16_t *__restrict__ B, int r, float s,
                                                          float *__restrict__ H_out, uint16_t *__restrict__ Y) {
  __shared__ float sh[GV_TOK * 256];
  for (int e = threadIdx.x; e < M * r; e += blockDim.x) {
    float h = 0.0f;
#pragma unroll 4
    for (int z = 0; z < nchunks; ++z) h += hpart[static_cast<int64_t>(z) * M * r + e];
    sh[e] = __fmul_rn(s, h);
    if (H_out && blockIdx.x == 0) H_out[e] = h;
  }
  __syncthreads();
  const int ldp = (M + 1) & ~1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int l8 = lane & 7;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * GV_RED_ROWS + warp * 4 + (lane >> 3);
  const bool live = n < N;
  float acc[GV_TOK];
#pragma unroll
  for (int m = 0; m < GV_TOK; ++m) acc[m] = 0.0f;
  if (live) {
    for (int c = l8; c < r / 8; c += 8) {
      const uint4 bv = __ldg(reinterpret_cast<const uint4 *>(B + n * r + 8 * c));
      const uint32_t b4[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int m = 0; m < GV_TOK; ++m) {
        if (m < M) {
          const float *shm = sh + m * r + 8 * c;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[m] = fmaf(shm[2 * e], __uint_as_float(b4[e] << 16), acc[m]);
            acc[m] = fmaf(shm[2 * e + 1], __uint_as_float(b4[e] & 0xFFFF0000u), acc[m]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < GV_TOK; ++m) {
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
  }
  if (live) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = l8 + 8 * h;
      if (m < M) {
        float v = 0.0f;
        for (int z = 0; z < nchunks; ++z) v += part[(static_cast<int64_t>(z) * N + n) * ldp + m];
        float lora = acc[0];
#pragma unroll
        for (int mm = 1; mm < GV_TOK; ++mm)
          if (mm == m) lora = acc[mm];
        const __nv_bfloat16 b = __float2bfloat16_rn(v + lora);
        Y[static_cast<int64_t>(m) * N + n] = *reinterpret_cast<const uint16_t *>(&b);
      }
    }
  }
}

}  // namespace

bool gemv_enabled() { return true; }

size_t gemv_partial_bytes(int64_t M, int64_t N, int64_t K) {
  return static_cast<size_t>(ceil_div(K, GV_KC) * N * ((M + 1) & ~int64_t(1))) * 4;
}

size_t gemv_hpartial_bytes(int64_t M, int64_t K, int r) {
  return static_cast<size_t>(ceil_div(K, GV_KC) * M * r) * 4;
}

qlora_status launch_gemv(const GemvArgs &a, cudaStream_t st) {
  if (a.M < 1 || a.M > kGemvMaxTokens) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t nchunks = ceil_div(a.wK, GV_KC);
  const dim3 grid(static_cast<unsigned>(ceil_div(a.wN, GV_ROWS)), static_cast<unsigned>(nchunks));
  prof_mark(kProfGemv, true, st);
  if (a.M <= 8)
    gemv_main_kernel<1><<<grid, GV_THREADS, 0, st>>>(a.X, static_cast<int>(a.M), a.wN, a.wK, a.codes, a.absmax_q,
                                                     a.group_scale, a.A, a.r, a.part, a.hpart, nf4_table());
  else
    gemv_main_kernel<2><<<grid, GV_THREADS, 0, st>>>(a.X, static_cast<int>(a.M), a.wN, a.wK, a.codes, a.absmax_q,
                                                     a.group_scale, a.A, a.r, a.part, a.hpart, nf4_table());
  prof_mark(kProfGemv, false, st);
  prof_mark(kProfGemv, true, st);
  gemv_reduce_kernel<<<static_cast<unsigned>(ceil_div(a.wN, GV_RED_ROWS)), 256, 0, st>>>(
      a.part, a.hpart, static_cast<int>(nchunks), static_cast<int>(a.M), a.wN, a.B, a.r, a.s, a.H_out, a.Y);
  prof_mark(kProfGemv, false, st);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
