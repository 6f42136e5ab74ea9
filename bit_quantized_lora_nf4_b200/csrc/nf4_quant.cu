// Blockwise NF4 quantizer with double quantization, and the standalone
// dequantizer to bf16.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "NormalFloat, double
// quantization, paged optimizers": 16 levels at normal quantiles, one scaling
// constant per block of weights, the constants themselves stored in 8 bits
// under a coarser set of constants.  Section "Where the memory goes": the base
// is quantized once up front and dequantized to 16-bit for every pass.
//
// Arithmetic contract (IEEE fp32 round-to-nearest, no FMA contraction, no
// flush-to-zero; this file is compiled with -fmad=false):
//   a_b = max |w| over the 64-element block (exact)
//   n   = fl32(w / a_b)            (0 when a_b == 0)
//   code = #{ i : n > thresh[i] }  == nearest level, ties to the lower index
//   c_g = max a_b over 256 blocks;  S_g = fl32(c_g / 255)
//   q_b = min(255, rint(fl32(a_b / S_g)))  (0 when S_g == 0)
//   W'  = bf16(fl32(level[code] * fl32(q_b * S_g)))
#include "internal.h"

namespace qlora {

namespace {

constexpr int kQuantThreads = 256;                       // one thread per block of the group
constexpr int kGroupElems = kBlock * kGroup;             // 16384

// Nearest-level code by binary search over the 15 ascending thresholds held in
// shared memory: the result is the number of thresholds strictly below n.
__device__ __forceinline__ uint32_t encode_nf4(float n, const float *thr) {
  uint32_t c = (n > thr[7]) ? 8u : 0u;
  c += (n > thr[c + 3]) ? 4u : 0u;
  c += (n > thr[c + 1]) ? 2u : 0u;
  c += (n > thr[c]) ? 1u : 0u;
  return c;
}

__device__ __forceinline__ float block_norm(float w, float a) { return a != 0.0f ? __fdiv_rn(w, a) : 0.0f; }

__device__ __forceinline__ bool finite4(float4 v) {
  return isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
}

// One CTA per group of 256 blocks (16384 weights).  Full, aligned groups take
// the vectorised path: each half-warp streams one block per iteration with
// 16-byte loads, reduces its absmax with shuffles and writes 8 bytes of codes
// per half-warp row.  A partial final group takes the per-block scalar path.
__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const float *__restrict__ W, int64_t numel,
                                                                     uint8_t *__restrict__ codes,
                                                                     uint8_t *__restrict__ absmax_q,
                                                                     float *__restrict__ group_scale, Nf4Table tab,
                                                                     int *status) {
  __shared__ float s_thr[16];
  __shared__ float s_abs[kGroup];
  __shared__ float s_wmax[kQuantThreads / 32];
  const int t = threadIdx.x;
  if (t < 15) s_thr[t] = tab.thresh[t];
  __syncthreads();

  const int64_t g = blockIdx.x;
  const int64_t base = g * kGroupElems;
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  bool bad = false;

  if (base + kGroupElems <= numel && (reinterpret_cast<uintptr_t>(W) & 15u) == 0) {
    const float4 *W4 = reinterpret_cast<const float4 *>(W + base);
    uint16_t *C2 = reinterpret_cast<uint16_t *>(codes + base / 2);
    float4 v[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) v[it] = __ldcs(W4 + it * kQuantThreads + t);
#pragma unroll
    for (int it = 0; it < 16; ++it) {
      const float4 x = v[it];
      bad |= !finite4(x);
      float m = fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w)));
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if ((t & 15) == 0) s_abs[it * 16 + (t >> 4)] = m;
      const uint32_t c0 = encode_nf4(block_norm(x.x, m), s_thr);
      const uint32_t c1 = encode_nf4(block_norm(x.y, m), s_thr);
      const uint32_t c2 = encode_nf4(block_norm(x.z, m), s_thr);
      const uint32_t c3 = encode_nf4(block_norm(x.w, m), s_thr);
      C2[it * kQuantThreads + t] = static_cast<uint16_t>(c0 | (c1 << 4) | (c2 << 8) | (c3 << 12));
    }
  } else {
    const int64_t blk = g * kGroup + t;
    float a = 0.0f;
    if (blk < nblocks) {
      const int64_t e0 = blk * kBlock;
      const int64_t e1 = (e0 + kBlock < numel) ? e0 + kBlock : numel;
      for (int64_t e = e0; e < e1; ++e) {
        const float w = W[e];
        bad |= !isfinite(w);
        a = fmaxf(a, fabsf(w));
      }
      for (int64_t e = e0; e < e1; e += 2) {
        const uint32_t lo = encode_nf4(block_norm(W[e], a), s_thr);
        const uint32_t hi = (e + 1 < e1) ? encode_nf4(block_norm(W[e + 1], a), s_thr) : 0u;
        codes[e / 2] = static_cast<uint8_t>(lo | (hi << 4));
      }
    }
    s_abs[t] = a;
  }
  __syncthreads();

  // Double quantization of this group's 256 block constants.
  const float a = s_abs[t];
  float m = a;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((t & 31) == 0) s_wmax[t >> 5] = m;
  __syncthreads();
  float c = s_wmax[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) c = fmaxf(c, s_wmax[w]);
  const float S = __fdiv_rn(c, 255.0f);
  const int64_t blk = g * kGroup + t;
  if (blk < nblocks) {
    uint32_t q = 0;
    if (S != 0.0f) q = static_cast<uint32_t>(fminf(rintf(__fdiv_rn(a, S)), 255.0f));
    absmax_q[blk] = static_cast<uint8_t>(q);
  }
  if (t == 0) group_scale[g] = S;
  if (bad) latch_status(status, QLORA_ERR_NONFINITE);
}

// Each thread turns one 32-bit word of codes (8 weights) into one 16-byte bf16
// chunk.  Levels come from a 16-entry shared-memory copy (conflict-free: at
// most 16 distinct words, one per bank).
constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads) nf4_dequantize_kernel(const uint8_t *__restrict__ codes,
                                                                     const uint8_t *__restrict__ absmax_q,
                                                                     const float *__restrict__ group_scale,
                                                                     int64_t numel, uint16_t *__restrict__ out,
                                                                     Nf4Table tab) {
  __shared__ float s_lv[16];
  if (threadIdx.x < 16) s_lv[threadIdx.x] = tab.level[threadIdx.x];
  __syncthreads();
  const int64_t nchunk = (numel + 7) / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunk; i += stride) {
    const int64_t e0 = i * 8;
    const int64_t blk = e0 >> 6;
    const float ap = __fmul_rn(static_cast<float>(__ldg(absmax_q + blk)), __ldg(group_scale + (blk >> 8)));
    if (e0 + 8 <= numel) {
      const uint32_t w = __ldcs(reinterpret_cast<const unsigned int *>(codes) + i);
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = __fmul_rn(s_lv[(w >> (8 * j)) & 15u], ap);
        const float hi = __fmul_rn(s_lv[(w >> (8 * j + 4)) & 15u], ap);
        o[j] = pack_bf16x2(lo, hi);
      }
      __stcs(reinterpret_cast<uint4 *>(out + e0), make_uint4(o[0], o[1], o[2], o[3]));
    } else {
      for (int64_t e = e0; e < numel; ++e) {
        const uint32_t c = (codes[e >> 1] >> (4 * (e & 1))) & 15u;
        const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(s_lv[c], ap));
        out[e] = *reinterpret_cast<const uint16_t *>(&b);
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const float *W, int64_t numel, uint8_t *codes, uint8_t *absmax_q, float *group_scale,
                            int *status, cudaStream_t st) {
  const int64_t ngroups = (numel + kGroupElems - 1) / kGroupElems;
  prof_mark(kProfQuant, true, st);
  nf4_quantize_kernel<<<static_cast<unsigned>(ngroups), kQuantThreads, 0, st>>>(W, numel, codes, absmax_q,
                                                                                 group_scale, nf4_table(), status);
  prof_mark(kProfQuant, false, st);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale, int64_t numel,
                              uint16_t *out, cudaStream_t st) {
  const int64_t nchunk = (numel + 7) / 8;
  int64_t blocks = (nchunk + kDeqThreads - 1) / kDeqThreads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  prof_mark(kProfDequant, true, st);
  nf4_dequantize_kernel<<<static_cast<unsigned>(blocks), kDeqThreads, 0, st>>>(codes, absmax_q, group_scale, numel,
                                                                               out, nf4_table());
  prof_mark(kProfDequant, false, st);
  return cudaGetLastError();
}

}  // namespace qlora
