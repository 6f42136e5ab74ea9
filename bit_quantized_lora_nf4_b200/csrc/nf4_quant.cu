// Blockwise NF4 quantizer with double quantization, and the standalone
// dequantizer to bf16.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "NormalFloat, double
// quantization, paged optimizers": 16 levels at normal quantiles, one scaling
// constant per block of weights, the constants themselves stored in 8 bits
// under one more, coarser level of constants.  Section "Where the memory
// goes": the frozen base is quantized a single time before training and
// expanded to 16-bit in every pass.
//
// Arithmetic contract (IEEE fp32 round-to-nearest, no FMA contraction, no
// flush-to-zero; this file is compiled with -fmad=false), w the weight as fp32
// (a bf16 weight widened exactly):
//   a_b = max |w| over the 64-element block (exact)
//   n   = fl32(w / a_b)            (0 when a_b == 0)
//   code = #{ i : n > thresh[i] }  == nearest level, ties to the lower index
//   plain block constants (QLORA_DQ_PLAIN):
//     c_g = max a_b over 256 blocks;  S_g = fl32(c_g / 255)
//     q_b = min(255, rint(fl32(a_b / S_g)))  (0 when S_g == 0);  a'_b = fl32(q_b * S_g)
//   signed block constants around their mean (QLORA_DQ_SIGNED):
//     mu  = fl32(fl64(fl64(exact sum of all a_b) / n_blocks))
//     c_b = fl32(a_b - mu);  S_g = fl32(max |c_b| / 127)
//     q_b = clamp(rint(fl32(c_b / S_g)), -127, 127)  (0 when S_g == 0), stored as int8
//     a'_b = fl32(fl32(q_b * S_g) + mu)
//   W'  = bf16(fl32(level[code] * a'_b))
//
// The signed constants take three launches: the quantizer writes the codes,
// the fp32 a_b and an exact, order-free sum of the a_b (integer digits added
// with 64-bit atomics); a second kernel turns the sum into mu and codes every
// group's constants against it.
#include <atomic>

#include "decode.cuh"
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

// ---- exact sum of non-negative fp32 values ------------------------------------
// Every finite fp32 value is an integer number of 2^-149 units; a value with
// biased exponent E and significand m (hidden bit included) is m << max(E - 1, 0)
// units, below 2^278.  The sum of fewer than 2^32 of them is below 2^310 and is
// kept as kSumDigits base-2^32 digits, each held in a 64-bit word that absorbs
// unnormalised additions (carries are propagated once, when the sum is read).
constexpr int kSumDigits = 10;

// Adds this warp's 32 values to the digit words `acc` (shared memory): per
// digit the 32 contributions are summed as two 16-bit halves with warp
// reductions, then one lane adds the total.
__device__ __forceinline__ void warp_exact_add(float a, unsigned long long *acc) {
  const uint32_t u = __float_as_uint(a);
  const uint32_t E = u >> 23;
  const uint32_t m = (u & 0x7FFFFFu) | (E ? 0x800000u : 0u);
  const uint32_t shift = E ? E - 1 : 0;
  const uint32_t d = shift >> 5;
  const unsigned long long x = static_cast<unsigned long long>(m) << (shift & 31);   // < 2^55
  const uint32_t lo = static_cast<uint32_t>(x), hi = static_cast<uint32_t>(x >> 32);
  const uint32_t dmin = __reduce_min_sync(0xffffffffu, d);
  const uint32_t dmax = __reduce_max_sync(0xffffffffu, d) + 1;
  for (uint32_t k = dmin; k <= dmax; ++k) {
    const uint32_t c = k == d ? lo : (k == d + 1 ? hi : 0u);
    const unsigned long long sum = __reduce_add_sync(0xffffffffu, c & 0xFFFFu) +
                                   (static_cast<unsigned long long>(__reduce_add_sync(0xffffffffu, c >> 16)) << 16);
    if ((threadIdx.x & 31) == 0 && sum != 0) atomicAdd(acc + k, sum);
  }
}

// 2^k as a double, -1022 <= k <= 1023.
__device__ __forceinline__ double pow2d(int k) { return __longlong_as_double(static_cast<long long>(k + 1023) << 52); }

// fl32(fl64(fl64(S) / n)) for the exact sum S held in the digit words (one thread).
__device__ float exact_mean(const unsigned long long *acc, int64_t n) {
  uint32_t dig[kSumDigits + 2];
  unsigned long long carry = 0;
  for (int i = 0; i < kSumDigits; ++i) {
    const unsigned long long v = acc[i] + carry;
    dig[i] = static_cast<uint32_t>(v);
    carry = v >> 32;
  }
  dig[kSumDigits] = static_cast<uint32_t>(carry);
  dig[kSumDigits + 1] = 0;
  int top = kSumDigits;
  while (top > 0 && dig[top] == 0) --top;
  if (dig[top] == 0 || n <= 0) return 0.0f;
  const int p = 32 * top + 31 - __clz(dig[top]);                  // highest set bit
  unsigned long long w;
  int lowbit = 0;
  if (p < 64) {
    w = (static_cast<unsigned long long>(dig[1]) << 32) | dig[0];
  } else {
    // the 64 bits p-63 .. p; anything set below them is folded into bit 0, which
    // lies under the rounding position of a 53-bit significand (a sticky bit)
    lowbit = p - 63;
    const int i0 = lowbit >> 5, off = lowbit & 31;
    const unsigned long long lo64 = (static_cast<unsigned long long>(dig[i0 + 1]) << 32) | dig[i0];
    w = off ? (lo64 >> off) | (static_cast<unsigned long long>(dig[i0 + 2]) << (64 - off)) : lo64;
    bool sticky = off && (dig[i0] & ((1u << off) - 1u)) != 0;
    for (int j = 0; j < i0; ++j) sticky |= dig[j] != 0;
    if (sticky) w |= 1ull;
  }
  const double s = __dmul_rn(__ull2double_rn(w), pow2d(lowbit - 149));   // exact scaling
  return __double2float_rn(__ddiv_rn(s, static_cast<double>(n)));
}

// Weights arrive as fp32 or bf16; a bf16 weight is widened to fp32 (exact) and
// every later step is the fp32 arithmetic above.
__device__ __forceinline__ float load_weight(const float *W, int64_t e) { return W[e]; }
__device__ __forceinline__ float load_weight(const uint16_t *W, int64_t e) {
  return __uint_as_float(static_cast<uint32_t>(W[e]) << 16);
}
// Four consecutive weights starting at a 4-element boundary (16 or 8 bytes), streamed once.
__device__ __forceinline__ float4 load_weight4(const float *W, int64_t i4) {
  return __ldcs(reinterpret_cast<const float4 *>(W) + i4);
}
__device__ __forceinline__ float4 load_weight4(const uint16_t *W, int64_t i4) {
  const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(W) + i4);
  return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u), __uint_as_float(v.y << 16),
                     __uint_as_float(v.y & 0xFFFF0000u));
}

// One CTA per group of 256 blocks (16384 weights).  Full, aligned groups take
// the vectorised path: each half-warp streams one block per iteration with
// 16-byte (fp32) or 8-byte (bf16) loads, reduces its absmax with shuffles and
// writes 8 bytes of codes per half-warp row.  A partial final group takes the
// per-block scalar path.
template <typename TW>
__global__ void __launch_bounds__(kQuantThreads) nf4_quantize_kernel(const TW *__restrict__ W, int64_t numel,
                                                                     uint8_t *__restrict__ codes,
                                                                     uint8_t *__restrict__ absmax_q,
                                                                     float *__restrict__ group_scale, Nf4Table tab,
                                                                     float *__restrict__ dq_abs,
                                                                     unsigned long long *__restrict__ dq_acc,
                                                                     int *status) {
  __shared__ float s_thr[16];
  __shared__ float s_abs[kGroup];
  __shared__ float s_wmax[kQuantThreads / 32];
  __shared__ unsigned long long s_acc[kSumDigits];
  const int t = threadIdx.x;
  if (t < 15) s_thr[t] = tab.thresh[t];
  if (t < kSumDigits) s_acc[t] = 0;
  __syncthreads();

  const int64_t g = blockIdx.x;
  const int64_t base = g * kGroupElems;
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  const int64_t code_bytes = (numel + 1) / 2, ngroups = (nblocks + kGroup - 1) / kGroup;
  (void)code_bytes;
  (void)ngroups;
  bool bad = false;

  if (base + kGroupElems <= numel && (reinterpret_cast<uintptr_t>(W) & 15u) == 0) {
    uint16_t *C2 = reinterpret_cast<uint16_t *>(codes + base / 2);
    float4 v[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) v[it] = load_weight4(W, base / 4 + it * kQuantThreads + t);
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
      if (QL_IN_BOUNDS(status, base / 2 + 2 * (it * kQuantThreads + t) + 1, code_bytes))
        C2[it * kQuantThreads + t] = static_cast<uint16_t>(c0 | (c1 << 4) | (c2 << 8) | (c3 << 12));
    }
  } else {
    const int64_t blk = g * kGroup + t;
    float a = 0.0f;
    if (blk < nblocks) {
      const int64_t e0 = blk * kBlock;
      const int64_t e1 = (e0 + kBlock < numel) ? e0 + kBlock : numel;
      for (int64_t e = e0; e < e1; ++e) {
        const float w = load_weight(W, e);
        bad |= !isfinite(w);
        a = fmaxf(a, fabsf(w));
      }
      for (int64_t e = e0; e < e1; e += 2) {
        const uint32_t lo = encode_nf4(block_norm(load_weight(W, e), a), s_thr);
        const uint32_t hi = (e + 1 < e1) ? encode_nf4(block_norm(load_weight(W, e + 1), a), s_thr) : 0u;
        if (QL_IN_BOUNDS(status, e / 2, code_bytes)) codes[e / 2] = static_cast<uint8_t>(lo | (hi << 4));
      }
    }
    s_abs[t] = a;
  }
  __syncthreads();

  if (dq_abs != nullptr) {
    // Signed constants: keep a_b for the second pass and add it to the exact sum.
    const float a = s_abs[t];
    const int64_t blk = g * kGroup + t;
    if (blk < nblocks && QL_IN_BOUNDS(status, blk, nblocks)) dq_abs[blk] = a;
    warp_exact_add(a, s_acc);
    __syncthreads();
    if (t < kSumDigits && s_acc[t] != 0) atomicAdd(dq_acc + t, s_acc[t]);
    if (bad) latch_status(status, QLORA_ERR_NONFINITE);
    return;
  }

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
    if (QL_IN_BOUNDS(status, blk, nblocks)) absmax_q[blk] = static_cast<uint8_t>(q);
  }
  if (t == 0 && QL_IN_BOUNDS(status, g, ngroups)) group_scale[g] = S;
  if (bad) latch_status(status, QLORA_ERR_NONFINITE);
}

// Signed block constants of one group (one thread per block) against the
// tensor-wide mean; every CTA derives mu from the exact sum itself.
__global__ void __launch_bounds__(kQuantThreads) nf4_dq_signed_kernel(const float *__restrict__ dq_abs,
                                                                      const unsigned long long *__restrict__ dq_acc,
                                                                      int64_t nblocks, uint8_t *__restrict__ absmax_q,
                                                                      float *__restrict__ group_scale,
                                                                      float *__restrict__ mu_out, int *status) {
  __shared__ float s_mu;
  __shared__ float s_wmax[kQuantThreads / 32];
  const int t = threadIdx.x;
  const int64_t g = blockIdx.x;
  if (t == 0) s_mu = exact_mean(dq_acc, nblocks);
  __syncthreads();
  const float mu = s_mu;
  const int64_t blk = g * kGroup + t;
  const float c = blk < nblocks ? __fsub_rn(__ldg(dq_abs + blk), mu) : 0.0f;
  float m = fabsf(c);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((t & 31) == 0) s_wmax[t >> 5] = m;
  __syncthreads();
  float cm = s_wmax[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) cm = fmaxf(cm, s_wmax[w]);
  const float S = __fdiv_rn(cm, 127.0f);
  if (blk < nblocks) {
    int q = 0;
    if (S != 0.0f) q = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(c, S)), -127.0f), 127.0f));
    if (QL_IN_BOUNDS(status, blk, nblocks)) absmax_q[blk] = static_cast<uint8_t>(q & 0xFF);
  }
  if (t == 0 && QL_IN_BOUNDS(status, g, (nblocks + kGroup - 1) / kGroup)) group_scale[g] = S;
  (void)status;
  if (g == 0 && t == 0) *mu_out = mu;
}

// Each thread turns 16 bytes of codes (32 weights, half of one block) into
// 64 bytes of bf16 through the block's byte-permute table (decode.cuh), so a
// warp streams 512 B in and 2 KB out per iteration.
constexpr int kDeqThreads = 256;

__global__ void __launch_bounds__(kDeqThreads) nf4_dequantize_kernel(const uint8_t *__restrict__ codes,
                                                                     const uint8_t *__restrict__ absmax_q,
                                                                     const float *__restrict__ group_scale,
                                                                     int64_t numel, uint16_t *__restrict__ out,
                                                                     Nf4Table tab, int *status) {
  (void)status;
  const int64_t nchunk = (numel + 31) / 32;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float mu = dq_offset(tab);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nchunk; i += stride) {
    const int64_t e0 = i * 32;
    const int64_t blk = e0 >> 6;
    const float ap = block_constant(__ldg(absmax_q + blk), __ldg(group_scale + (blk >> 8)), tab.qx, mu);
    uint32_t LO[4], HI[4];
    nf4_block_table(ap, tab, LO, HI);
    if (e0 + 32 <= numel) {
      const uint4 c = __ldcs(reinterpret_cast<const uint4 *>(codes) + i);
      const uint32_t words[4] = {c.x, c.y, c.z, c.w};
      uint4 *dst = reinterpret_cast<uint4 *>(out + e0);
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t o[4];
        nf4_lut8(words[w], LO, HI, o);
        if (QL_IN_BOUNDS(status, e0 + 8 * w + 7, numel)) __stcs(dst + w, make_uint4(o[0], o[1], o[2], o[3]));
      }
    } else {
      for (int64_t e = e0; e < numel; ++e) {
        const uint32_t cd = (codes[e >> 1] >> (4 * (e & 1))) & 15u;
        uint32_t o[4];
        nf4_lut8(cd, LO, HI, o);                 // code in nibble 0 -> T[cd] in the low half of o[0]
        if (QL_IN_BOUNDS(status, e, numel)) out[e] = static_cast<uint16_t>(o[0] & 0xFFFFu);
      }
    }
  }
}

// SMs of the current device, looked up once per device (148 when no device
// answers: sizing only).
int device_sm_count_cached() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  int v = cache[dev].load();
  if (v <= 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      return 148;
    }
    cache[dev].store(v);
  }
  return v;
}

// Persistent dequantizer for whole chunks of 8192 weights (128 blocks): the
// 4 KB of codes and the chunk's 128 block constants arrive by 1-D bulk copies
// into a ring of kDqStages stages issued kDqStages - 1 chunks ahead, 256
// threads decode 32 weights each into a 16 KB shared buffer, and one thread
// streams it out with a bulk store (two output buffers).
constexpr int kDqChunk = 8192;
constexpr int kDqCodeBytes = kDqChunk / 2;
constexpr int kDqConstBytes = kDqChunk / kBlock;                 // 128 u8 block constants
constexpr int kDqStageBytes = kDqCodeBytes + kDqConstBytes;
constexpr int kDqOutBytes = kDqChunk * 2;
#ifndef QLORA_DQ_STAGES
#define QLORA_DQ_STAGES 4
#endif
#ifndef QLORA_DQ_CTAS_PER_SM
#define QLORA_DQ_CTAS_PER_SM 4
#endif
constexpr int kDqStages = QLORA_DQ_STAGES;
constexpr int kDqSmem = kDqStages * kDqStageBytes + 2 * kDqOutBytes + kDqStages * 8 + 16;

__global__ void __launch_bounds__(kDeqThreads) nf4_dequantize_bulk_kernel(const uint8_t *__restrict__ codes,
                                                                          const uint8_t *__restrict__ absmax_q,
                                                                          const float *__restrict__ group_scale,
                                                                          int64_t nchunks, uint16_t *__restrict__ out,
                                                                          int64_t out_elems, Nf4Table tab, int *status,
                                                                          uint64_t wait_limit) {
  (void)out_elems;
  extern __shared__ __align__(128) uint8_t dq_smem[];
  uint8_t *cbuf = dq_smem;                                         // [kDqStages][kDqStageBytes]
  uint8_t *obuf = dq_smem + kDqStages * kDqStageBytes;             // [2][kDqOutBytes]
  uint64_t *bar = reinterpret_cast<uint64_t *>(obuf + 2 * kDqOutBytes);
  int *abort_flag = reinterpret_cast<int *>(bar + kDqStages);
  const int t = threadIdx.x;
  const int64_t first = blockIdx.x;
  const int64_t step = gridDim.x;
  int issued = 0;   // chunks whose load thread 0 has issued
  // The next kernel on the stream may be scheduled now (its launch overlaps this
  // one's tail); no global memory is touched before the previous kernel's
  // writes are visible.
  griddep_launch_dependents();
  griddep_wait();
  auto issue = [&](int j) {   // the load of this CTA's chunk number j into stage j % kDqStages
    const int64_t ch = first + j * step;
    uint8_t *dst = cbuf + (j % kDqStages) * kDqStageBytes;
    mbar_arrive_expect_tx(&bar[j % kDqStages], kDqStageBytes);
    bulk_load(dst, codes + ch * kDqCodeBytes, kDqCodeBytes, &bar[j % kDqStages]);
    bulk_load(dst + kDqCodeBytes, absmax_q + ch * kDqConstBytes, kDqConstBytes, &bar[j % kDqStages]);
  };
  if (t == 0) {
    for (int i = 0; i < kDqStages; ++i) mbar_init(&bar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (; issued < kDqStages && first + issued * step < nchunks; ++issued) issue(issued);
  }
  __syncthreads();
  int it = 0;
  const float mu = dq_offset(tab);
  float S = first < nchunks ? __ldg(group_scale + (first >> 1)) : 0.0f;   // one group per two chunks
  for (int64_t ch = first; ch < nchunks; ch += step, ++it) {
    const int ls = it % kDqStages, ob = it & 1;
    const float S_next = ch + step < nchunks ? __ldg(group_scale + ((ch + step) >> 1)) : 0.0f;
    // obuf[ob] was last used by the store issued two iterations ago
    if (t == 0) bulk_wait_read<1>();
    const bool ok = mbar_wait(&bar[ls], (it / kDqStages) & 1, wait_limit);
    if (!ok) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag) break;
    const uint8_t *stage = cbuf + ls * kDqStageBytes;
    const float ap = block_constant(stage[kDqCodeBytes + (t >> 1)], S, tab.qx, mu);
    uint32_t LO[4], HI[4];
    nf4_block_table(ap, tab, LO, HI);
    const uint4 cw = ld_shared_v4(smem_addr(stage + t * 16));
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t o[4];
      nf4_lut8(words[w], LO, HI, o);
      st_shared_v4(smem_addr(obuf + ob * kDqOutBytes + t * 64 + w * 16), o[0], o[1], o[2], o[3]);
    }
    fence_proxy_async_smem();
    __syncthreads();   // stage ls is consumed and obuf[ob] is written
    if (t == 0) {
      if (QL_IN_BOUNDS(status, (ch + 1) * kDqChunk - 1, out_elems))
        bulk_store(out + ch * kDqChunk, obuf + ob * kDqOutBytes, kDqOutBytes);
      bulk_commit();
      if (first + issued * step < nchunks) issue(issued++);   // refill stage ls, kDqStages chunks ahead
    }
    S = S_next;
  }
  if (t == 0) {
    bulk_wait_all<0>();
    if (*abort_flag) {
      latch_status(status, QLORA_ERR_DEVICE_TIMEOUT);
      // let the loads still in flight (chunks it .. issued - 1) land before exiting
      for (int j = it; j < issued; ++j) mbar_wait(&bar[j % kDqStages], (j / kDqStages) & 1, 4000000000ull);
    }
  }
}

}  // namespace

size_t quantize_workspace_bytes(int64_t numel) {
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  return static_cast<size_t>((128 + 4 * nblocks + 255) / 256 * 256);
}

cudaError_t launch_quantize(const void *W, int dtype, int64_t numel, uint8_t *codes, uint8_t *absmax_q,
                            float *group_scale, const Nf4Table &tab, void *ws, int *status, cudaStream_t st) {
  const int64_t ngroups = (numel + kGroupElems - 1) / kGroupElems;
  const int64_t nblocks = (numel + kBlock - 1) / kBlock;
  const bool sgn = tab.qx != 0;
  unsigned long long *acc = sgn ? static_cast<unsigned long long *>(ws) : nullptr;
  float *abs_ws = sgn ? reinterpret_cast<float *>(static_cast<char *>(ws) + 128) : nullptr;
  prof_mark(kProfQuant, true, st);
  if (sgn) {
    cudaError_t e = cudaMemsetAsync(acc, 0, kSumDigits * sizeof(unsigned long long), st);
    if (e != cudaSuccess) return e;
  }
  if (dtype == QLORA_DTYPE_BF16)
    nf4_quantize_kernel<uint16_t><<<static_cast<unsigned>(ngroups), kQuantThreads, 0, st>>>(
        static_cast<const uint16_t *>(W), numel, codes, absmax_q, group_scale, tab, abs_ws, acc, status);
  else
    nf4_quantize_kernel<float><<<static_cast<unsigned>(ngroups), kQuantThreads, 0, st>>>(
        static_cast<const float *>(W), numel, codes, absmax_q, group_scale, tab, abs_ws, acc, status);
  if (sgn)
    nf4_dq_signed_kernel<<<static_cast<unsigned>(ngroups), kQuantThreads, 0, st>>>(
        abs_ws, acc, nblocks, absmax_q, group_scale, const_cast<float *>(tab.offset), status);
  prof_mark(kProfQuant, false, st);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale, int64_t numel,
                              const Nf4Table &tab, uint16_t *out, cudaStream_t st) {
  // whole double-quantization groups (two chunks each) on the bulk path
  const int64_t nfull = (numel / (kBlock * kGroup)) * (kBlock * kGroup / kDqChunk);
  prof_mark(kProfDequant, true, st);
  if (nfull > 0) {
    int *status = device_status_ptr();
    // as many CTAs as are co-resident, each taking the same number of chunks (so no
    // last round runs with a part of the grid idle)
    const int64_t slots = static_cast<int64_t>(device_sm_count_cached()) * QLORA_DQ_CTAS_PER_SM;
    const int64_t per = (nfull + slots - 1) / slots;
    const int64_t blocks = (nfull + per - 1) / per;
    cudaError_t e = cudaFuncSetAttribute(nf4_dequantize_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDqSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(kDeqThreads);
    cfg.dynamicSmemBytes = kDqSmem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the previous kernel's tail
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, nf4_dequantize_bulk_kernel, codes, absmax_q, group_scale, nfull, out, numel, tab,
                           status, wait_limit());
    if (e != cudaSuccess) return e;
  }
  const int64_t done = nfull * kDqChunk;
  if (done < numel) {
    // ragged tail (less than one group of 16384 weights): the per-thread kernel on the
    // remainder; the offset is a whole number of groups, so block and group indices line up.
    const int64_t rest = numel - done;
    const int64_t nchunk = (rest + 31) / 32;
    int64_t blocks = (nchunk + kDeqThreads - 1) / kDeqThreads;
    nf4_dequantize_kernel<<<static_cast<unsigned>(blocks), kDeqThreads, 0, st>>>(
        codes + done / 2, absmax_q + done / kBlock, group_scale + done / (kBlock * kGroup), rest, out + done, tab,
        device_status_ptr());
  }
  prof_mark(kProfDequant, false, st);
  return cudaGetLastError();
}

}  // namespace qlora
