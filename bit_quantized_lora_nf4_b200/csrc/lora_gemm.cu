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
// Each is C[i,j] = sum_k opA(i,k) opB(j,k), computed on tcgen05 tensor cores
// (lora_tc.cu) as fp32 partial sums over slices of the reduction; the kernels
// here add the slices in a fixed order (deterministic) and apply the scale.
// fp32 operands (H, G) enter as a bf16 hi/lo pair: x = hi + lo with
// hi = bf16(x), lo = bf16(x - hi), i.e. two stacked operands, which keeps
// about 16 significant bits.
#include "internal.h"

namespace qlora {

namespace {

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
