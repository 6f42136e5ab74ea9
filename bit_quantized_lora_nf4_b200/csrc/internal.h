// Host-side declarations shared by the translation units of libqlora.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "qlora.h"

namespace qlora {

// NF4 table computed once on the host (normal quantiles, see api.cu).
const Nf4Table &nf4_table();
// The table of a QLORA_FORMAT_* (the NF4 one for QLORA_FORMAT_NF4); format must be valid.
const Nf4Table &format_table(int format);
// The decode description of a validated weight: its format's table plus the
// reading of its block constants (signed ones point `offset` at mu, stored
// after the group scales).
Nf4Table weight_table(const qlora_nf4_weight *w);
// Pointer, size, format and alignment checks of a weight header (QLORA_OK or the error).
qlora_status validate_weight(const qlora_nf4_weight *w);

// Address of the device status word on the current device (nullptr on error).
int *device_status_ptr();

// Current bound on pipeline waits, in clock cycles.
uint64_t wait_limit();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- kernel timing hook (see qlora_profile_enable) --------------------------
enum ProfKind { kProfAll = 0, kProfGemmFwd = 1, kProfGemmDgrad = 2, kProfLora = 3, kProfQuant = 4, kProfDequant = 5,
                kProfGemv = 6, kProfLqProduct = 7, kProfLqResidual = 8, kProfLqChol = 9, kProfLqJacobi = 10,
                kProfLqSmall = 11, kProfKinds = 12 };
// Records an event before (begin=true) or after a launch of `kind` on `st` when profiling is on.
void prof_mark(int kind, bool begin, cudaStream_t st);
// Whether the timing hook is recording (the backward then keeps every launch on the caller's stream).
bool prof_on();

// ---- tensor maps ------------------------------------------------------------
// 2D tiled map over a row-major [outer, inner] array.
bool make_tmap_2d(CUtensorMap *tm, const void *base, CUtensorMapDataType dtype, uint64_t inner, uint64_t outer,
                  uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// ---- kernels (launchers return the launch error) -------------------------------
// Quantizer.  tab.qx != 0 selects signed block constants; those need `ws`
// (quantize_workspace_bytes(numel) bytes) and write mu to tab.offset.
size_t quantize_workspace_bytes(int64_t numel);
// W holds QLORA_DTYPE_F32 or QLORA_DTYPE_BF16 elements.
cudaError_t launch_quantize(const void *W, int dtype, int64_t numel, uint8_t *codes, uint8_t *absmax_q,
                            float *group_scale, const Nf4Table &tab, void *ws, int *status, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t *codes, const uint8_t *absmax_q, const float *group_scale,
                              int64_t numel, const Nf4Table &tab, uint16_t *out, cudaStream_t st);

// Fused dequant-GEMM on tensor cores.
//   forward: out[M, wN] = act[M, wK] . W'^T + lora_act[M, r] . lora_w[wN, r]^T
//   dgrad  : out[M, wK] = act[M, wN] . W'   + lora_act[M, r] . lora_w[r, wK]
struct QGemmArgs {
  bool dgrad;
  int64_t M;
  int64_t wN, wK;
  const uint16_t *act;
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *lora_act;
  const uint16_t *lora_w;
  int r;
  uint16_t *out;
  Nf4Table tab;        // weight_table() of the weight
  const uint16_t *wdense = nullptr;   // dense bf16 W' [wN, wK] instead of the packed weight (pair kernel only)
  void *sk_ws = nullptr;              // pair kernel: pair_sk_workspace_bytes(M) for its stream-K tail (null: none)
  bool sk_zeroed = false;             // qgemm_prepare_split already cleared the tail's counters on the stream
};
// Workspace of the pair kernel's stream-K tail (fp32 pieces of shared tiles and their counters).
size_t pair_sk_workspace_bytes(int64_t M);
// QLORA_STREAM_K_* set by qlora_set_stream_k.
int stream_k_mode();
qlora_status launch_qgemm(const QGemmArgs &a, cudaStream_t st);
// The same product on a CTA pair (256-row tiles); launch_qgemm dispatches to it
// for M > kPairMinRows and for a dense W'.
constexpr int64_t kPairMinRows = 128;
qlora_status launch_qgemm_pair(const QGemmArgs &a, cudaStream_t st);
// Clears the stream-K tail's counters on `st` now when the launch of `a` will
// split its last round (the same decision the launch makes), so that the
// launch can follow the kernel before it with programmatic dependent launch;
// sets *zeroed accordingly.  Issue it before the products the GEMM depends on.
qlora_status qgemm_prepare_split(const QGemmArgs &a, cudaStream_t st, bool *zeroed);

// Few-token forward: Y[M, N] = X W'^T + (s X A^T) B^T for M <= 16.
struct GemvArgs {
  int64_t M, wN, wK;
  const uint16_t *X;
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *A;   // [r, K]
  const uint16_t *B;   // [N, r]
  int r;
  float s;
  uint16_t *Y;
  float *H_out;        // optional [M, r]
  void *workspace;     // gemv_workspace_bytes(M, N, K, r) bytes, 256-byte aligned
  Nf4Table tab;        // weight_table() of the weight
};
size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
qlora_status launch_gemv(const GemvArgs &a, cudaStream_t st);
constexpr int kGemvMaxTokens = 16;
bool gemv_enabled();

// Tall-skinny adapter products on tcgen05 tensor cores (lora_tc.cu), split over
// the reduction with fp32 partials part[z][I][J]:  C[i,j] = sum_k opA(i,k) opB(j,k),
// opX(i,k) = X[i*ld + k] when K-major, X[k*ld + i] otherwise.
// What the product's epilogue writes.  With kind != kSkinnyPartial the splits
// of one output tile run as a thread-block cluster and are added in split
// order inside the kernel (no partial buffer, no second kernel):
//   kSkinnyH     H = sum; out_f = H, out_b = bf16(s H), out_hl = [hi | lo] of H (optional)
//   kSkinnyG     G = s sum; out_b = bf16(G), out_hl = [hi | lo] of G; and, when aux is set,
//                aux_hl = [hi | lo] of the fp32 matrix aux (same [I, J] shape) for the tile's rows
//   kSkinnyCols  out_f[i][j] = s * sum (C[i][j] + C[i][half + j]),  j < half = J / 2
//   kSkinnyRows  out_f[i][j] = sum (C[i][j] + C[half + i][j]),      i < half = I / 2
enum SkinnyKind { kSkinnyPartial = 0, kSkinnyH = 1, kSkinnyG = 2, kSkinnyCols = 3, kSkinnyRows = 4 };
struct SkinnyEpilogue {
  int kind = kSkinnyPartial;
  float s = 1.0f;
  float *out_f = nullptr;
  uint16_t *out_b = nullptr;
  uint16_t *out_hl = nullptr;
  const float *aux = nullptr;
  uint16_t *aux_hl = nullptr;
};
struct SkinnyArgs {
  const uint16_t *A;
  int64_t lda;
  bool a_kmajor;
  const uint16_t *B;
  int64_t ldb;
  bool b_kmajor;
  int64_t I, J, Kred;
  int splits;
  int64_t k_per_split;
  float *part;                 // [splits][I][J] fp32, written only by kSkinnyPartial
  SkinnyEpilogue ep;
};
// Whether the product can finish inside the kernel (cluster of its splits).
bool skinny_fused_ok(const SkinnyArgs &a);
cudaError_t launch_skinny(const SkinnyArgs &a, cudaStream_t st);
// fp32 partial sums a product's launch may write (part): the larger of the
// fused layout [tile][split][128 x min(128, J)] and the plain [split][I][J].
// Two products in one launch take the first's floats and then the second's.
size_t skinny_part_floats(int64_t I, int64_t J, int splits);
// Two fused products in one launch: same operand layouts and split count.
bool skinny_pair_ok(const SkinnyArgs &a, const SkinnyArgs &b);
cudaError_t launch_skinny_pair(const SkinnyArgs &a, const SkinnyArgs &b, cudaStream_t st);
// Pick the split count for a skinny product, or for two sharing one launch
// and one reduction length (deterministic in the sizes).
void skinny_plan(int64_t I, int64_t J, int64_t Kred, int *splits, int64_t *k_per_split);
void skinny_plan_pair(int64_t I0, int64_t J0, int64_t I1, int64_t J1, int64_t Kred, int *splits,
                      int64_t *k_per_split);

// Epilogues of the skinny products.
//   H  = sum_z part            -> H (fp32 [M,r]); sH = bf16(s*H) [M,r]; Hs = [bf16 hi | bf16 lo] [M,2r] (optional)
cudaError_t launch_finalize_h(const float *part, int splits, int64_t M, int r, float s, float *H, uint16_t *sH,
                              uint16_t *Hs, cudaStream_t st);
//   Hs from an existing fp32 H (backward with a saved H)
cudaError_t launch_split_hilo(const float *H, int64_t M, int r, uint16_t *Hs, cudaStream_t st);
//   G = s * sum_z part -> Gb = bf16(G) [M,r], Gs = [hi | lo] [M,2r]
cudaError_t launch_finalize_g(const float *part, int splits, int64_t M, int r, float s, uint16_t *Gb, uint16_t *Gs,
                              cudaStream_t st);
//   out[i,j] = scale * sum_z (part[z][i][j] + part[z][i][j + half])  for j < half  (row-split layout, I rows)
cudaError_t launch_finalize_cols(const float *part, int splits, int64_t I, int64_t half, float scale, float *out,
                                 cudaStream_t st);
//   out[i,j] = sum_z (part[z][i][j] + part[z][i + half][j])          for i < half  (J cols)
cudaError_t launch_finalize_rows(const float *part, int splits, int64_t half, int64_t J, float *out,
                                 cudaStream_t st);

}  // namespace qlora
