// NF4 block decode shared by the fused GEMM kernels and the GEMV.
//
// One 64-weight block has one dequantized constant a' = fl32(q * S), so its 16
// possible bf16 values T[c] = bf16(fl32(level[c] * a')) are computed once and
// every code of the block is looked up with byte permutes (prmt) from eight
// registers: LO[j] / HI[j] hold the low / high bytes of T[4j .. 4j+3].
#pragma once

#include "common.cuh"

namespace qlora {

// prmt.b32 in its default mode.  Callers pass selectors whose nibbles never
// have bit 3 set, so no byte is sign-replicated (this is why the intrinsic,
// which masks its selector, is not used: the mask costs an instruction).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// LO/HI byte tables of T[c] = bf16(fl32(level[c] * ap)).
__device__ __forceinline__ void nf4_block_table(float ap, const Nf4Table &tab, uint32_t (&LO)[4],
                                                uint32_t (&HI)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t p0 = pack_bf16x2(__fmul_rn(tab.level[4 * j + 0], ap), __fmul_rn(tab.level[4 * j + 1], ap));
    const uint32_t p1 = pack_bf16x2(__fmul_rn(tab.level[4 * j + 2], ap), __fmul_rn(tab.level[4 * j + 3], ap));
    LO[j] = prmt(p0, p1, 0x6420);
    HI[j] = prmt(p0, p1, 0x7531);
  }
}

// 8 codes in one word (element i in nibble i) -> 4 words of bf16 pairs,
// o[i] = T[code 2i] | T[code 2i+1] << 16.
__device__ __forceinline__ void nf4_lut8(uint32_t x, const uint32_t (&LO)[4], const uint32_t (&HI)[4],
                                         uint32_t (&o)[4]) {
  const uint32_t sel = x & 0x77777777u;                          // index within a half table
  const uint32_t pick = ((x >> 1) & 0x44444444u) | 0x32103210u;  // byte i from lower (i) or upper (i+4) half
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? (sel >> 16) : sel;
    const uint32_t q = h ? (pick >> 16) : pick;
    const uint32_t lo = prmt(prmt(LO[0], LO[1], s), prmt(LO[2], LO[3], s), q);
    const uint32_t hi = prmt(prmt(HI[0], HI[1], s), prmt(HI[2], HI[3], s), q);
    o[2 * h + 0] = prmt(lo, hi, 0x5140);
    o[2 * h + 1] = prmt(lo, hi, 0x7362);
  }
}

// Decode one block (codes: two 16-byte chunks at shared addresses c_lo, c_hi)
// into 8 16-byte chunks of a 128B-swizzled operand row: chunk w goes to
// row_addr + ((w ^ swz) << 4).
__device__ __forceinline__ void nf4_decode_row(uint32_t c_lo, uint32_t c_hi, uint32_t row_addr, uint32_t swz,
                                               float ap, const Nf4Table &tab) {
  uint32_t LO[4], HI[4];
  nf4_block_table(ap, tab, LO, HI);
  const uint4 a = ld_shared_v4(c_lo);
  const uint4 b = ld_shared_v4(c_hi);
  const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint32_t o[4];
    nf4_lut8(words[w], LO, HI, o);
    st_shared_v4(row_addr + ((static_cast<uint32_t>(w) ^ swz) << 4), o[0], o[1], o[2], o[3]);
  }
}

}  // namespace qlora
