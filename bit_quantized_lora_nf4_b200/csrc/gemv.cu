// Few-token forward (M <= 16): memory-bound dequant-GEMV.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": every pass expands the 4-bit base to 16-bit as it runs.  With a
// handful of tokens the packed weight stream (0.516 B per weight) is the whole
// cost: the codes stream into shared memory by TMA and are decoded straight
// into tensor-core register fragments.  The decode (a per-block 16-entry bf16
// table and byte permutes) runs on the integer pipe, which puts this path's
// ceiling below the HBM roofline.
//
// One cooperative launch (every CTA resident), three phases:
//   1. H CTAs (one per 16 adapter rows) compute s H = s X A^T on mma.sync with
//      a fixed-order reduction over their warps and store it as a bf16 hi/lo
//      pair (and H in fp32 when asked).  Weight CTAs stream the weight: it is
//      cut into positions (16-row tile, 256-wide K step) and weight warp g of
//      G takes positions [g U / G, (g+1) U / G), so every SM gets the same
//      decode work to within one position.  Per position a thread decodes one
//      64-weight block of two rows into m16n8k16 A fragments (tokens are the
//      8-column B operand; two column tiles when M > 8).  A warp stores its
//      fp32 sum for every tile it touches as that tile's piece number
//      g - g0(t), g0(t) being the first warp on the tile.
//   2. One grid-wide barrier (bounded wait).
//   3. Every warp finishes tiles t = w, w + W, ...: adds the tile's pieces in
//      piece order (a fixed order, so results are deterministic), adds
//      (s H) B^T with two more mma chains, stores bf16 Y.
#include <atomic>
#include <random>

#include "decode.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int GV_WARPS = 8;            // warps per CTA
constexpr int GV_THREADS = 32 * GV_WARPS;
#ifndef QLORA_GEMV_CTAS_PER_SM
#define QLORA_GEMV_CTAS_PER_SM 2
#endif
constexpr int GV_CTAS_PER_SM = QLORA_GEMV_CTAS_PER_SM;

// One position's codes arrive by TMA as a 16-row x 128-byte box (256 codes of
// each of the tile's rows), 128-byte swizzled, into a per-warp ring.
constexpr int GV_STAGE_BYTES = 16 * 128;
#ifndef QLORA_GEMV_STAGES
#define QLORA_GEMV_STAGES 2
#endif
constexpr int GV_STAGES = QLORA_GEMV_STAGES;
constexpr int GV_RING_BYTES = GV_WARPS * GV_STAGES * GV_STAGE_BYTES;
constexpr int GV_RED_OFFSET = GV_RING_BYTES + 1024;          // after the ring and its barriers
constexpr int GV_RED_BYTES = GV_WARPS * 2 * 4 * 32 * 4;      // H CTAs: per-warp C fragments (two token tiles)
constexpr int GV_XS_OFFSET = GV_RED_OFFSET + GV_RED_BYTES;
constexpr int GV_SMEM_BASE = GV_XS_OFFSET + 1024;             // + alignment slack of the dynamic segment
constexpr int GV_XS_MAX = 64 * 1024;                          // activations kept in shared memory up to this size

// Activations in shared memory: token row m at m * xs_row (rows copied whole by
// one bulk copy each, so every CTA asks L2 for whole rows, not 16-byte pieces),
// element k at 2 k.  xs_row / 16 = 4 (mod 8) puts consecutive rows in different
// bank groups.
__host__ __device__ constexpr int xs_row_bytes(int KB) { return 16 * (KB * 8 + 4); }

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Loads with L1 eviction hints: the activations are re-read by every warp of
// the SM (keep them), the block constants are touched once.
__device__ __forceinline__ uint4 ldg_keep_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::evict_last.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint32_t ldg_once_u8(const uint8_t *p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float ldg_once_f32(const float *p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}


// Grid-wide barrier of the cooperative launch (every CTA resident), on a 64-bit
// word of the workspace: the high half holds the launch's epoch (unique per
// launch in this process, from a random start), the low half the arrivals of
// that launch so far.  CTA 0 stamps the word with its epoch and a zero count
// when the kernel starts (grid_barrier_open); every CTA counts itself in with an
// atomic add only once it sees that epoch, so whatever the word held before
// (an earlier launch's tag, or never written) is neither counted nor needs
// clearing.  Round `round` (1, 2, ...) is complete once round x CTAs have
// arrived.  Each CTA's writes before the barrier are published by its thread
// 0 (after the CTA barrier) with a GPU-scope fence before it counts itself in.
// Waits are bounded; on timeout the status is latched and the CTA goes on.
__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const unsigned long long *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void grid_barrier_open(unsigned long long *word, uint32_t epoch) {
  if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(word, static_cast<unsigned long long>(epoch) << 32);
}
__device__ __forceinline__ void grid_barrier(unsigned long long *word, uint32_t epoch, uint32_t round, int *status,
                                             uint64_t limit) {
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t n = gridDim.x * gridDim.y * gridDim.z;
    __threadfence();
    const long long t0 = clock64();
    bool ok = true;
    while ((ld_acquire_gpu_u64(word) >> 32) != epoch) {   // the launch's stamp is in place
      if (static_cast<uint64_t>(clock64() - t0) > limit) {
        ok = false;
        break;
      }
    }
    if (ok) {
      atomicAdd(word, 1ull);
      while (true) {
        const uint64_t w = ld_acquire_gpu_u64(word);
        if ((w >> 32) == epoch && static_cast<uint32_t>(w) >= round * n) break;
        if (static_cast<uint64_t>(clock64() - t0) > limit) {
          ok = false;
          break;
        }
      }
    }
    if (!ok) latch_status(status, QLORA_ERR_DEVICE_TIMEOUT);
  }
  __syncthreads();
}

// First position of weight warp g's range, and the warp whose range holds position u.
__device__ __forceinline__ int range_start(int g, int U, int G) {
  return static_cast<int>(static_cast<int64_t>(g) * U / G);
}
__device__ __forceinline__ int range_owner(int u, int U, int G) {
  return static_cast<int>((static_cast<int64_t>(u + 1) * G - 1) / U);
}

struct GemvParams {
  const uint16_t *X;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *A;        // [r, K]
  const uint16_t *B;        // [N, r]
  float s;
  uint16_t *Y;              // [M, N]
  float *H_out;             // optional [M, r]
  uint16_t *sh_hi;          // [8 NT, r16] s H, high bf16 part
  uint16_t *sh_lo;          //              and the remainder
  float *pieces;            // [T][P][M][16] tile sums, one per weight warp that touches the tile
  float *hpart;             // [JT][HS][8 NT][16] partial H of the H CTAs (HS > 1)
  unsigned long long *bar;  // grid barrier word (see grid_barrier)
  uint32_t epoch;           // this launch's tag on it
  int M, r, r16;
  int JT, HS;               // H CTAs: blockIdx.x < JT * HS, adapter tile blockIdx.x / HS, K split blockIdx.x % HS
  int G;                    // weight warps (CTA blockIdx.x - JT HS holds weight warps 8 (that) .. +7)
  int S, U, T, P;           // K steps per tile, positions, tiles, piece slots per tile
  int xs_row;               // row pitch of the activations in shared memory (0: global memory)
  int64_t N, K;
  int *status;
  uint64_t wait_limit;
  Nf4Table tab;
};

// Quantized constants of one position for rows n0 = 16 t + g and n0 + 8, block 4 step + c.
struct PosConst {
  uint32_t q0, q1;   // 8-bit block constants; bit 8 set for rows past N / blocks past K
  float S0, S1;      // 32-bit group constants
};

// a' of one position's block, and 0 for the padding positions (bit 8 of q set).
__device__ __forceinline__ float pos_constant(uint32_t q, float S, uint32_t qx, float mu) {
  return (q & 0x100u) ? 0.0f : block_constant(q, S, qx, mu);
}

// Where a thread reads its activation fragments: token rows past M read the
// last live token (those output columns are never stored), blocks past K read
// the last block (their weights are zero).
template <int NT, bool XS>
struct XSource {
  const uint16_t *row[NT];
  uint32_t srow[NT];
  __device__ __forceinline__ XSource(const GemvParams &p, uint32_t xs, int g) {
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) {
      const int m = min(tt * 8 + g, p.M - 1);
      row[tt] = p.X + static_cast<int64_t>(m) * p.K;
      srow[tt] = xs + m * p.xs_row;
    }
  }
  // 16 bytes: X[token][64 kb + 8 w .. +7]
  __device__ __forceinline__ uint4 load(int tt, int kb, int w) const {
    if (XS) return ld_shared_v4(srow[tt] + kb * 128 + w * 16);
    return ldg_keep_v4(reinterpret_cast<const uint4 *>(row[tt] + kb * kBlock) + w);
  }
};

// s H (and H) from the C fragment of one adapter tile.
template <int NT>
__device__ __forceinline__ void write_sh(const GemvParams &p, int j0, int t, int e, int lane, float h) {
  const int g = lane >> 2, c = lane & 3;
  // C fragment: H^T[j][tok], j = j0 + g + 8 (e >> 1), tok = 8 t + 2 c + (e & 1)
  const int j = j0 + g + 8 * (e >> 1);
  const int tok = 8 * t + 2 * c + (e & 1);
  if (p.H_out && tok < p.M && j < p.r) p.H_out[static_cast<int64_t>(tok) * p.r + j] = h;
  const float sh = __fmul_rn(p.s, h);
  const __nv_bfloat16 hi = __float2bfloat16_rn(sh);
  const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(sh, __bfloat162float(hi)));
  p.sh_hi[tok * p.r16 + j] = *reinterpret_cast<const uint16_t *>(&hi);
  p.sh_lo[tok * p.r16 + j] = *reinterpret_cast<const uint16_t *>(&lo);
}

// Phase 1, H CTA (adapter tile jt = blockIdx.x / HS: rows j0 .. j0+15; K part
// hs = blockIdx.x % HS).  H warp q = 8 hs + warp takes K steps q, q + 8 HS, ...;
// in a step thread (g, c) covers columns 256 step + 64 c .. +63 of A rows j0 + g
// and j0 + g + 8, in the same K order as the weight.  The 8 warps are added in
// a fixed order; with one K part the CTA writes s H, otherwise its partial sum.
template <int NT, bool XS>
__device__ __forceinline__ void h_role(const GemvParams &p, const XSource<NT, XS> &x, float *red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int jt = blockIdx.x / p.HS, hs = blockIdx.x - jt * p.HS;
  const int j0 = jt * 16;
  const int KB = static_cast<int>(p.K / kBlock);
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;
  const int ja = j0 + g, jb = j0 + g + 8;
  const uint4 *arow = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(min(ja, p.r - 1)) * p.K);
  const uint4 *brow = reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(min(jb, p.r - 1)) * p.K);
  for (int st = hs * GV_WARPS + warp; st < p.S; st += GV_WARPS * p.HS) {
    const int kb = 4 * st + c;
    const int kbc = min(kb, KB - 1);
    const bool va = kb < KB && ja < p.r, vb = kb < KB && jb < p.r;
#pragma unroll
    for (int h = 0; h < 2; ++h) {   // half a block of each row in flight at once
      uint4 ua[4], ub[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        ua[w] = __ldg(arow + kbc * 8 + 4 * h + w);
        ub[w] = __ldg(brow + kbc * 8 + 4 * h + w);
      }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const uint4 a4 = va ? ua[w] : make_uint4(0, 0, 0, 0);
        const uint4 b4 = vb ? ub[w] : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint4 xv = x.load(t, kbc, 4 * h + w);
          mma16816(acc[t], a4.x, b4.x, a4.y, b4.y, xv.x, xv.y);
          mma16816(acc[t], a4.z, b4.z, a4.w, b4.w, xv.z, xv.w);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) red[((warp * NT + t) * 4 + e) * 32 + lane] = acc[t][e];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float h = 0.0f;
#pragma unroll
        for (int w = 0; w < GV_WARPS; ++w) h += red[((w * NT + t) * 4 + e) * 32 + lane];
        if (p.HS == 1) {
          write_sh<NT>(p, j0, t, e, lane, h);
        } else {   // partial: [jt][hs][tok][16 j]
          const int tok = 8 * t + 2 * c + (e & 1), jl = g + 8 * (e >> 1);
          p.hpart[((static_cast<int64_t>(jt) * p.HS + hs) * 8 * NT + tok) * 16 + jl] = h;
        }
      }
    }
  }
}

// Between the two grid barriers (HS > 1): warp jt of all warps adds the HS
// partial sums of adapter tile jt in K-part order and writes s H.
template <int NT>
__device__ __forceinline__ void h_finish(const GemvParams &p) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int jt = blockIdx.x * GV_WARPS + (threadIdx.x >> 5);
  if (jt >= p.JT) return;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = 8 * t + 2 * c + (e & 1), jl = g + 8 * (e >> 1);
      float h = 0.0f;
      for (int hs = 0; hs < p.HS; ++hs) h += __ldcg(p.hpart + ((static_cast<int64_t>(jt) * p.HS + hs) * 8 * NT + tok) * 16 + jl);
      write_sh<NT>(p, jt * 16, t, e, lane, h);
    }
  }
}

// The code stream of one weight warp: lane 0 keeps GV_STAGES positions of the
// warp's range in flight (issue cursor: position iu = it S + is).
struct CodeStream {
  uint8_t *ring;
  uint64_t *bar;
  int it, is, iu;
  __device__ __forceinline__ void issue(const CUtensorMap *tm, int slot, int S) {
    mbar_arrive_expect_tx(&bar[slot], GV_STAGE_BYTES);   // the box is always full: TMA zero-fills past N / K
    tma_load_2d(ring + slot * GV_STAGE_BYTES, tm, &bar[slot], is * 128, it * 16);
    ++iu;
    if (++is == S) {
      is = 0;
      ++it;
    }
  }
};

// Phase 1, weight warp gw: positions [a, b).  The sum over the warp's part of
// each tile it touches is stored, as soon as that part is done, as the tile's
// piece gw - g0 (g0: the first warp on the tile).
template <int NT, bool XS>
__device__ __forceinline__ void weight_role(const CUtensorMap *tm, const GemvParams &p, const XSource<NT, XS> &x,
                                            CodeStream &cs, int gw, int a, int b) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int S = p.S;
  const int KB = static_cast<int>(p.K / kBlock);
  const int N = static_cast<int>(p.N);
  const int first_tile = a / S;
  int g0 = range_owner(first_tile * S, p.U, p.G);   // first warp on the current tile

  // Block constants one position ahead in registers.  Rows past N and blocks
  // past K read a clamped, valid address and are marked in bit 8 of q, so
  // their weights decode to (signed) zero.
  const float mu = dq_offset(p.tab);
  int ft = first_tile, fs = a - first_tile * S, fu = a;
  auto fetch = [&](PosConst &f) {
    const int kb = 4 * fs + c;
    const int kbc = min(kb, KB - 1);
    const int n0 = ft * 16 + g;
    const int bi0 = min(n0, N - 1) * KB + kbc, bi1 = min(n0 + 8, N - 1) * KB + kbc;   // < 2^31 (host check)
    const bool kv = kb < KB;
    f.q0 = ldg_once_u8(p.absmax_q + bi0) | ((kv && n0 < N) ? 0u : 0x100u);
    f.q1 = ldg_once_u8(p.absmax_q + bi1) | ((kv && n0 + 8 < N) ? 0u : 0x100u);
    f.S0 = ldg_once_f32(p.group_scale + (bi0 >> 8));
    f.S1 = ldg_once_f32(p.group_scale + (bi1 >> 8));
    if (fu + 1 < b) {   // advance, staying on the last position of the range
      ++fu;
      if (++fs == S) {
        fs = 0;
        ++ft;
      }
    }
  };
  PosConst q;
  fetch(q);

  float acc[NT][4];
#pragma unroll
  for (int tt = 0; tt < NT; ++tt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;

  int t = first_tile, step = a - first_tile * S;
  int ip = 0;   // index of position u within the range
  for (int u = a; u < b; ++u, ++ip) {
    const PosConst f = q;
    fetch(q);

    const int kbc = min(4 * step + c, KB - 1);
    uint4 xv[2][NT];   // activation words, read one word ahead
#pragma unroll
    for (int tt = 0; tt < NT; ++tt) xv[0][tt] = x.load(tt, kbc, 0);

    uint32_t LO[2][4], HI[2][4];
    nf4_block_table(pos_constant(f.q0, f.S0, p.tab.qx, mu), p.tab, LO[0], HI[0]);
    nf4_block_table(pos_constant(f.q1, f.S1, p.tab.qx, mu), p.tab, LO[1], HI[1]);

    // codes of rows g and g + 8, 32 bytes each at column 32 c: 16-byte chunks 2c
    // and 2c+1, stored at chunk ^ (row & 7) by the 128-byte swizzle
    const int slot = ip % GV_STAGES;
    if (!__all_sync(0xffffffffu, mbar_wait(&cs.bar[slot], (ip / GV_STAGES) & 1, p.wait_limit))) {
      if (lane == 0) {
        latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
        // let the copies still in flight land before the ring is abandoned
        for (int j = ip; j < cs.iu - a; ++j)
          mbar_wait(&cs.bar[j % GV_STAGES], (j / GV_STAGES) & 1, 4000000000ull);
      }
      __syncwarp();
      return;
    }
    const uint32_t rb = smem_addr(cs.ring + slot * GV_STAGE_BYTES);
    const uint32_t c0 = static_cast<uint32_t>((2 * c) ^ g) << 4, c1 = static_cast<uint32_t>((2 * c + 1) ^ g) << 4;
    const uint4 w0 = ld_shared_v4(rb + g * 128 + c0), w1 = ld_shared_v4(rb + g * 128 + c1);
    const uint4 w2 = ld_shared_v4(rb + (g + 8) * 128 + c0), w3 = ld_shared_v4(rb + (g + 8) * 128 + c1);
    const uint32_t wa[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const uint32_t wb[8] = {w2.x, w2.y, w2.z, w2.w, w3.x, w3.y, w3.z, w3.w};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      if (w + 1 < 8) {
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) xv[(w + 1) & 1][tt] = x.load(tt, kbc, w + 1);
      }
      uint32_t o0[4], o1[4];
      nf4_lut8(wa[w], LO[0], HI[0], o0);
      nf4_lut8(wb[w], LO[1], HI[1], o1);
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) {
        const uint4 xw = xv[w & 1][tt];
        mma16816(acc[tt], o0[0], o1[0], o0[1], o1[1], xw.x, xw.y);
        mma16816(acc[tt], o0[2], o1[2], o0[3], o1[3], xw.z, xw.w);
      }
    }
    // every lane has used its codes: the slot takes the position GV_STAGES ahead
    __syncwarp();
    if (lane == 0 && cs.iu < b) {
      fence_proxy_async_smem();
      cs.issue(tm, slot, S);
    }

    const int tile = t;
    if (++step == S) {
      step = 0;
      ++t;
    } else if (u + 1 < b) {
      continue;   // the tile continues in this warp's range
    }
    // this warp's part of the tile is done: piece gw - g0
    float *pc = p.pieces + (static_cast<int64_t>(tile) * p.P + (gw - g0)) * 16 * p.M;
    g0 = gw;   // every later tile of the range starts in this warp
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tt * 8 + 2 * c + (e & 1);
        if (tok < p.M) pc[tok * 16 + g + 8 * (e >> 1)] = acc[tt][e];
      }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
  }
}

// acc += (s H) B^T for the 16 rows of tile t: the rows of B are the A operand
// (the adapter index j is the reduction index), s H the B operand, hi part then
// lo part.  The loads of four 16-wide adapter steps are issued together.
template <int NT>
__device__ __forceinline__ void add_lora(const GemvParams &p, int t, float (&acc)[NT][4], int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int64_t n0 = static_cast<int64_t>(t) * 16 + g, n1 = n0 + 8;
  const bool v0 = n0 < p.N, v1 = n1 < p.N;
  const uint32_t *B0 = reinterpret_cast<const uint32_t *>(p.B + min(n0, p.N - 1) * p.r);
  const uint32_t *B1 = reinterpret_cast<const uint32_t *>(p.B + min(n1, p.N - 1) * p.r);
  for (int j0 = 0; j0 < p.r; j0 += 64) {
    uint32_t a[4][4], h[4][NT][2], l[4][NT][2];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int ja = j0 + 16 * q + 2 * c, jb = ja + 8;   // ja < r whenever j0 + 16 q < r (r % 8 == 0)
      const bool va = ja < p.r, vb = jb < p.r;
      const int jac = va ? ja : 0, jbc = vb ? jb : 0;
      a[q][0] = (v0 && va) ? __ldg(B0 + jac / 2) : 0u;
      a[q][1] = (v1 && va) ? __ldg(B1 + jac / 2) : 0u;
      a[q][2] = (v0 && vb) ? __ldg(B0 + jbc / 2) : 0u;
      a[q][3] = (v1 && vb) ? __ldg(B1 + jbc / 2) : 0u;
#pragma unroll
      for (int tt = 0; tt < NT; ++tt) {   // s H is padded to r16 columns
        const int ra = min(ja, p.r16 - 2), rb = min(jb, p.r16 - 2);
        const uint32_t *hr = reinterpret_cast<const uint32_t *>(p.sh_hi + (tt * 8 + g) * p.r16);
        const uint32_t *lr = reinterpret_cast<const uint32_t *>(p.sh_lo + (tt * 8 + g) * p.r16);
        // s H is read by every finishing warp: L1-cached loads (no SM holds a line
        // of it from before the grid barrier, so none can be stale)
        h[q][tt][0] = hr[ra / 2];
        h[q][tt][1] = hr[rb / 2];
        l[q][tt][0] = lr[ra / 2];
        l[q][tt][1] = lr[rb / 2];
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + 16 * q < p.r) {
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
          mma16816(acc[tt], a[q][0], a[q][1], a[q][2], a[q][3], h[q][tt][0], h[q][tt][1]);
          mma16816(acc[tt], a[q][0], a[q][1], a[q][2], a[q][3], l[q][tt][0], l[q][tt][1]);
        }
      }
    }
  }
}

template <int NT>
__device__ __forceinline__ void store_y(const GemvParams &p, int t, const float (&acc)[NT][4], int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int64_t n0 = static_cast<int64_t>(t) * 16 + g;
#pragma unroll
  for (int tt = 0; tt < NT; ++tt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int tok = tt * 8 + 2 * c + (e & 1);
      const int64_t n = n0 + 8 * (e >> 1);
      if (tok < p.M && n < p.N) {
        const __nv_bfloat16 y = __float2bfloat16_rn(acc[tt][e]);
        p.Y[static_cast<int64_t>(tok) * p.N + n] = *reinterpret_cast<const uint16_t *>(&y);
      }
    }
  }
}

// Phase 3: warp w of all W warps finishes tiles w, w + W, ...: the tile's
// pieces in warp order (a fixed order), then the adapter term, then Y.  The
// loads of the pieces, of the tile's rows of B and of s H are issued together.
template <int NT>
__device__ __forceinline__ void finish_role(const GemvParams &p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int W = gridDim.x * GV_WARPS;
  for (int t = blockIdx.x * GV_WARPS + warp; t < p.T; t += W) {
    const int np = range_owner((t + 1) * p.S - 1, p.U, p.G) - range_owner(t * p.S, p.U, p.G) + 1;
    const float *src = p.pieces + static_cast<int64_t>(t) * p.P * 16 * p.M;
    float acc[NT][4];
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
    constexpr int GV_PIECE_BATCH = 16 / NT;   // pieces loaded together
    for (int i0 = 0; i0 < np; i0 += GV_PIECE_BATCH) {
      float v[GV_PIECE_BATCH][NT][4];
#pragma unroll
      for (int i = 0; i < GV_PIECE_BATCH; ++i)
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tt * 8 + 2 * c + (e & 1);
            v[i][tt][e] = (i0 + i < np && tok < p.M) ? __ldcg(src + ((i0 + i) * p.M + tok) * 16 + g + 8 * (e >> 1)) : 0.0f;
          }
#pragma unroll
      for (int i = 0; i < GV_PIECE_BATCH; ++i)
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[tt][e] += v[i][tt][e];
    }
    add_lora<NT>(p, t, acc, lane);
    store_y<NT>(p, t, acc, lane);
  }
}

#ifndef QLORA_GEMV_MAXNREG
#define QLORA_GEMV_MAXNREG 128
#endif
template <int NT, bool XS>
__global__ void __maxnreg__(QLORA_GEMV_MAXNREG) gemv_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                          const GemvParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // The next kernel on the stream may be scheduled once every CTA has passed
  // here; nothing is read before the previous kernel's writes are visible.
  griddep_launch_dependents();
  griddep_wait();
  grid_barrier_open(p.bar, p.epoch);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool h_cta = static_cast<int>(blockIdx.x) < p.JT * p.HS;
  const int gw = (static_cast<int>(blockIdx.x) - p.JT * p.HS) * GV_WARPS + warp;   // weight warp index
  const bool weight = !h_cta && gw < p.G;
  const int a = weight ? range_start(gw, p.U, p.G) : 0, b = weight ? range_start(gw + 1, p.U, p.G) : 0;
  float *red = reinterpret_cast<float *>(smem + GV_RED_OFFSET);

  // The activations first (every warp needs them before its first product),
  // then the first code boxes.
  const uint32_t xs = smem_addr(smem + GV_XS_OFFSET);
  uint64_t *xbar = reinterpret_cast<uint64_t *>(smem + GV_RING_BYTES) + GV_WARPS * GV_STAGES;
  if (XS && threadIdx.x == 0) {
    mbar_init(xbar, 1);
    fence_mbar_init();
    const uint32_t row = static_cast<uint32_t>(p.K * 2);
    mbar_arrive_expect_tx(xbar, row * p.M);
    for (int m = 0; m < p.M; ++m)
      bulk_load(smem + GV_XS_OFFSET + m * p.xs_row, p.X + static_cast<int64_t>(m) * p.K, row, xbar);
  }
  CodeStream cs{smem + warp * GV_STAGES * GV_STAGE_BYTES,
                reinterpret_cast<uint64_t *>(smem + GV_RING_BYTES) + warp * GV_STAGES, a / p.S, a - (a / p.S) * p.S, a};
  if (weight && lane == 0) {
    for (int i = 0; i < GV_STAGES; ++i) mbar_init(&cs.bar[i], 1);
    fence_mbar_init();
    for (int i = 0; i < GV_STAGES && cs.iu < b; ++i) cs.issue(&tm_codes, i, p.S);
  }
  if (XS) {
    __syncthreads();   // the barrier is initialised
    if (!mbar_wait(xbar, 0, p.wait_limit)) latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
  }
  __syncwarp();
  const XSource<NT, XS> x(p, xs, lane >> 2);

  if (h_cta) {
    h_role<NT, XS>(p, x, red);
  } else {
    if (weight) weight_role<NT, XS>(&tm_codes, p, x, cs, gw, a, b);
  }

  grid_barrier(p.bar, p.epoch, 1, p.status, p.wait_limit);   // pieces (and s H or its partial sums) complete and visible
  if (p.HS > 1) {
    h_finish<NT>(p);
    grid_barrier(p.bar, p.epoch, 2, p.status, p.wait_limit);
  }
  finish_role<NT>(p);
}

int device_sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
      v > 0)
    return v;
  cudaGetLastError();   // no device here (sizing only): assume the largest part this library targets
  return 148;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Work split and workspace carve-up shared by the size query and the launch.
// The piece slots per tile are sized for the largest weight-warp count the
// device can hold, so the layout does not depend on the occupancy found at launch.
struct GemvLayout {
  int NT, r16, JT, HS, P;
  int64_t T, S, U, G_max;
  bool fits32;
  size_t off_pieces, off_hpart, off_hi, off_lo, off_bar, total;
};

GemvLayout gemv_layout(int64_t M, int64_t N, int64_t K, int r) {
  GemvLayout L{};
  L.NT = M <= 8 ? 1 : 2;
  L.r16 = (r + 15) / 16 * 16;
  L.JT = L.r16 / 16;
  L.T = ceil_div(N, int64_t(16));
  L.S = ceil_div(K / kBlock, int64_t(4));
  L.U = L.T * L.S;
  // K parts of the adapter product: at most two 256-wide steps per H warp, at most ~32 H CTAs
  L.HS = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(ceil_div(L.S, int64_t(2 * GV_WARPS)),
                                                                  std::max(1, 32 / L.JT))));
  const int64_t slots = static_cast<int64_t>(GV_CTAS_PER_SM) * device_sm_count() - static_cast<int64_t>(L.JT) * L.HS;
  L.G_max = std::min<int64_t>(L.U, std::max<int64_t>(slots, 1) * GV_WARPS);
  const int64_t lmin = std::max<int64_t>(L.U / L.G_max, 1);   // shortest weight-warp range
  L.P = static_cast<int>(std::min<int64_t>(L.G_max, ceil_div(L.S, lmin) + 1));
  L.fits32 = L.U <= INT32_MAX && N * (K / kBlock) <= INT32_MAX && L.T * L.P * 16 * M <= INT32_MAX;
  size_t off = 0;
  L.off_pieces = off;
  off += align256(static_cast<size_t>(L.T) * L.P * 16 * M * sizeof(float));
  L.off_hpart = off;
  off += align256(static_cast<size_t>(L.JT) * L.HS * 8 * L.NT * 16 * sizeof(float));
  const size_t sh = static_cast<size_t>(8 * L.NT) * L.r16 * sizeof(uint16_t);
  L.off_hi = off;
  off += align256(sh);
  L.off_lo = off;
  off += align256(sh);
  L.off_bar = off;
  off += 256;
  L.total = off;
  return L;
}

// A tag for each launch's barrier word: consecutive from a random start.
uint32_t next_epoch() {
  static std::atomic<uint32_t> next{static_cast<uint32_t>(std::random_device{}())};
  return next.fetch_add(1);
}

template <int NT>
qlora_status launch_gemv_nt(const GemvArgs &a, const GemvLayout &L, cudaStream_t st) {
  char *ws = static_cast<char *>(a.workspace);
  int *status = device_status_ptr();
  if (!status) return QLORA_ERR_CUDA;
  int dev = 0, sms = 0, smem_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess)
    return QLORA_ERR_CUDA;

  const int KB = static_cast<int>(a.wK / kBlock);
  const int64_t xs_bytes = a.M * static_cast<int64_t>(xs_row_bytes(KB));
  const bool xs = xs_bytes <= GV_XS_MAX;
  const int smem = GV_SMEM_BASE + (xs ? static_cast<int>(xs_bytes) : 0);
  auto kern = xs ? gemv_kernel<NT, true> : gemv_kernel<NT, false>;
  const int64_t need = static_cast<int64_t>(GV_CTAS_PER_SM) * (smem + 1024);
  const int pct = static_cast<int>(std::min<int64_t>(100, (need * 100 + smem_sm - 1) / smem_sm));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct) != cudaSuccess)
    return QLORA_ERR_CUDA;
  int occ = 0;   // every CTA must be resident at once (cooperative launch)
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, GV_THREADS, smem) != cudaSuccess || occ < 1)
    return QLORA_ERR_CUDA;
  const int64_t hctas = static_cast<int64_t>(L.JT) * L.HS;
  const int64_t resident = static_cast<int64_t>(std::min(occ, GV_CTAS_PER_SM)) * sms;
  if (resident <= hctas) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int64_t ctas = std::min<int64_t>(hctas + ceil_div(L.U, int64_t(GV_WARPS)), resident);
  const int64_t G = std::min<int64_t>(L.U, (ctas - hctas) * GV_WARPS);
  if (G > L.G_max) return QLORA_ERR_CUDA;   // the piece slots were sized for at most G_max warps

  CUtensorMap tm;   // codes as [N rows][K/2 bytes], boxes of 16 rows x 128 bytes
  if (!make_tmap_2d(&tm, a.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<uint64_t>(a.wK / 2),
                    static_cast<uint64_t>(a.wN), static_cast<uint64_t>(a.wK / 2), 128, 16,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  GemvParams p{a.X, a.absmax_q, a.group_scale, a.A, a.B, a.s, a.Y, a.H_out,
               reinterpret_cast<uint16_t *>(ws + L.off_hi), reinterpret_cast<uint16_t *>(ws + L.off_lo),
               reinterpret_cast<float *>(ws + L.off_pieces), reinterpret_cast<float *>(ws + L.off_hpart),
               reinterpret_cast<unsigned long long *>(ws + L.off_bar), next_epoch(), static_cast<int>(a.M), a.r, L.r16, L.JT, L.HS, static_cast<int>(G), static_cast<int>(L.S),
               static_cast<int>(L.U), static_cast<int>(L.T), L.P, xs ? xs_row_bytes(KB) : 0, a.wN, a.wK, status,
               wait_limit(), a.tab};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(GV_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // launch during the previous kernel's tail
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, tm, p) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}

}  // namespace

bool gemv_enabled() { return true; }

size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) { return gemv_layout(M, N, K, r).total; }

qlora_status launch_gemv(const GemvArgs &a, cudaStream_t st) {
  if (a.M < 1 || a.M > kGemvMaxTokens) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const GemvLayout L = gemv_layout(a.M, a.wN, a.wK, a.r);
  if (!L.fits32) return QLORA_ERR_UNSUPPORTED_SHAPE;
  prof_mark(kProfGemv, true, st);
  const qlora_status s = L.NT == 1 ? launch_gemv_nt<1>(a, L, st) : launch_gemv_nt<2>(a, L, st);
  prof_mark(kProfGemv, false, st);
  if (s != QLORA_OK) return s;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
