// Few-token forward (M <= 16): memory-bound dequant-GEMV.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": every pass expands the 4-bit base to 16-bit as it runs.  With a
// handful of tokens the packed weight stream (0.516 B per weight) is the whole
// cost: the codes stream into shared memory by TMA and are decoded straight
// into tensor-core register fragments.  The decode (a per-block 16-entry bf16
// table and byte permutes) runs on the integer pipe.
//
// One cooperative launch (every CTA resident, so the bounded waits below on
// other CTAs' flags always end).  The weight is cut into units (16-row tile,
// 256-wide K step), numbered tile-major; CTA c takes the contiguous range
// [start(c), start(c+1)) (a closed-form split by cost, see cta_start) and its
// GV_WARPS warps split that range contiguously again.
//   1. H = X A^T is cut into JT S parts (16 adapter rows x one 256-wide K
//      step); CTA c computes parts c, c + G, ... first (their two 16-byte
//      loads of A per thread are the first loads it issues), publishes each
//      under a flag; CTA jt < JT then adds the S parts of adapter tile jt in
//      K order and publishes that tile of H under its own flag.  Those CTAs'
//      weight ranges are shorter by that cost.
//   2. Every warp streams its units (per-warp TMA code ring, constants fetched
//      one unit ahead) and decodes each 64-weight block of two rows into
//      m16n8k16 A fragments (tokens are the 8-column B operand; two column
//      tiles when M > 8).  For every tile it touches it stores its fp32 sum
//      as a piece in the CTA's slot (tile - first tile of the CTA) + warp.
//   3. Each warp stamps its own flag once its pieces are stored and finishes
//      the tiles whose last unit lies in its range: once the tiles of H are
//      in, (s H) B^T on mma.sync (s H as a bf16 hi/lo pair formed from the
//      tiles of H in L2; its loads overlap the wait for the pieces), then the
//      pieces of every CTA on the tile, in CTA order and warp order within a
//      CTA (a fixed order, so results do not depend on timing), waiting only
//      for the flags of the warps holding those pieces (lanes poll in
//      parallel); then bf16 Y.
// Nothing waits before it has published what others wait for, so the waits
// form no cycle.  A flag is published by one thread with a release store after
// a CTA or warp barrier (which orders the other threads' stores before it) and
// read with acquire loads, whose thread then meets the others at a warp or CTA barrier
// before any of them reads what the flag covers.  Flags carry a 64-bit tag unique to the launch (consecutive
// from a random start), so no word needs clearing between launches.
#include <algorithm>
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

// One unit's codes arrive by TMA as a 16-row x 128-byte box (256 codes of each
// of the tile's rows), 128-byte swizzled, into a per-warp ring.
constexpr int GV_STAGE_BYTES = 16 * 128;
#ifndef QLORA_GEMV_STAGES
#define QLORA_GEMV_STAGES 4
#endif
constexpr int GV_STAGES = QLORA_GEMV_STAGES;
constexpr int GV_RING_BYTES = GV_WARPS * GV_STAGES * GV_STAGE_BYTES;
constexpr int GV_BAR_OFFSET = GV_RING_BYTES;               // ring barriers, then the activation barrier
constexpr int GV_MAX_CTAS = 511;                            // CTA starts kept in shared memory
constexpr int GV_START_OFFSET = GV_RING_BYTES + 512;        // int starts[GV_MAX_CTAS + 1]
constexpr int GV_AUX_OFFSET = GV_RING_BYTES + 512 + 2048 + 512;   // H reduction, then s H (hi, lo); 1024-aligned
// Units a warp brings into L2 before the previous kernel's results are waited for
// (its TMA ring asks for the next ones right after the wait; prefetching the
// whole range queues the activation copies behind it: 2 measured best on B200).
#ifndef QLORA_GEMV_PREFETCH_UNITS
#define QLORA_GEMV_PREFETCH_UNITS 2
#endif
constexpr int GV_PREFETCH_UNITS = QLORA_GEMV_PREFETCH_UNITS;
// Weight units a CTA gives up for a part of H and for adding a tile of H (tuned on B200).
#ifndef QLORA_GEMV_PC
#define QLORA_GEMV_PC 1
#endif
#ifndef QLORA_GEMV_HC
#define QLORA_GEMV_HC 3
#endif

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

// Flags between the CTAs of one launch: 64-bit words stamped with the launch's tag.
__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const unsigned long long *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu_u64(unsigned long long *p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Wait (bounded) until *f carries `tag`; false when the bound ran out.
__device__ __forceinline__ bool wait_flag(const unsigned long long *f, uint64_t tag, uint64_t limit) {
  const long long t0 = clock64();
  while (ld_acquire_gpu_u64(f) != tag)
    if (static_cast<uint64_t>(clock64() - t0) > limit) return false;
  return true;
}

struct GemvParams {
  const uint16_t *X;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *A;            // [r, K]
  const uint16_t *B;            // [N, r]
  float s;
  uint16_t *Y;                  // [M, N]
  float *H_out;                 // optional [M, r]
  float *pieces;                // [G][SLOTS][M][16] tile sums, one per warp and tile it touches
  float *hpart;                 // [JT S][8 NT][16] parts of H^T (adapter tile i / S, K step i % S)
  float *hsum;                  // [JT][8 NT][16] tiles of H^T
  unsigned long long *hpflag;   // [JT S] a part of H is stored
  unsigned long long *hflag;    // [JT] a tile of H is stored
  unsigned long long *wflag;    // [G][GV_WARPS] a warp's pieces are stored
  unsigned long long tag;       // this launch's flag value
  int M, r, r16;
  int JT, HP;                   // adapter tiles, parts of H (JT S)
  int pc, hc;                   // weight units a CTA gives up for an H part / for adding a tile of H
  int G;                        // CTAs
  int S, U, T;                  // K steps per tile, units (T S), tiles
  int SLOTS;                    // piece slots per CTA
  int xs_row;                   // row pitch of the activations in shared memory (0: global memory)
  int cs_rows;                  // block constants of up to cs_rows rows per CTA in shared memory (0: none)
  int64_t N, K;
  int *status;
  uint64_t wait_limit;
  Nf4Table tab;
};

// First unit of CTA c (0 <= c <= G): an even split of U + P pc + JT hc units
// of work (P = min(HP, G) CTAs with an H part, JT CTAs adding a tile of H),
// each such CTA's share shortened by pc or hc.  Non-decreasing in c (the host
// keeps pc + hc <= U / G); start(0) = 0, start(G) = U.
__host__ __device__ __forceinline__ int cta_start(int c, int U, int G, int P, int pc, int JT, int hc) {
  const int64_t total = static_cast<int64_t>(U) + static_cast<int64_t>(P) * pc + static_cast<int64_t>(JT) * hc;
  return static_cast<int>(static_cast<int64_t>(c) * total / G - static_cast<int64_t>(c < P ? c : P) * pc -
                          static_cast<int64_t>(c < JT ? c : JT) * hc);
}
__device__ __forceinline__ int cta_start(const GemvParams &p, int c) {
  return cta_start(c, p.U, p.G, min(p.HP, p.G), p.pc, p.JT, p.hc);
}
// Every CTA's first unit, computed once per CTA into shared memory (G + 1 ints).
__device__ __forceinline__ void fill_starts(const GemvParams &p, int *starts) {
  for (int c = threadIdx.x; c <= p.G; c += GV_THREADS) starts[c] = cta_start(p, c);
}
// The CTA whose range holds unit u: the largest c with start(c) <= u.
__device__ __forceinline__ int cta_owner(const int *starts, int G, int u) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (starts[mid] <= u) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}
// Warp w of a CTA with range [a, a + L) starts at a + floor(w L / GV_WARPS); the
// warp whose range holds unit u (a <= u < a + L) is the largest such w.  (U <
// 2^27, so these products fit 32 bits.)
__device__ __forceinline__ int warp_start(int a, int L, int w) { return a + ((w * L) >> 3); }
__device__ __forceinline__ int warp_owner(int a, int L, int u) {
  return static_cast<int>(static_cast<uint32_t>((u - a + 1) * GV_WARPS - 1) / static_cast<uint32_t>(L));
}

// Quantized constants of one unit for rows n0 = 16 t + g and n0 + 8, block 4 step + c.
struct PosConst {
  uint32_t q0, q1;   // 8-bit block constants; bit 8 set for rows past N / blocks past K
  float S0, S1;      // 32-bit group constants
};

// a' of one unit's block, and 0 for the padding units (bit 8 of q set).
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

// Phase 1: part i of H^T (adapter rows j0 = 16 (i / S) .. +15, K step i % S).
// Warp w covers K columns 256 step + 32 w .. +31; thread (g, c) the eight
// columns from +8 c of A rows j0 + g and j0 + g + 8, loaded (16 bytes each)
// before anything else, in the K order the weight uses.
struct HLoad {
  uint4 a, b;
};
__device__ __forceinline__ HLoad h_load(const GemvParams &p, int i) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int j0 = (i / p.S) * 16, step = i - (i / p.S) * p.S;
  const int64_t k = static_cast<int64_t>(step) * 256 + warp * 32 + c * 8;   // a multiple of 8; K % 64 == 0
  const int ja = j0 + g, jb = j0 + g + 8;
  HLoad h;
  h.a = (k < p.K && ja < p.r) ? __ldg(reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(ja) * p.K + k))
                              : make_uint4(0, 0, 0, 0);
  h.b = (k < p.K && jb < p.r) ? __ldg(reinterpret_cast<const uint4 *>(p.A + static_cast<int64_t>(jb) * p.K + k))
                              : make_uint4(0, 0, 0, 0);
  return h;
}

// The part's products (two m16n8k16 steps per warp), the 8 warps added in a
// fixed order, stored and published under the part's flag.
template <int NT, bool XS>
__device__ __forceinline__ void h_part(const GemvParams &p, const XSource<NT, XS> &x, const HLoad &h, int i,
                                       float *red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int step = i - (i / p.S) * p.S;
  const int64_t k = static_cast<int64_t>(step) * 256 + warp * 32 + c * 8;
  const int KB = static_cast<int>(p.K / kBlock);
  const int kb = static_cast<int>(min(k, p.K - 8) / kBlock), w8 = static_cast<int>((min(k, p.K - 8) % kBlock) / 8);
  (void)KB;
  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.0f;
    const uint4 xv = x.load(t, kb, w8);
    mma16816(acc[t], h.a.x, h.b.x, h.a.y, h.b.y, xv.x, xv.y);
    mma16816(acc[t], h.a.z, h.b.z, h.a.w, h.b.w, xv.z, xv.w);
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) red[((warp * NT + t) * 4 + e) * 32 + lane] = acc[t][e];
  __syncthreads();
  if (warp == 0) {
    float *dst = p.hpart + static_cast<int64_t>(i) * 8 * NT * 16;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < GV_WARPS; ++w) v += red[((w * NT + t) * 4 + e) * 32 + lane];
        // C fragment: H^T[j0 + g + 8 (e >> 1)][tok = 8 t + 2 c + (e & 1)]
        [[maybe_unused]] const int64_t o =   // checked in the bounds-checked build only
            static_cast<int64_t>(i) * 8 * NT * 16 + (8 * t + 2 * c + (e & 1)) * 16 + g + 8 * (e >> 1);
        if (QL_IN_BOUNDS(p.status, o, static_cast<int64_t>(p.HP) * 8 * NT * 16))
          __stcg(dst + (8 * t + 2 * c + (e & 1)) * 16 + g + 8 * (e >> 1), v);
      }
    }
  }
  __syncthreads();   // the part is stored (and ordered before the release below), and red is free again
  if (threadIdx.x == 0 && QL_IN_BOUNDS(p.status, i, p.HP)) st_release_gpu_u64(p.hpflag + i, p.tag);
}

// CTA jt < JT: tile jt of H^T, the sum of its S parts in K order, once their
// flags are up (one thread per flag), published under the tile's flag (and
// stored as fp32 H when asked).
template <int NT>
__device__ __forceinline__ void h_tile(const GemvParams &p, int jt) {
  for (int s = threadIdx.x; s < p.S; s += GV_THREADS)
    if (!wait_flag(p.hpflag + jt * p.S + s, p.tag, p.wait_limit)) latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
  __syncthreads();
  const int n = 8 * NT * 16;
  for (int e = threadIdx.x; e < n; e += GV_THREADS) {
    const float *src = p.hpart + static_cast<int64_t>(jt) * p.S * n + e;
    float h = 0.0f;
    for (int s0 = 0; s0 < p.S; s0 += 16) {   // sixteen loads in flight, added in order
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = (s0 + u < p.S && QL_IN_BOUNDS(p.status, (static_cast<int64_t>(jt) * p.S + s0 + u) * n + e,
                                             static_cast<int64_t>(p.HP) * n))
                   ? __ldcg(src + static_cast<int64_t>(s0 + u) * n)
                   : 0.0f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (s0 + u < p.S) h += v[u];
    }
    if (QL_IN_BOUNDS(p.status, jt * n + e, p.JT * n)) __stcg(p.hsum + jt * n + e, h);
    const int tok = e >> 4, j = jt * 16 + (e & 15);
    if (p.H_out && tok < p.M && j < p.r && QL_IN_BOUNDS(p.status, tok * p.r + j, p.M * p.r))
      p.H_out[static_cast<int64_t>(tok) * p.r + j] = h;
  }
  __syncthreads();   // every thread's stores are ordered before the release below
  if (threadIdx.x == 0 && QL_IN_BOUNDS(p.status, jt, p.JT)) st_release_gpu_u64(p.hflag + jt, p.tag);
}

// The code stream of one weight warp: lane 0 keeps GV_STAGES units of the
// warp's range in flight (issue cursor: unit iu = it S + is).
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

// Block constants of a warp's units, one unit ahead in registers.  Rows past
// N and blocks past K read a clamped, valid address and are marked in bit 8 of
// q, so their weights decode to (signed) zero.
// With p.cs_rows > 0 the CTA's constants are in shared memory: the bytes of
// its rows from row r0 = 16 ta on (cq) and the group scales from group g0 on
// (cs), see stage_constants.
struct ConstStream {
  int ft, fs, fu, b;   // cursor: unit fu = ft S + fs; the range ends at b
  const uint8_t *cq;
  const float *cs;
  int r0, g0;
  __device__ __forceinline__ ConstStream(int S, int a, int b_, const uint8_t *cq_, const float *cs_, int r0_, int g0_)
      : ft(a / S), fs(a - (a / S) * S), fu(a), b(b_), cq(cq_), cs(cs_), r0(r0_), g0(g0_) {}
  __device__ __forceinline__ void fetch(const GemvParams &p, PosConst &f) {
    const int lane = threadIdx.x & 31, g = lane >> 2, c = lane & 3;
    const int KB = static_cast<int>(p.K / kBlock);
    const int N = static_cast<int>(p.N);
    const int kb = 4 * fs + c;
    const int kbc = min(kb, KB - 1);
    const int n0 = ft * 16 + g;
    const int bi0 = min(n0, N - 1) * KB + kbc, bi1 = min(n0 + 8, N - 1) * KB + kbc;   // < 2^31 (host check)
    const bool kv = kb < KB;
    if (p.cs_rows > 0) {
      const int o = r0 * KB;
      const int64_t nq = static_cast<int64_t>(p.cs_rows) * KB, ns = nq / 256 + 2;
      (void)nq;
      (void)ns;
      const bool in = QL_IN_BOUNDS(p.status, bi0 - o, nq) && QL_IN_BOUNDS(p.status, bi1 - o, nq) &&
                      QL_IN_BOUNDS(p.status, (bi0 >> 8) - g0, ns) && QL_IN_BOUNDS(p.status, (bi1 >> 8) - g0, ns);
      f.q0 = (in ? static_cast<uint32_t>(cq[bi0 - o]) : 0u) | ((kv && n0 < N) ? 0u : 0x100u);
      f.q1 = (in ? static_cast<uint32_t>(cq[bi1 - o]) : 0u) | ((kv && n0 + 8 < N) ? 0u : 0x100u);
      f.S0 = in ? cs[(bi0 >> 8) - g0] : 0.0f;
      f.S1 = in ? cs[(bi1 >> 8) - g0] : 0.0f;
    } else {
      f.q0 = ldg_once_u8(p.absmax_q + bi0) | ((kv && n0 < N) ? 0u : 0x100u);
      f.q1 = ldg_once_u8(p.absmax_q + bi1) | ((kv && n0 + 8 < N) ? 0u : 0x100u);
      f.S0 = ldg_once_f32(p.group_scale + (bi0 >> 8));
      f.S1 = ldg_once_f32(p.group_scale + (bi1 >> 8));
    }
    if (fu + 1 < b) {   // advance, staying on the last unit of the range
      ++fu;
      if (++fs == p.S) {
        fs = 0;
        ++ft;
      }
    }
  }
};

// Phase 2, warp `warp` of CTA c: units [a, b), the constants of unit a already
// in q (fetched as early as the kernel may read the weight).  The warp's sum
// over its part of each tile it touches is stored, as soon as that part is
// done, in the CTA's piece slot (tile - ta) + warp (ta: the CTA's first tile).
template <int NT, bool XS>
__device__ __forceinline__ void weight_role(const CUtensorMap *tm, const GemvParams &p, const XSource<NT, XS> &x,
                                            CodeStream &cs, ConstStream &cst, PosConst q, int cta, int ta, int a,
                                            int b) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int S = p.S;
  const int KB = static_cast<int>(p.K / kBlock);
  const int first_tile = a / S;
  const float mu = dq_offset(p.tab);

  float acc[NT][4];
#pragma unroll
  for (int tt = 0; tt < NT; ++tt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;

  int t = first_tile, step = a - first_tile * S;
  int ip = 0;   // index of unit u within the range
  for (int u = a; u < b; ++u, ++ip) {
    const PosConst f = q;
    cst.fetch(p, q);

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
    // every lane has used its codes: the slot takes the unit GV_STAGES ahead
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
    // this warp's part of the tile is done: its piece
    const int64_t pbase = (static_cast<int64_t>(cta) * p.SLOTS + (tile - ta) + warp) * 16 * p.M;
    float *pc = p.pieces + pbase;
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int tok = tt * 8 + 2 * c + (e & 1);
        if (tok < p.M &&
            QL_IN_BOUNDS(p.status, pbase + tok * 16 + g + 8 * (e >> 1), static_cast<int64_t>(p.G) * p.SLOTS * 16 * p.M))
          __stcg(pc + tok * 16 + g + 8 * (e >> 1), acc[tt][e]);
      }
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
  }
}

// acc += (s H) B^T for the 16 rows of tile t: the rows of B are the A operand
// (the adapter index j is the reduction index), s H the B operand as a bf16
// pair hi + lo (hi = bf16(s H), lo = bf16(s H - hi)), formed from the tiles of
// H in L2; the loads of four 16-wide adapter steps are issued together.
template <int NT>
__device__ __forceinline__ void add_lora(const GemvParams &p, int t, float (&acc)[NT][4], int lane) {
  const int g = lane >> 2, c = lane & 3;
  const int64_t n0 = static_cast<int64_t>(t) * 16 + g, n1 = n0 + 8;
  const bool v0 = n0 < p.N, v1 = n1 < p.N;
  const uint32_t *B0 = reinterpret_cast<const uint32_t *>(p.B + min(n0, p.N - 1) * p.r);
  const uint32_t *B1 = reinterpret_cast<const uint32_t *>(p.B + min(n1, p.N - 1) * p.r);
  for (int j0 = 0; j0 < p.r; j0 += 64) {
    uint32_t a[4][4];
    float hv[4][NT][4];   // H at token 8 tt + g, adapter indices ja, ja + 1, jb, jb + 1
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
      for (int tt = 0; tt < NT; ++tt) {
        const int tok = tt * 8 + g;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = (i < 2 ? ja : jb) + (i & 1);
          hv[q][tt][i] = (j < p.r && QL_IN_BOUNDS(p.status, ((j >> 4) * 8 * NT + tok) * 16 + (j & 15), p.JT * 8 * NT * 16))
                             ? __ldcg(p.hsum + ((j >> 4) * 8 * NT + tok) * 16 + (j & 15))
                             : 0.0f;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (j0 + 16 * q < p.r) {
#pragma unroll
        for (int tt = 0; tt < NT; ++tt) {
          uint32_t hi[2], lo[2];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const float s0 = __fmul_rn(p.s, hv[q][tt][2 * h2]), s1 = __fmul_rn(p.s, hv[q][tt][2 * h2 + 1]);
            const __nv_bfloat16 b0 = __float2bfloat16_rn(s0), b1 = __float2bfloat16_rn(s1);
            hi[h2] = pack_bf16x2(__bfloat162float(b0), __bfloat162float(b1));
            lo[h2] = pack_bf16x2(__fsub_rn(s0, __bfloat162float(b0)), __fsub_rn(s1, __bfloat162float(b1)));
          }
          mma16816(acc[tt], a[q][0], a[q][1], a[q][2], a[q][3], hi[0], hi[1]);
          mma16816(acc[tt], a[q][0], a[q][1], a[q][2], a[q][3], lo[0], lo[1]);
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
      if (tok < p.M && n < p.N && QL_IN_BOUNDS(p.status, tok * p.N + n, p.M * p.N)) {
        const __nv_bfloat16 y = __float2bfloat16_rn(acc[tt][e]);
        p.Y[static_cast<int64_t>(tok) * p.N + n] = *reinterpret_cast<const uint16_t *>(&y);
      }
    }
  }
}

// Phase 3, per warp: the tiles whose last unit lies in this warp's range
// [aw, bw).  The adapter term comes first (the tiles of H are waited for once
// per warp), then the tile's pieces CTA by CTA (CTA order is K order) and,
// within a CTA, warp by warp, each CTA's after the flags of its warps on the
// tile (lanes poll in parallel).
template <int NT>
__device__ __forceinline__ void finish_tiles(const GemvParams &p, const int *starts, int cta, int aw, int bw) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int S = p.S;
  bool h_ready = false;
  for (int t = aw / S; t <= (bw - 1) / S; ++t) {
    const int last = (t + 1) * S - 1;
    if (last < aw || last >= bw) continue;    // finished by a later warp
    if (!h_ready) {
      for (int i = lane; i < p.JT; i += 32)
        if (!wait_flag(p.hflag + i, p.tag, p.wait_limit)) latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
      __syncwarp();   // orders each lane's acquire before every lane's reads of H
      h_ready = true;
    }
    float acc[NT][4];
#pragma unroll
    for (int tt = 0; tt < NT; ++tt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[tt][e] = 0.0f;
    add_lora<NT>(p, t, acc, lane);   // its loads are in flight while the pieces are waited for
    const int c_first = cta_owner(starts, p.G, t * S);
    for (int cp = c_first; cp <= cta; ++cp) {
      const int ap = starts[cp], bp = starts[cp + 1];
      if (bp <= ap) continue;
      const int Lp = bp - ap, tap = ap / S;
      const int ulo = max(t * S, ap), uhi = min((t + 1) * S, bp) - 1;
      const int w0 = warp_owner(ap, Lp, ulo), w1 = warp_owner(ap, Lp, uhi);
      // lane w polls warp w's flag (this warp's own piece needs none)
      if (lane >= w0 && lane <= w1 && lane < GV_WARPS && !(cp == cta && lane == warp) &&
          warp_start(ap, Lp, lane) != warp_start(ap, Lp, lane + 1) &&
          !wait_flag(p.wflag + cp * GV_WARPS + lane, p.tag, p.wait_limit))
        latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
      __syncwarp();
      // the CTA's pieces of tile t sit in consecutive slots: all loads in flight, then added in warp order
      const float *src = p.pieces + (static_cast<int64_t>(cp) * p.SLOTS + (t - tap)) * 16 * p.M;
      float v[GV_WARPS][NT][4];
#pragma unroll
      for (int w = 0; w < GV_WARPS; ++w) {
        const bool live = w >= w0 && w <= w1 && warp_start(ap, Lp, w) != warp_start(ap, Lp, w + 1);
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tt * 8 + 2 * c + (e & 1);
            v[w][tt][e] = (live && tok < p.M &&
                           QL_IN_BOUNDS(p.status, (static_cast<int64_t>(cp) * p.SLOTS + (t - tap) + w) * 16 * p.M +
                                                      tok * 16 + g + 8 * (e >> 1),
                                        static_cast<int64_t>(p.G) * p.SLOTS * 16 * p.M))
                              ? __ldcg(src + w * 16 * p.M + tok * 16 + g + 8 * (e >> 1))
                              : 0.0f;
          }
      }
#pragma unroll
      for (int w = 0; w < GV_WARPS; ++w) {
        if (w < w0 || w > w1 || warp_start(ap, Lp, w) == warp_start(ap, Lp, w + 1)) continue;
#pragma unroll
        for (int tt = 0; tt < NT; ++tt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[tt][e] += v[w][tt][e];
      }
    }
    store_y<NT>(p, t, acc, lane);
  }
}

// The CTA's block constants into shared memory: the bytes of rows [r0, r1)
// (one bulk copy of the 16-byte-aligned part, counted on `bar`; plain loads for
// the rest) and the group scales g0 .. g1.  r0 = 16 ta is a multiple of 16, so
// the copy starts on a 16-byte boundary.
__device__ __forceinline__ uint32_t constants_bulk_bytes(const GemvParams &p, int r0, int r1) {
  return static_cast<uint32_t>((static_cast<int64_t>(r1 - r0) * (p.K / kBlock)) & ~int64_t(15));
}
__device__ __forceinline__ void stage_constants(const GemvParams &p, uint8_t *cq, float *cs, int r0, int r1, int g0,
                                                int g1, uint64_t *bar) {
  const int KB = static_cast<int>(p.K / kBlock);
  const int64_t o = static_cast<int64_t>(r0) * KB, n = static_cast<int64_t>(r1 - r0) * KB;
  const uint32_t bulk = constants_bulk_bytes(p, r0, r1);
  if (threadIdx.x == 0 && bulk > 0) bulk_load(cq, p.absmax_q + o, bulk, bar);
  if (threadIdx.x < static_cast<int>(n - bulk)) cq[bulk + threadIdx.x] = p.absmax_q[o + bulk + threadIdx.x];
  for (int i = threadIdx.x; i <= g1 - g0; i += GV_THREADS) cs[i] = __ldg(p.group_scale + g0 + i);
}

template <int NT, bool XS>
__global__ void __launch_bounds__(GV_THREADS, GV_CTAS_PER_SM) gemv_kernel(const __grid_constant__ CUtensorMap tm_codes,
                                                          const GemvParams p, int aux_off, int xs_off, int cq_off,
                                                          int cs_off) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  int *starts = reinterpret_cast<int *>(smem + GV_START_OFFSET);
  fill_starts(p, starts);   // read after the first CTA barrier below
  const int a = cta_start(p, cta), b = cta_start(p, cta + 1);
  const int L = b - a;
  const int aw = warp_start(a, L, warp), bw = warp_start(a, L, warp + 1);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + GV_BAR_OFFSET);
  uint64_t *xbar = bars + GV_WARPS * GV_STAGES;
  CodeStream cs{smem + warp * GV_STAGES * GV_STAGE_BYTES, bars + warp * GV_STAGES, aw / p.S, aw - (aw / p.S) * p.S,
                aw};

  // Barriers, and the warp's first units brought into L2, while the kernel
  // before this one may still be running (the weight is not written by it;
  // a prefetch only warms L2, which stays coherent either way).
  if (lane == 0) {
    for (int i = 0; i < GV_STAGES; ++i) mbar_init(&cs.bar[i], 1);
    if (warp == 0) mbar_init(xbar, 1);
    fence_mbar_init();
    int pt = cs.it, ps = cs.is;
    for (int u = aw; u < bw && u < aw + GV_PREFETCH_UNITS; ++u) {
      tma_prefetch_2d(&tm_codes, ps * 128, pt * 16);
      if (++ps == p.S) {
        ps = 0;
        ++pt;
      }
    }
  }
  // The next kernel on the stream may be scheduled once every CTA has passed
  // here; nothing the previous kernel writes is read before its results are visible.
  griddep_launch_dependents();
  griddep_wait();

  // This CTA's first part of H is loaded first (its result is waited for by
  // every tile), then the activations (every warp needs them before its first
  // product), then the first code boxes.
  HLoad hl{};
  if (cta < p.HP) hl = h_load(p, cta);
  const uint32_t xs = smem_addr(smem + xs_off);
  // the CTA's block constants (when they fit) and the activations arrive on xbar
  const int KB = static_cast<int>(p.K / kBlock);
  const int r0 = (a / p.S) * 16, r1 = L > 0 ? static_cast<int>(min(p.N, static_cast<int64_t>((b - 1) / p.S + 1) * 16)) : r0;
  const int g0 = static_cast<int>((static_cast<int64_t>(r0) * KB) >> 8);
  const int g1 = r1 > r0 ? static_cast<int>((static_cast<int64_t>(r1) * KB - 1) >> 8) : g0 - 1;
  uint8_t *cq = smem + cq_off;
  float *csc = reinterpret_cast<float *>(smem + cs_off);
  if (threadIdx.x == 0)   // every byte the copies below bring (possibly none: the phase then ends here)
    mbar_arrive_expect_tx(xbar, (p.cs_rows > 0 ? constants_bulk_bytes(p, r0, r1) : 0u) +
                                    (XS ? static_cast<uint32_t>(p.K * 2 * p.M) : 0u));
  if (p.cs_rows > 0) stage_constants(p, cq, csc, r0, r1, g0, g1, xbar);
  if (XS && threadIdx.x == 0) {
    const uint32_t row = static_cast<uint32_t>(p.K * 2);
    for (int m = 0; m < p.M; ++m)
      bulk_load(smem + xs_off + m * p.xs_row, p.X + static_cast<int64_t>(m) * p.K, row, xbar);
  }
  if (lane == 0)
    for (int i = 0; i < GV_STAGES && cs.iu < bw; ++i) cs.issue(&tm_codes, i, p.S);
  // the rows of B of the tiles this CTA finishes (the adapter term reads them
  // last) are brought into L2 now as well
  ConstStream cst(p.S, aw, bw, cq, csc, r0, g0);
  if (L > 0 && threadIdx.x < 8) {
    const int t = (b - 1) / p.S - static_cast<int>(threadIdx.x);   // a tile of the range, from the last
    const int last = (t + 1) * p.S - 1;
    if (t >= a / p.S && last >= a && last < b) {
      const int64_t rows = min(static_cast<int64_t>(16), p.N - static_cast<int64_t>(t) * 16);
      bulk_prefetch_l2(p.B + static_cast<int64_t>(t) * 16 * p.r, static_cast<uint32_t>(rows * p.r * 2));
    }
  }
  __syncthreads();   // every barrier is initialised, the plain constant loads are in shared memory
  if (!mbar_wait(xbar, 0, p.wait_limit)) latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
  PosConst q0{};
  if (aw < bw) cst.fetch(p, q0);
  const XSource<NT, XS> x(p, xs, lane >> 2);

  for (int i = cta; i < p.HP; i += p.G) {
    if (i != cta) hl = h_load(p, i);
    h_part<NT, XS>(p, x, hl, i, reinterpret_cast<float *>(smem + aux_off));
  }
  if (cta < p.JT) h_tile<NT>(p, cta);
  if (aw >= bw) return;
  weight_role<NT, XS>(&tm_codes, p, x, cs, cst, q0, cta, a / p.S, aw, bw);
  // this warp's pieces are stored: publish them (the warp barrier orders every
  // lane's stores before lane 0's release)
  __syncwarp();
  if (lane == 0 && QL_IN_BOUNDS(p.status, cta * GV_WARPS + warp, p.G * GV_WARPS))
    st_release_gpu_u64(p.wflag + cta * GV_WARPS + warp, p.tag);
  finish_tiles<NT>(p, starts, cta, aw, bw);
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
// The piece slots are sized for the longest CTA range of a launch with one CTA
// per SM (more CTAs only shorten the ranges), and the per-CTA arrays for the
// most CTAs a launch can have, so the layout does not depend on the occupancy
// found at launch.
struct GemvLayout {
  int NT, r16, JT, G_max, SLOTS;
  int64_t T, S, U, HP;
  bool ok;
  size_t off_pieces, off_hpart, off_hsum, off_hpflag, off_hflag, off_wflag, total;
};

GemvLayout gemv_layout(int64_t M, int64_t N, int64_t K, int r) {
  GemvLayout L{};
  L.NT = M <= 8 ? 1 : 2;
  L.r16 = (r + 15) / 16 * 16;
  L.JT = L.r16 / 16;
  L.T = ceil_div(N, int64_t(16));
  L.S = ceil_div(K / kBlock, int64_t(4));
  L.U = L.T * L.S;
  L.HP = static_cast<int64_t>(L.JT) * L.S;   // parts of H
  const int sms = device_sm_count();
  L.G_max = GV_CTAS_PER_SM * sms;
  const int64_t g_min = sms;   // fewest CTAs a launch runs with (one per SM)
  L.ok = g_min > L.JT && L.G_max <= GV_MAX_CTAS && L.U < (int64_t(1) << 27) && L.HP <= INT32_MAX &&
         N * (K / kBlock) <= INT32_MAX;
  if (!L.ok) return L;
  // longest CTA range at g_min CTAs or more: at most ceil(total / G) with total <=
  // U + G pc + JT hc (pc, hc as the launch sets them)
  const int64_t maxlen = ceil_div(L.U + static_cast<int64_t>(L.JT) * (QLORA_GEMV_HC + L.S / 16), g_min) + QLORA_GEMV_PC;
  L.SLOTS = static_cast<int>(ceil_div(maxlen, L.S) + 1 + (GV_WARPS - 1));
  L.ok = static_cast<int64_t>(L.G_max) * L.SLOTS * 16 * M <= INT32_MAX;
  size_t off = 0;
  L.off_pieces = off;
  off += align256(static_cast<size_t>(L.G_max) * L.SLOTS * 16 * M * sizeof(float));
  L.off_hpart = off;
  off += align256(static_cast<size_t>(L.HP) * 8 * L.NT * 16 * sizeof(float));
  L.off_hsum = off;
  off += align256(static_cast<size_t>(L.JT) * 8 * L.NT * 16 * sizeof(float));
  L.off_hpflag = off;
  off += align256(static_cast<size_t>(L.HP) * sizeof(unsigned long long));
  L.off_hflag = off;
  off += align256(static_cast<size_t>(L.JT) * sizeof(unsigned long long));
  L.off_wflag = off;
  off += align256(static_cast<size_t>(L.G_max) * GV_WARPS * sizeof(unsigned long long));
  L.total = off;
  return L;
}

// A tag for each launch's flags: consecutive from a random 64-bit start.
uint64_t next_tag() {
  static std::atomic<uint64_t> next{(static_cast<uint64_t>(std::random_device{}()) << 32) ^ std::random_device{}()};
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
  // shared memory: ring, barriers and CTA starts, the H reduction, then (when they
  // fit the per-CTA budget) the CTA's block constants and the activations
  const int aux = GV_WARPS * NT * 4 * 32 * 4;
  const int xs_off = GV_AUX_OFFSET + aux;
  const int budget = smem_sm / GV_CTAS_PER_SM - 1024 - 1024;   // per-CTA reserve and alignment slack
  const int cs_rows = 16 * (L.SLOTS - (GV_WARPS - 1));          // rows of the most tiles a CTA touches
  const int64_t cq_bytes = (static_cast<int64_t>(cs_rows) * KB + 15) / 16 * 16 + 16;
  const int64_t cs_bytes = ((static_cast<int64_t>(cs_rows) * KB / 256 + 2) * 4 + 15) / 16 * 16;
  const bool cs_on = xs_off + cq_bytes + cs_bytes <= budget;
  const int64_t c_total = cs_on ? cq_bytes + cs_bytes : 0;
  const int64_t xs_bytes = a.M * static_cast<int64_t>(xs_row_bytes(KB));
  const bool xs = xs_off + c_total + xs_bytes <= budget;
  const int cq_off = xs_off + (xs ? static_cast<int>(xs_bytes) : 0);
  const int cs_off = cq_off + (cs_on ? static_cast<int>(cq_bytes) : 0);
  const int smem = static_cast<int>(cq_off + c_total) + 1024;
  auto kern = xs ? gemv_kernel<NT, true> : gemv_kernel<NT, false>;
  const int64_t need = static_cast<int64_t>(GV_CTAS_PER_SM) * (smem + 1024);
  const int pct = static_cast<int>(std::min<int64_t>(100, (need * 100 + smem_sm - 1) / smem_sm));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, pct) != cudaSuccess)
    return QLORA_ERR_CUDA;
  int occ = 0;   // every CTA must be resident at once (cooperative launch)
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, GV_THREADS, smem) != cudaSuccess || occ < 1)
    return QLORA_ERR_CUDA;
  const int G = std::min(occ, GV_CTAS_PER_SM) * sms;
  if (G > L.G_max || G <= L.JT) return QLORA_ERR_UNSUPPORTED_SHAPE;
  // weight units given up for a part of H (one round trip for 16 bytes of A per thread)
  // and for adding a tile of H (waiting for its parts, S loads per element), capped so
  // the CTA ranges stay ordered
  const int64_t per = L.U / G;
  const int64_t pc = std::min<int64_t>(QLORA_GEMV_PC, per);
  const int64_t hc = std::min<int64_t>(QLORA_GEMV_HC + L.S / 16, per - pc);

  CUtensorMap tm;   // codes as [N rows][K/2 bytes], boxes of 16 rows x 128 bytes
  if (!make_tmap_2d(&tm, a.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<uint64_t>(a.wK / 2),
                    static_cast<uint64_t>(a.wN), static_cast<uint64_t>(a.wK / 2), 128, 16,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  GemvParams p{};
  p.X = a.X;
  p.absmax_q = a.absmax_q;
  p.group_scale = a.group_scale;
  p.A = a.A;
  p.B = a.B;
  p.s = a.s;
  p.Y = a.Y;
  p.H_out = a.H_out;
  p.pieces = reinterpret_cast<float *>(ws + L.off_pieces);
  p.hpart = reinterpret_cast<float *>(ws + L.off_hpart);
  p.hsum = reinterpret_cast<float *>(ws + L.off_hsum);
  p.hpflag = reinterpret_cast<unsigned long long *>(ws + L.off_hpflag);
  p.hflag = reinterpret_cast<unsigned long long *>(ws + L.off_hflag);
  p.wflag = reinterpret_cast<unsigned long long *>(ws + L.off_wflag);
  p.tag = next_tag();
  p.M = static_cast<int>(a.M);
  p.r = a.r;
  p.r16 = L.r16;
  p.JT = L.JT;
  p.HP = static_cast<int>(L.HP);
  p.pc = static_cast<int>(pc);
  p.G = G;
  p.S = static_cast<int>(L.S);
  p.U = static_cast<int>(L.U);
  p.T = static_cast<int>(L.T);
  p.SLOTS = L.SLOTS;
  p.hc = static_cast<int>(hc);
  p.xs_row = xs ? xs_row_bytes(KB) : 0;
  p.cs_rows = cs_on ? cs_rows : 0;
  p.N = a.wN;
  p.K = a.wK;
  p.status = status;
  p.wait_limit = wait_limit();
  p.tab = a.tab;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
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
  if (cudaLaunchKernelEx(&cfg, kern, tm, p, GV_AUX_OFFSET, xs_off, cq_off, cs_off) != cudaSuccess)
    return QLORA_ERR_CUDA;
  return QLORA_OK;
}

}  // namespace

bool gemv_enabled() { return true; }

size_t gemv_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  const GemvLayout L = gemv_layout(M, N, K, r);
  return L.ok ? L.total : 256;
}

qlora_status launch_gemv(const GemvArgs &a, cudaStream_t st) {
  if (a.M < 1 || a.M > kGemvMaxTokens) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const GemvLayout L = gemv_layout(a.M, a.wN, a.wK, a.r);
  if (!L.ok) return QLORA_ERR_UNSUPPORTED_SHAPE;
  prof_mark(kProfGemv, true, st);
  const qlora_status s = L.NT == 1 ? launch_gemv_nt<1>(a, L, st) : launch_gemv_nt<2>(a, L, st);
  prof_mark(kProfGemv, false, st);
  if (s != QLORA_OK) return s;
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
