// Adapter (low-rank) products on 5th-generation tensor cores.
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": small trainable low-rank adapters beside the frozen base; only they
// receive gradients.  With X [M,K], dY [M,N], A [r,K], B [N,r]:
//   H  = X A^T            C[i=m, j]  = sum_k X[m,k] A[j,k]     (A K-major, B K-major)
//   G  = dY B             C[i=m, j]  = sum_n dY[m,n] B[n,j]    (A K-major, B MN-major)
//   dB = dY^T [H_hi|H_lo] C[i=n, j]  = sum_m dY[m,n] Hs[m,j]   (A MN-major, B MN-major)
//   dA = [G_hi|G_lo]^T X  C[i=j, k]  = sum_m Gs[m,j] X[m,k]    (A MN-major, B MN-major)
// One CTA computes a 128 x BN tile (BN = 64 .. 256) over one slice of the
// reduction, staged by TMA in 64-deep steps into a ring of up to 8 stages
// (128B swizzle, K-major or MN-major as the operand is stored), issued by one
// thread as tcgen05.mma (M = 128) into TMEM.  The Z slices of one tile run as
// a thread-block cluster and finish it in the kernel: the epilogue warps write
// the accumulator from TMEM to the slice's row-major fp32 partial tile in the
// workspace (through shared memory, so the stores are 128-byte row runs; the
// tile stays in L2), one cluster barrier orders those writes, and CTA q
// then reads the output rows q*per .. of all Z partial tiles, adds them in
// slice order and applies the epilogue (scale, bf16, hi/lo split, the halves
// of a stacked operand) with 16-byte stores.  The exchange goes through L2
// rather than distributed shared memory, whose SM-to-SM bandwidth is several
// times lower.  When a tile cannot finish in its cluster the kernel writes
// fp32 partial sums part[z][i][j] instead and a second kernel adds them in the
// same fixed order.  A launch may carry two products with the same operand
// layouts and split count (dB and dA): blocks x < x_split take the first.
#include "internal.h"

namespace qlora {

namespace {

constexpr int TBM = 128;
constexpr int TBN_MAX = 256;
constexpr int TBK = 64;
constexpr int TMAX_STAGES = 8;
constexpr int TA_BYTES = TBM * TBK * 2;         // 16 KB
#ifndef QLORA_TC_RING_KB
#define QLORA_TC_RING_KB 104
#endif
constexpr int TRING_BYTES = QLORA_TC_RING_KB * 1024;   // stages (104 KB: two CTAs per SM)
constexpr int TCTAS_PER_SM = TRING_BYTES > 110 * 1024 ? 1 : 2;
constexpr int TTHREADS = 192;                   // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int TSMEM = TRING_BYTES + 1024 + 256;

// Stage = A tile (16 KB) + B tile (bn x 64 bf16); as many stages as fit in the ring.
__host__ __device__ constexpr int t_stage_bytes(int bn) { return TA_BYTES + bn * TBK * 2; }
__host__ __device__ constexpr int t_stages(int bn) {
  return TRING_BYTES / t_stage_bytes(bn) > TMAX_STAGES ? TMAX_STAGES : TRING_BYTES / t_stage_bytes(bn);
}
constexpr uint64_t kTDrain = 4000000000ull;
constexpr int kMaxZ = 8;        // most slices of one tile (the portable cluster size)

// One product of a launch.
struct TJob {
  int64_t I, J, Kred, kps;
  int bn;              // N of the MMA (multiple of 64, <= 256)
  int gx;              // tiles along I: tile t is i-tile t % gx, j-tile t / gx
  int pw;              // columns of a fused partial tile: min(bn, J)
  float *part;         // fused: [tile][slice][128 x pw] row-major; else [slice][I][J]
  SkinnyEpilogue ep;
};
struct TParams {
  TJob job[2];         // blocks with blockIdx.x < x_split run job 0, the others job 1
  int x_split;
  int *status;
  uint64_t wait_limit;
};

struct TSmem {
  uint64_t full[TMAX_STAGES];
  uint64_t empty[TMAX_STAGES];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool t_wait(uint64_t *bar, uint32_t parity, const TParams &p, TSmem *sm) {
  const uint32_t a = smem_addr(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = clock64();
  volatile int *abort_flag = &sm->abort_flag;
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > p.wait_limit) {
      *abort_flag = 1;
      latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ uint16_t t_bf16(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float t_bf16_val(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }
__device__ __forceinline__ uint2 t_bf16x4(float a, float b, float c, float d) {
  return make_uint2(static_cast<uint32_t>(t_bf16(a)) | (static_cast<uint32_t>(t_bf16(b)) << 16),
                    static_cast<uint32_t>(t_bf16(c)) | (static_cast<uint32_t>(t_bf16(d)) << 16));
}
// hi = bf16(x), lo = bf16(x - hi), four at a time
__device__ __forceinline__ void t_hilo4(const float (&x)[4], uint2 &hi, uint2 &lo) {
  uint16_t h[4];
  float l[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    h[c] = t_bf16(x[c]);
    l[c] = __fsub_rn(x[c], t_bf16_val(h[c]));
  }
  hi = make_uint2(h[0] | (static_cast<uint32_t>(h[1]) << 16), h[2] | (static_cast<uint32_t>(h[3]) << 16));
  lo = t_bf16x4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// How a tile's output rows are shared among the Z slices of its cluster: CTA
// q finishes output rows q*per .. q*per + rows_of(q) - 1.  For the stacked-rows
// kind (dA) output row o gathers tile rows o and o + half.
struct SliceMap {
  int Z, per, trows, half;
  bool stacked;
  __host__ __device__ SliceMap(int kind, int64_t I, int z_count) {
    Z = z_count;
    stacked = kind == kSkinnyRows;
    half = static_cast<int>(I / 2);
    trows = stacked ? half : TBM;
    per = (trows + Z - 1) / Z;
  }
  __host__ __device__ int rows_of(int q) const {
    const int n = trows - q * per;
    return n < 0 ? 0 : (n > per ? per : n);
  }
};

// Float index of element (row, 4-column group c4) of a row-major 128 x pw
// partial tile.
__device__ __forceinline__ int64_t part_index(int row, int c4, int pw) {
  return static_cast<int64_t>(row) * pw + 4 * c4;
}

// This warp's 32 accumulator rows (tile rows quarter * 32 .., from TMEM) into
// its slice's row-major partial tile: each 32-column chunk goes through a
// padded shared-memory buffer (stage, 32 x 36 floats, conflict-free both ways)
// so that the global stores are 128-byte row runs.
__device__ __forceinline__ void write_partial(const TJob &jb, float *pt, uint32_t tmem, uint32_t stage,
                                              int quarter, int lane, bool live, int cw) {
  constexpr int SP = 36;   // staged row pitch (floats)
  for (int cc = 0; cc * 32 < cw; ++cc) {
    uint32_t v[32];
    if (live) {
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + cc * 32, v);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0u;   // aborted slice: zero
    }
#pragma unroll
    for (int q4 = 0; q4 < 8; ++q4)
      st_shared_v4(stage + static_cast<uint32_t>((lane * SP + 4 * q4) * 4), v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2],
                   v[4 * q4 + 3]);
    __syncwarp();
    const int ncol4 = (cw - cc * 32) < 32 ? (cw - cc * 32) / 4 : 8;   // 4-column groups of this chunk
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = k * 4 + lane / 8, c4 = lane % 8;   // 4 rows x 8 groups per instruction
      if (c4 < ncol4) {
        const uint4 x = ld_shared_v4(stage + static_cast<uint32_t>((r * SP + 4 * c4) * 4));
        *reinterpret_cast<uint4 *>(pt + part_index(quarter * 32 + r, cc * 8 + c4, jb.pw)) = x;
      }
    }
    __syncwarp();
  }
}

// Outputs of one item: 4 consecutive columns (gj ..) of output row gi.
__device__ __forceinline__ void store4(const SkinnyEpilogue &ep, int kind, int64_t J, int half_j, int64_t gi,
                                       int64_t gj, int orow, const float (&v)[4]) {
  if (kind == kSkinnyH) {
    const int64_t idx = gi * J + gj;
    *reinterpret_cast<float4 *>(ep.out_f + idx) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<uint2 *>(ep.out_b + idx) =
        t_bf16x4(__fmul_rn(ep.s, v[0]), __fmul_rn(ep.s, v[1]), __fmul_rn(ep.s, v[2]), __fmul_rn(ep.s, v[3]));
    if (ep.out_hl) {
      uint2 hi, lo;
      t_hilo4(v, hi, lo);
      *reinterpret_cast<uint2 *>(ep.out_hl + gi * 2 * J + gj) = hi;
      *reinterpret_cast<uint2 *>(ep.out_hl + gi * 2 * J + J + gj) = lo;
    }
  } else if (kind == kSkinnyG) {
    const float g[4] = {__fmul_rn(ep.s, v[0]), __fmul_rn(ep.s, v[1]), __fmul_rn(ep.s, v[2]), __fmul_rn(ep.s, v[3])};
    uint2 hi, lo;
    t_hilo4(g, hi, lo);
    *reinterpret_cast<uint2 *>(ep.out_b + gi * J + gj) = hi;
    *reinterpret_cast<uint2 *>(ep.out_hl + gi * 2 * J + gj) = hi;
    *reinterpret_cast<uint2 *>(ep.out_hl + gi * 2 * J + J + gj) = lo;
  } else if (kind == kSkinnyCols) {
    *reinterpret_cast<float4 *>(ep.out_f + gi * half_j + gj) =
        make_float4(__fmul_rn(ep.s, v[0]), __fmul_rn(ep.s, v[1]), __fmul_rn(ep.s, v[2]), __fmul_rn(ep.s, v[3]));
  } else {   // kSkinnyRows
    *reinterpret_cast<float4 *>(ep.out_f + static_cast<int64_t>(orow) * J + gj) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// CTA z of the cluster, after every slice's partial tile is written: add its
// output rows over the Z (<= ZMAX) partial tiles in slice order and write the
// kind's outputs.  An item is CW (4 or 8) consecutive columns of one output
// row; consecutive threads take consecutive items of a row, so the partial
// loads and the output stores are contiguous runs, and every slice's loads of
// an item (at most 16 x 16 bytes) are in flight before the adds.  PAIRED: the
// stacked kinds, which add a second element per slice (dB: column + J/2; dA:
// row + I/2).
template <int ZMAX, bool PAIRED, int CW>
__device__ __forceinline__ void finish_rows(const TJob &jb, const SliceMap &map, int z, const float *tiles,
                                            int64_t i0, int64_t j0) {
  constexpr int NV = CW / 4;   // float4 per item and slice
  const SkinnyEpilogue &ep = jb.ep;
  const int kind = ep.kind;
  const int64_t J = jb.J;
  const int half_j = static_cast<int>(J / 2);
  const int pw = jb.pw;
  const int64_t slice_floats = static_cast<int64_t>(TBM) * pw;
  // columns this kind produces (a multiple of 8 for every fused kind: r % 8 == 0, K % 64 == 0)
  const int tcols = kind == kSkinnyCols ? half_j : static_cast<int>(J - j0 < jb.bn ? J - j0 : jb.bn);
  const int tcw = tcols / CW;
  const int n = map.rows_of(z) * tcw;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int lr = e / tcw, col = (e - lr * tcw) * CW;
    const int orow = z * map.per + lr;            // output row within the tile
    const int64_t gi = i0 + orow;
    if (kind != kSkinnyRows && gi >= jb.I) continue;
    const int64_t ia = part_index(orow, col / 4, pw);
    const int64_t ib = !PAIRED ? ia : kind == kSkinnyCols ? part_index(orow, (col + half_j) / 4, pw)
                                                          : part_index(orow + map.half, col / 4, pw);
    float4 a[ZMAX][NV], b[PAIRED ? ZMAX : 1][NV];
#pragma unroll
    for (int zz = 0; zz < ZMAX; ++zz) {
      if (zz < map.Z) {
#pragma unroll
        for (int u = 0; u < NV; ++u) {
          a[zz][u] = __ldcg(reinterpret_cast<const float4 *>(tiles + zz * slice_floats + ia) + u);
          if (PAIRED) b[PAIRED ? zz : 0][u] = __ldcg(reinterpret_cast<const float4 *>(tiles + zz * slice_floats + ib) + u);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < NV; ++u) {
      float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
      for (int zz = 0; zz < ZMAX; ++zz) {   // slice order: fixed, so the result is deterministic
        if (zz < map.Z) {
          const float av[4] = {a[zz][u].x, a[zz][u].y, a[zz][u].z, a[zz][u].w};
          if (PAIRED) {
            const float4 bb = b[PAIRED ? zz : 0][u];
            const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = __fadd_rn(v[c], __fadd_rn(av[c], bv[c]));
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) v[c] = __fadd_rn(v[c], av[c]);
          }
        }
      }
      store4(ep, kind, J, half_j, gi, j0 + col + 4 * u, orow, v);
    }
  }
}

// G's side output, independent of the reduction: [hi | lo] of the saved fp32
// H for this CTA's output rows, written by the epilogue warps while the main
// loop runs (thread t of nt).
__device__ __forceinline__ void split_aux_rows(const TJob &jb, const SliceMap &map, int z, int64_t i0, int t,
                                               int nt) {
  const SkinnyEpilogue &ep = jb.ep;
  const int64_t J = jb.J;
  const int tc4 = static_cast<int>(J / 4);
  const int n4 = map.rows_of(z) * tc4;
  for (int e4 = t; e4 < n4; e4 += nt) {
    const int lr = e4 / tc4, c4 = e4 - lr * tc4;
    const int64_t gi = i0 + z * map.per + lr;
    if (gi >= jb.I) continue;
    const float4 h4 = __ldg(reinterpret_cast<const float4 *>(ep.aux + gi * J + 4 * c4));
    const float h[4] = {h4.x, h4.y, h4.z, h4.w};
    uint2 hi, lo;
    t_hilo4(h, hi, lo);
    *reinterpret_cast<uint2 *>(ep.aux_hl + gi * 2 * J + 4 * c4) = hi;
    *reinterpret_cast<uint2 *>(ep.aux_hl + gi * 2 * J + J + 4 * c4) = lo;
  }
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TTHREADS, TCTAS_PER_SM)   // the split plan counts on this many CTAs per SM
    lora_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
                   const __grid_constant__ TParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TSmem *sm = reinterpret_cast<TSmem *>(smem + TRING_BYTES);
  const bool second = static_cast<int>(blockIdx.x) >= p.x_split;
  const TJob &jb = second ? p.job[1] : p.job[0];
  const CUtensorMap *tmA = second ? &tmA1 : &tmA0;
  const CUtensorMap *tmB = second ? &tmB1 : &tmB0;
  const int tile = static_cast<int>(blockIdx.x) - (second ? p.x_split : 0);
  const int bn = jb.bn;
  const int nstages = t_stages(bn);
  const int stage_bytes = t_stage_bytes(bn);     // a multiple of 8 KB
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i0 = static_cast<int64_t>(tile % jb.gx) * TBM;
  const int64_t j0 = static_cast<int64_t>(tile / jb.gx) * bn;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.z) * jb.kps;
  const int64_t kend = (kbeg + jb.kps < jb.Kred) ? kbeg + jb.kps : jb.Kred;
  const int nsteps = kend > kbeg ? static_cast<int>((kend - kbeg + TBK - 1) / TBK) : 0;
  const bool fused = jb.ep.kind != kSkinnyPartial;
  // the cluster is the tile's slices: Z = gridDim.z, this CTA is slice z
  const int Z = fused ? static_cast<int>(gridDim.z) : 1;
  const int z = fused ? static_cast<int>(blockIdx.z) : 0;
  const SliceMap map(jb.ep.kind, jb.I, Z);

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->acc_full, 1);
    sm->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmB);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, TBN_MAX);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  // The next kernel on the stream may be scheduled once every CTA of this grid
  // has passed here (so it never takes a slot one of these still needs); no
  // global memory is touched before the previous kernel's writes are visible.
  griddep_launch_dependents();
  // The first stages' tiles into L2 while the previous kernel finishes (a
  // prefetch changes no data and L2 is where writes become visible, so it
  // cannot observe a stale value).
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < nstages && i < nsteps; ++i) {
      const int k0 = static_cast<int>(kbeg + static_cast<int64_t>(i) * TBK);
      if (A_MN) {
        tma_prefetch_2d(tmA, static_cast<int>(i0), k0);
        tma_prefetch_2d(tmA, static_cast<int>(i0) + 64, k0);
      } else {
        tma_prefetch_2d(tmA, k0, static_cast<int>(i0));
      }
      if (B_MN) {
        for (int b = 0; b < bn / 64; ++b) tma_prefetch_2d(tmB, static_cast<int>(j0) + 64 * b, k0);
      } else {
        tma_prefetch_2d(tmB, k0, static_cast<int>(j0));
      }
    }
  }
  griddep_wait();

  bool acc_ok = true;
  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      const uint32_t b_bytes = static_cast<uint32_t>(bn) * TBK * 2;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % nstages;
        const uint32_t ph = (i / nstages) & 1;
        if (i >= nstages && !t_wait(&sm->empty[s], ph ^ 1, p, sm)) break;
        uint8_t *sa = smem + s * stage_bytes;
        uint8_t *sb = sa + TA_BYTES;
        const int k0 = static_cast<int>(kbeg + static_cast<int64_t>(i) * TBK);
        mbar_arrive_expect_tx(&sm->full[s], TA_BYTES + b_bytes);
        if (A_MN) {
          tma_load_2d(sa, tmA, &sm->full[s], static_cast<int>(i0), k0);
          tma_load_2d(sa + 8192, tmA, &sm->full[s], static_cast<int>(i0) + 64, k0);
        } else {
          tma_load_2d(sa, tmA, &sm->full[s], k0, static_cast<int>(i0));
        }
        if (B_MN) {
          for (int b = 0; b < bn / 64; ++b)
            tma_load_2d(sb + 8192 * b, tmB, &sm->full[s], static_cast<int>(j0) + 64 * b, k0);
        } else {
          tma_load_2d(sb, tmB, &sm->full[s], k0, static_cast<int>(j0));
        }
        issued = i + 1;
      }
      for (int j = (issued > nstages ? issued - nstages : 0); j < issued; ++j)
        mbar_wait(&sm->full[j % nstages], (j / nstages) & 1, kTDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TBM, bn, A_MN ? 1 : 0, B_MN ? 1 : 0);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % nstages;
        if (!t_wait(&sm->full[s], (i / nstages) & 1, p, sm)) break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + s * stage_bytes);
        const uint32_t b_base = a_base + TA_BYTES;
        for (int kk = 0; kk < TBK / 16; ++kk) {
          const uint64_t ad = A_MN ? sdesc_sw128(a_base + kk * 2048, 8192, 1024) : sdesc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? sdesc_sw128(b_base + kk * 2048, 8192, 1024) : sdesc_sw128(b_base + kk * 32, 16, 1024);
          tc_mma_bf16(tmem, ad, bd, idesc, (i | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&sm->empty[s]);
      }
      tc_commit(&sm->acc_full);
    }
  } else {
    if (fused && jb.ep.kind == kSkinnyG && jb.ep.aux)
      split_aux_rows(jb, map, z, i0, static_cast<int>(threadIdx.x) - 64, TTHREADS - 64);
    // epilogue warps: the accumulator is complete (and the ring no longer read by the MMAs)
    acc_ok = mbar_wait(&sm->acc_full, 0, kTDrain);
    tc_fence_after();
  }
  __syncwarp();
  volatile int *abort_flag = &sm->abort_flag;
  if (fused) {
    float *tiles = jb.part + static_cast<int64_t>(tile) * Z * TBM * jb.pw;   // this tile's Z partial tiles
    if (warp >= 2) {
      const bool live = __all_sync(0xffffffffu, acc_ok && *abort_flag == 0 && nsteps > 0);
      const int cw = static_cast<int>(jb.J - j0 < bn ? jb.J - j0 : bn);
      // staging: 4.5 KB per epilogue warp at the start of the ring (free: the MMAs are done)
      const uint32_t stage = smem_addr(smem) + static_cast<uint32_t>((warp - 2) * 32 * 36 * 4);
      write_partial(jb, tiles + static_cast<int64_t>(z) * TBM * jb.pw, tmem, stage, warp & 3, lane, live, cw);
    }
    // every slice of the tile has written its partial tile
    cluster_arrive_release();
    cluster_wait_acquire();
    if (A_MN && B_MN) {   // dB, dA (stacked operands)
      if (Z <= 4)
        finish_rows<4, true, 8>(jb, map, z, tiles, i0, j0);
      else
        finish_rows<8, true, 4>(jb, map, z, tiles, i0, j0);
    } else {              // H, G
      finish_rows<8, false, 8>(jb, map, z, tiles, i0, j0);
    }
  } else if (warp >= 2) {
    const int quarter = warp & 3;
    if (__all_sync(0xffffffffu, acc_ok && *abort_flag == 0 && nsteps > 0)) {
      const int64_t row = i0 + quarter * 32 + lane;
      float *out = jb.part + static_cast<int64_t>(blockIdx.z) * jb.I * jb.J + row * jb.J;
      for (int cc = 0; cc < bn / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + cc * 32, v);
        tmem_ld_wait();
        const int64_t c0 = j0 + cc * 32;
        if (row < jb.I) {
          if (c0 + 32 <= jb.J && (jb.J & 3) == 0) {
            float4 *dst = reinterpret_cast<float4 *>(out + c0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                    __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          } else {
            for (int e = 0; e < 32; ++e)
              if (c0 + e < jb.J) out[c0 + e] = __uint_as_float(v[e]);
          }
        }
      }
    } else if (nsteps == 0 && i0 < jb.I) {
      // empty reduction slice: its partial sums are zero
      const int64_t row = i0 + quarter * 32 + lane;
      if (row < jb.I) {
        float *out = jb.part + static_cast<int64_t>(blockIdx.z) * jb.I * jb.J + row * jb.J;
        for (int64_t c = j0; c < j0 + bn && c < jb.J; ++c) out[c] = 0.0f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TBN_MAX);
  }
}

}  // namespace

namespace {
constexpr int kMaxSkinnyCluster = kMaxZ;   // portable cluster size
// Tile width: the whole J up to 128 columns.  Wider matrices (dA, J = K) take
// 128-column tiles: twice the tiles of 256-column ones, so more of the
// machine at the same number of splits, and the staged tile of a cluster
// epilogue still fits the ring.
int64_t tc_bn(int64_t J) {
  const int64_t b = ceil_div(J, 64) * 64;
  return b > 128 ? 128 : b;
}
}  // namespace

namespace {
int64_t skinny_tiles(int64_t I, int64_t J) {
  const int64_t t = ceil_div(I, TBM) * ceil_div(J, tc_bn(J));
  return t < 1 ? 1 : t;
}
// Clusters of z CTAs that are co-resident: a cluster sits in one GPC, so each
// of the 8 GPCs (at least 18 SMs, TCTAS_PER_SM CTAs per SM) holds
// floor(36 / z) of them (32 clusters of 8 measured on B200).  A fixed bound,
// so that workspace sizes do not depend on the device a query runs on.
int64_t coresident_clusters(int64_t z) { return 8 * ((18 * TCTAS_PER_SM) / z); }

// Splits of the reduction for `tiles` tiles sharing one launch: every split of
// every tile in one wave of co-resident clusters, at least four 64-deep steps
// per split, at most a portable cluster.
void plan_splits(int64_t tiles, int64_t Kred, int *splits, int64_t *k_per_split) {
  if (Kred < 1) Kred = 1;
  int64_t sp = 148 * TCTAS_PER_SM / tiles;
  const int64_t max_sp = Kred / (4 * TBK) > 0 ? Kred / (4 * TBK) : 1;
  if (sp > max_sp) sp = max_sp;
  if (sp > kMaxSkinnyCluster) sp = kMaxSkinnyCluster;   // the splits of a tile form one cluster
  while (sp > 1 && tiles > coresident_clusters(sp)) --sp;
  if (sp < 1) sp = 1;
  const int64_t kps = ceil_div(ceil_div(Kred, sp), TBK) * TBK;
  *splits = static_cast<int>(ceil_div(Kred, kps));
  *k_per_split = kps;
}

bool fill_job(const SkinnyArgs &a, TJob &j, CUtensorMap &tmA, CUtensorMap &tmB) {
  const int64_t bn = tc_bn(a.J);
  bool ok;
  if (a.a_kmajor)
    ok = make_tmap_2d(&tmA, a.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Kred, a.I, a.lda * 2, TBK, TBM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = make_tmap_2d(&tmA, a.A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.I, a.Kred, a.lda * 2, 64, TBK,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (a.b_kmajor)
    ok = ok && make_tmap_2d(&tmB, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Kred, a.J, a.ldb * 2, TBK,
                            static_cast<uint32_t>(bn), CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_tmap_2d(&tmB, a.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.J, a.Kred, a.ldb * 2, 64, TBK,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  j.I = a.I;
  j.J = a.J;
  j.Kred = a.Kred;
  j.kps = a.k_per_split;
  j.bn = static_cast<int>(bn);
  j.gx = static_cast<int>(ceil_div(a.I, TBM));
  j.pw = static_cast<int>(a.J < bn ? a.J : bn);
  j.part = a.part;
  j.ep = a.ep;
  return ok && a.k_per_split > 0 && ceil_div(a.Kred, a.k_per_split) <= a.splits;
}

// One launch of one or two products (n = 1, 2) of the same operand layouts.
cudaError_t launch_jobs(const SkinnyArgs *a, int n, cudaStream_t st) {
  CUtensorMap tm[4];
  TParams p{};
  int64_t tiles = 0;
  for (int k = 0; k < n; ++k) {
    if (!fill_job(a[k], p.job[k], tm[2 * k], tm[2 * k + 1])) return cudaErrorInvalidValue;
    tiles += skinny_tiles(a[k].I, a[k].J);
    if (k == 0) p.x_split = static_cast<int>(tiles);
  }
  if (n == 1) {
    p.job[1] = p.job[0];
    tm[2] = tm[0];
    tm[3] = tm[1];
  }
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  if (!p.status || tiles > (int64_t(1) << 30)) return cudaErrorInvalidValue;
  const bool fused = a[0].ep.kind != kSkinnyPartial;
  const dim3 grid(static_cast<unsigned>(tiles), 1u, static_cast<unsigned>(a[0].splits));
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TSMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(TTHREADS);
    cfg.dynamicSmemBytes = TSMEM;
    cfg.stream = st;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;   // the splits of one tile: one cluster
    at[0].val.clusterDim.x = 1;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = fused ? static_cast<unsigned>(a[0].splits) : 1u;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the previous kernel's tail
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tm[0], tm[1], tm[2], tm[3], p);
  };
  prof_mark(kProfLora, true, st);
  cudaError_t e;
  if (a[0].a_kmajor && a[0].b_kmajor)
    e = go(lora_tc_kernel<false, false>);
  else if (a[0].a_kmajor && !a[0].b_kmajor)
    e = go(lora_tc_kernel<false, true>);
  else if (!a[0].a_kmajor && a[0].b_kmajor)
    e = go(lora_tc_kernel<true, false>);
  else
    e = go(lora_tc_kernel<true, true>);
  prof_mark(kProfLora, false, st);
  return e;
}
}  // namespace

void skinny_plan(int64_t I, int64_t J, int64_t Kred, int *splits, int64_t *k_per_split) {
  plan_splits(skinny_tiles(I, J), Kred, splits, k_per_split);
}

void skinny_plan_pair(int64_t I0, int64_t J0, int64_t I1, int64_t J1, int64_t Kred, int *splits,
                      int64_t *k_per_split) {
  plan_splits(skinny_tiles(I0, J0) + skinny_tiles(I1, J1), Kred, splits, k_per_split);
}

bool skinny_fused_ok(const SkinnyArgs &a) {
  const int64_t bn = tc_bn(a.J);
  if (a.ep.kind == kSkinnyPartial || a.splits < 1 || a.splits > kMaxSkinnyCluster) return false;
  // The in-kernel finish handles H and G in the kernels with a K-major first
  // operand and the stacked kinds (dB, dA) in the all-MN-major one, in runs of
  // eight columns.
  const bool stacked_layout = !a.a_kmajor && !a.b_kmajor;
  switch (a.ep.kind) {
    case kSkinnyH:
    case kSkinnyG:
      return !stacked_layout && a.a_kmajor && a.J <= bn && a.J % 8 == 0;   // one tile covers every column
    case kSkinnyCols:
      return stacked_layout && a.J <= bn && a.J % 16 == 0;                 // ... and both halves
    case kSkinnyRows:
      return stacked_layout && a.I <= TBM && a.I % 2 == 0 && a.J % 8 == 0;   // one tile covers both row halves
    default:
      return false;
  }
}

size_t skinny_part_floats(int64_t I, int64_t J, int splits) {
  const int64_t bn = tc_bn(J);
  // the fused layout [tile][slice][128 x pw] only where some kind can finish in-kernel:
  // one tile across J (H, G, dB) or one tile across I (dA)
  const bool fusable = J <= bn || I <= TBM;
  const int64_t fused = fusable ? skinny_tiles(I, J) * splits * TBM * (J < bn ? J : bn) : 0;
  const int64_t plain = static_cast<int64_t>(splits) * I * J;                     // [slice][I][J]
  return static_cast<size_t>(fused > plain ? fused : plain);
}

bool skinny_pair_ok(const SkinnyArgs &a, const SkinnyArgs &b) {
  return skinny_fused_ok(a) && skinny_fused_ok(b) && a.a_kmajor == b.a_kmajor && a.b_kmajor == b.b_kmajor &&
         a.splits == b.splits;
}

cudaError_t launch_skinny(const SkinnyArgs &a, cudaStream_t st) {
  if (a.ep.kind != kSkinnyPartial && !skinny_fused_ok(a)) return cudaErrorInvalidValue;   // callers check first
  return launch_jobs(&a, 1, st);
}

cudaError_t launch_skinny_pair(const SkinnyArgs &a, const SkinnyArgs &b, cudaStream_t st) {
  if (!skinny_pair_ok(a, b)) return cudaErrorInvalidValue;   // callers check first
  SkinnyArgs ab[2] = {a, b};
  ab[1].part = a.part + skinny_part_floats(a.I, a.J, a.splits);   // the second product's partial tiles follow
  return launch_jobs(ab, 2, st);
}

}  // namespace qlora
