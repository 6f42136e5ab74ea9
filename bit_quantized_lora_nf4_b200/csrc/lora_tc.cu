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
// reduction, staged by TMA in 64-deep steps into a 4-deep ring (128B swizzle,
// K-major or MN-major as the operand is stored), issued by one thread as
// tcgen05.mma (M = 128) into TMEM.  The slices of one tile run as a thread-
// block cluster: each CTA stages its fp32 tile in shared memory, and after a
// cluster barrier CTA z adds rows z*128/Z .. of all Z tiles in slice order
// through distributed shared memory and applies the epilogue (scale, bf16,
// hi/lo split, the halves of a stacked operand).  When a tile cannot finish in
// its cluster the kernel writes fp32 partial sums part[z][i][j] instead and a
// second kernel adds them in the same fixed order.
#include <cooperative_groups.h>

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

struct TParams {
  int64_t I, J, Kred, kps;
  int bn;              // N of the MMA (multiple of 64, <= 256)
  float *part;
  SkinnyEpilogue ep;
  int *status;
  uint64_t wait_limit;
};
constexpr int TPITCH_PAD = 4;   // staged tile row pitch = bn + 4 floats (spreads rows over banks)

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

constexpr int kMaxZ = 8;   // most slices of one tile (the portable cluster size)

// After every slice of the tile is staged: CTA z of the Z in the cluster adds
// its share of the rows over all Z staged tiles in slice order (distributed
// shared memory) and writes the epilogue's outputs; a second cluster barrier
// keeps every staged tile alive until all its readers are done.
__device__ __forceinline__ void cluster_finish(const TParams &p, float *stage, int64_t i0, int64_t j0) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int Z = static_cast<int>(cl.num_blocks());
  const int z = static_cast<int>(cl.block_rank());
  cluster_sync_all();
  const int pitch = p.bn + TPITCH_PAD;
  const SkinnyEpilogue &ep = p.ep;
  const int kind = ep.kind;
  const int64_t J = p.J;
  const int half_j = static_cast<int>(J / 2), half_i = static_cast<int>(p.I / 2);
  // rows of the tile this kind produces, and columns
  const int trows = kind == kSkinnyRows ? half_i : TBM;
  const int tcols = kind == kSkinnyCols ? half_j : static_cast<int>(J - j0 < p.bn ? J - j0 : p.bn);
  const int per = (trows + Z - 1) / Z;
  const int rbeg = z * per, rend = rbeg + per < trows ? rbeg + per : trows;
  // four consecutive columns per item: every slice's values are fetched with
  // independent 16-byte loads before they are added (one round trip through
  // distributed shared memory instead of one per slice)
  const int tc4 = tcols / 4;   // tcols % 4 == 0 for every kind (J, r multiples of 4)
  const int n4 = rend > rbeg ? (rend - rbeg) * tc4 : 0;
  const bool paired = kind == kSkinnyCols || kind == kSkinnyRows;
  const int off2 = kind == kSkinnyCols ? half_j : half_i * pitch;   // the second half's offset
  for (int e4 = threadIdx.x; e4 < n4; e4 += blockDim.x) {
    const int row = rbeg + e4 / tc4, col0 = (e4 - (e4 / tc4) * tc4) * 4;
    const int64_t gi = i0 + row;
    if (kind != kSkinnyRows && gi >= p.I) continue;
    float4 a[kMaxZ], b[kMaxZ];
#pragma unroll
    for (int q = 0; q < kMaxZ; ++q) {
      if (q < Z) {
        const float *t = cl.map_shared_rank(stage, q) + row * pitch + col0;
        a[q] = *reinterpret_cast<const float4 *>(t);
        if (paired) b[q] = *reinterpret_cast<const float4 *>(t + off2);
      }
    }
    float v4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int q = 0; q < kMaxZ; ++q) {   // slice order: fixed, so the result is deterministic
      if (q < Z) {
        const float av[4] = {a[q].x, a[q].y, a[q].z, a[q].w};
        if (paired) {
          const float bv[4] = {b[q].x, b[q].y, b[q].z, b[q].w};
#pragma unroll
          for (int c = 0; c < 4; ++c) v4[c] = __fadd_rn(v4[c], __fadd_rn(av[c], bv[c]));
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) v4[c] = __fadd_rn(v4[c], av[c]);
        }
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
    const int col = col0 + c;
    const int64_t gj = j0 + col;
    const float v = v4[c];
    if (kind == kSkinnyH) {
      const int64_t idx = gi * J + gj;
      ep.out_f[idx] = v;
      ep.out_b[idx] = t_bf16(__fmul_rn(ep.s, v));
      if (ep.out_hl) {
        const uint16_t hi = t_bf16(v);
        ep.out_hl[gi * 2 * J + gj] = hi;
        ep.out_hl[gi * 2 * J + J + gj] = t_bf16(__fsub_rn(v, t_bf16_val(hi)));
      }
    } else if (kind == kSkinnyG) {
      const int64_t idx = gi * J + gj;
      const float g = __fmul_rn(ep.s, v);
      const uint16_t hi = t_bf16(g);
      ep.out_b[idx] = hi;
      ep.out_hl[gi * 2 * J + gj] = hi;
      ep.out_hl[gi * 2 * J + J + gj] = t_bf16(__fsub_rn(g, t_bf16_val(hi)));
      if (ep.aux) {
        const float h = ep.aux[idx];
        const uint16_t hh = t_bf16(h);
        ep.aux_hl[gi * 2 * J + gj] = hh;
        ep.aux_hl[gi * 2 * J + J + gj] = t_bf16(__fsub_rn(h, t_bf16_val(hh)));
      }
    } else if (kind == kSkinnyCols) {
      ep.out_f[gi * half_j + gj] = __fmul_rn(ep.s, v);
    } else {   // kSkinnyRows
      ep.out_f[static_cast<int64_t>(row) * J + gj] = v;
    }
    }
  }
  cluster_sync_all();
}

template <bool A_MN, bool B_MN>
__global__ void __launch_bounds__(TTHREADS, 1)
    lora_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const TParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  TSmem *sm = reinterpret_cast<TSmem *>(smem + TRING_BYTES);
  const int nstages = t_stages(p.bn);
  const int stage_bytes = t_stage_bytes(p.bn);     // a multiple of 8 KB
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * TBM;
  const int64_t j0 = static_cast<int64_t>(blockIdx.y) * p.bn;
  const int64_t kbeg = static_cast<int64_t>(blockIdx.z) * p.kps;
  const int64_t kend = (kbeg + p.kps < p.Kred) ? kbeg + p.kps : p.Kred;
  const int nsteps = kend > kbeg ? static_cast<int>((kend - kbeg + TBK - 1) / TBK) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nstages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->acc_full, 1);
    sm->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
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
  griddep_wait();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      const uint32_t b_bytes = static_cast<uint32_t>(p.bn) * TBK * 2;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % nstages;
        const uint32_t ph = (i / nstages) & 1;
        if (i >= nstages && !t_wait(&sm->empty[s], ph ^ 1, p, sm)) break;
        uint8_t *sa = smem + s * stage_bytes;
        uint8_t *sb = sa + TA_BYTES;
        const int k0 = static_cast<int>(kbeg + static_cast<int64_t>(i) * TBK);
        mbar_arrive_expect_tx(&sm->full[s], TA_BYTES + b_bytes);
        if (A_MN) {
          tma_load_2d(sa, &tmA, &sm->full[s], static_cast<int>(i0), k0);
          tma_load_2d(sa + 8192, &tmA, &sm->full[s], static_cast<int>(i0) + 64, k0);
        } else {
          tma_load_2d(sa, &tmA, &sm->full[s], k0, static_cast<int>(i0));
        }
        if (B_MN) {
          for (int b = 0; b < p.bn / 64; ++b)
            tma_load_2d(sb + 8192 * b, &tmB, &sm->full[s], static_cast<int>(j0) + 64 * b, k0);
        } else {
          tma_load_2d(sb, &tmB, &sm->full[s], k0, static_cast<int>(j0));
        }
        issued = i + 1;
      }
      for (int j = (issued > nstages ? issued - nstages : 0); j < issued; ++j)
        mbar_wait(&sm->full[j % nstages], (j / nstages) & 1, kTDrain);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(TBM, p.bn, A_MN ? 1 : 0, B_MN ? 1 : 0);
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
    // epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = rows of the tile
    const bool ok = mbar_wait(&sm->acc_full, 0, kTDrain);
    tc_fence_after();
    volatile int *abort_flag = &sm->abort_flag;
    if (p.ep.kind != kSkinnyPartial) {
      // stage this slice's tile (rows of this warp's TMEM lanes) for the cluster reduction;
      // the ring is free: every MMA that read it has completed
      const int quarter = warp & 3;
      float *st = reinterpret_cast<float *>(smem) + (quarter * 32 + lane) * (p.bn + TPITCH_PAD);
      const bool live = __all_sync(0xffffffffu, ok && *abort_flag == 0 && nsteps > 0);
      for (int cc = 0; cc < p.bn / 32; ++cc) {
        uint32_t v[32];
        if (live) {
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + cc * 32, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;   // empty slice (or aborted): zero
        }
        float4 *dst = reinterpret_cast<float4 *>(st + cc * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
      }
    } else if (__all_sync(0xffffffffu, ok && *abort_flag == 0 && nsteps > 0)) {
      const int quarter = warp & 3;
      const int64_t row = i0 + quarter * 32 + lane;
      float *out = p.part + static_cast<int64_t>(blockIdx.z) * p.I * p.J + row * p.J;
      for (int cc = 0; cc < p.bn / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + cc * 32, v);
        tmem_ld_wait();
        const int64_t c0 = j0 + cc * 32;
        if (row < p.I) {
          if (c0 + 32 <= p.J && (p.J & 3) == 0) {
            float4 *dst = reinterpret_cast<float4 *>(out + c0);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(__uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                                    __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          } else {
            for (int e = 0; e < 32; ++e)
              if (c0 + e < p.J) out[c0 + e] = __uint_as_float(v[e]);
          }
        }
      }
    } else if (nsteps == 0 && i0 < p.I) {
      // empty reduction slice: its partial sums are zero
      const int quarter = warp & 3;
      const int64_t row = i0 + quarter * 32 + lane;
      if (row < p.I) {
        float *out = p.part + static_cast<int64_t>(blockIdx.z) * p.I * p.J + row * p.J;
        for (int64_t c = j0; c < j0 + p.bn && c < p.J; ++c) out[c] = 0.0f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (p.ep.kind != kSkinnyPartial) cluster_finish(p, reinterpret_cast<float *>(smem), i0, j0);
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

void skinny_plan(int64_t I, int64_t J, int64_t Kred, int *splits, int64_t *k_per_split) {
  int64_t tiles = ceil_div(I, TBM) * ceil_div(J, tc_bn(J));
  if (tiles < 1) tiles = 1;
  if (Kred < 1) Kred = 1;
  // keep every split of every tile in one wave
  int64_t sp = 148 * TCTAS_PER_SM / tiles;
  const int64_t max_sp = Kred / (4 * TBK) > 0 ? Kred / (4 * TBK) : 1;
  if (sp > max_sp) sp = max_sp;
  if (sp > kMaxSkinnyCluster) sp = kMaxSkinnyCluster;   // the splits of a tile form one cluster
  if (sp < 1) sp = 1;
  const int64_t kps = ceil_div(ceil_div(Kred, sp), TBK) * TBK;
  *splits = static_cast<int>(ceil_div(Kred, kps));
  *k_per_split = kps;
}

bool skinny_fused_ok(const SkinnyArgs &a) {
  const int64_t bn = tc_bn(a.J);
  if (a.ep.kind == kSkinnyPartial || a.splits < 1 || a.splits > kMaxSkinnyCluster) return false;
  if (static_cast<int64_t>(TBM) * (bn + TPITCH_PAD) * 4 > TRING_BYTES) return false;   // staged tile fits the ring
  switch (a.ep.kind) {
    case kSkinnyH:
    case kSkinnyG:
      return a.J <= bn && a.J % 4 == 0;           // one tile covers every column
    case kSkinnyCols:
      return a.J <= bn && a.J % 8 == 0;           // ... and both halves, in runs of four
    case kSkinnyRows:
      return a.I <= TBM && a.I % 2 == 0 && a.J % 4 == 0;   // one tile covers both row halves
    default:
      return false;
  }
}

cudaError_t launch_skinny(const SkinnyArgs &a, cudaStream_t st) {
  const int64_t bn = tc_bn(a.J);
  CUtensorMap tmA, tmB;
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
  if (!ok) return cudaErrorInvalidValue;
  TParams p{};
  p.I = a.I;
  p.J = a.J;
  p.Kred = a.Kred;
  p.kps = a.k_per_split;
  p.bn = static_cast<int>(bn);
  p.part = a.part;
  const bool fused = skinny_fused_ok(a);
  if (a.ep.kind != kSkinnyPartial && !fused) return cudaErrorInvalidValue;   // callers check first
  p.ep = a.ep;
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  if (!p.status) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(ceil_div(a.I, TBM)), static_cast<unsigned>(ceil_div(a.J, bn)),
                  static_cast<unsigned>(a.splits));
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
    at[0].val.clusterDim.z = fused ? static_cast<unsigned>(a.splits) : 1u;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // overlap the previous kernel's tail
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, tmA, tmB, p);
  };
  prof_mark(kProfLora, true, st);
  cudaError_t e;
  if (a.a_kmajor && a.b_kmajor)
    e = go(lora_tc_kernel<false, false>);
  else if (a.a_kmajor && !a.b_kmajor)
    e = go(lora_tc_kernel<false, true>);
  else if (!a.a_kmajor && a.b_kmajor)
    e = go(lora_tc_kernel<true, false>);
  else
    e = go(lora_tc_kernel<true, true>);
  prof_mark(kProfLora, false, st);
  return e;
}

}  // namespace qlora
