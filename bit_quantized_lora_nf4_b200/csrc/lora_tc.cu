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
// tcgen05.mma (M = 128) into TMEM, and written as fp32 partial sums
// part[z][i][j]; a second kernel adds the slices in a fixed order.
#include "internal.h"

namespace qlora {

namespace {

constexpr int TBM = 128;
constexpr int TBN_MAX = 256;
constexpr int TBK = 64;
constexpr int TMAX_STAGES = 8;
constexpr int TA_BYTES = TBM * TBK * 2;         // 16 KB
constexpr int TRING_BYTES = 196608;             // 192 KB of stages: one CTA per SM
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
    if (__all_sync(0xffffffffu, ok && *abort_flag == 0 && nsteps > 0)) {
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
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TBN_MAX);
  }
}

}  // namespace

namespace {
int64_t tc_bn(int64_t J) {
  const int64_t b = ceil_div(J, 64) * 64;
  return b > TBN_MAX ? TBN_MAX : b;
}
}  // namespace

void skinny_plan(int64_t I, int64_t J, int64_t Kred, int *splits, int64_t *k_per_split) {
  int64_t tiles = ceil_div(I, TBM) * ceil_div(J, tc_bn(J));
  if (tiles < 1) tiles = 1;
  if (Kred < 1) Kred = 1;
  // one CTA per SM (192 KB of stages): keep every split of every tile in one wave
  int64_t sp = 148 / tiles;
  const int64_t max_sp = Kred / (4 * TBK) > 0 ? Kred / (4 * TBK) : 1;
  if (sp > max_sp) sp = max_sp;
  if (sp > 64) sp = 64;
  if (sp < 1) sp = 1;
  const int64_t kps = ceil_div(ceil_div(Kred, sp), TBK) * TBK;
  *splits = static_cast<int>(ceil_div(Kred, kps));
  *k_per_split = kps;
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
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  if (!p.status) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(ceil_div(a.I, TBM)), static_cast<unsigned>(ceil_div(a.J, bn)),
                  static_cast<unsigned>(a.splits));
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TSMEM);
    if (e != cudaSuccess) return e;
    kern<<<grid, TTHREADS, TSMEM, st>>>(tmA, tmB, p);
    return cudaGetLastError();
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
