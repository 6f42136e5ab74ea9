// Fused NF4 dequant-GEMM on 5th-generation tensor cores (tcgen05, TMEM, TMA).
//
// "QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory
// goes": every forward and backward pass expands the 4-bit base to 16-bit as it
// and backward pass, and gradients flow through the dequantized weights into
// the adapters.  "Qlora 4 Bit Quantization With Nf4 Fp4 Data Types And Lora
// Adapters", entry "quantization-aware-lora-training-with-kernel-fusion":
// quantized matmul and the low-rank term computed in one kernel invocation.
//
// One CTA computes a 128 x 256 fp32 tile in TMEM:
//   forward : Y [M, N]  = X [M, K] . W'^T        + sH [M, r] . B [N, r]^T
//   dgrad   : dX[M, K]  = dY[M, N] . W'          + Gb [M, r] . A [r, K]
// The adapter product is simply the last ceil(r/64) K-steps of the same
// accumulation (operands bf16(s*H) / bf16(G) and the adapter weight).
//
// Warp roles (320 threads):
//   warp 0      TMA producer: activation tile (128 x 64 bf16, 128B swizzle)
//               and the packed code tile (forward: 256 rows x 32 B, 32B
//               swizzle; dgrad: 64 rows x 128 B, 128B swizzle).
//   warp 1      allocates TMEM; one lane issues tcgen05.mma (M=128, N=256,
//               K=16) and commits to the stage's "empty" barrier.
//   warps 2-9   decode: each thread owns one 64-weight block per K-step.  It
//               forms a' = q*S, builds the block's 16-entry bf16 table
//               T[c] = bf16(level[c] * a') once, looks the 64 codes up with
//               byte permutes and writes the 128 bytes into the operand tile
//               in the 128B-swizzled canonical layout (K-major for the
//               forward, MN-major for dgrad).  After the last K-step the same
//               warps drain TMEM (tcgen05.ld) and store bf16 results.
//
// Every mbarrier wait is bounded; on expiry the CTA latches
// QLORA_ERR_DEVICE_TIMEOUT, lets outstanding TMA loads and MMAs land, frees
// TMEM and exits.
#include "decode.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int P_BYTES = BN * BK / 2;          //  8 KB
constexpr int D_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + P_BYTES + D_BYTES;
constexpr int NUM_DEC_WARPS = 8;
constexpr int THREADS = 32 * (2 + NUM_DEC_WARPS);
constexpr int TMEM_COLS = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint64_t kDrainLimit = 4000000000ull;   // bound for the exit drains

struct Params {
  int64_t M;
  int64_t n_out;     // output columns (forward: wN, dgrad: wK)
  int64_t ldo;
  int64_t wN, wK;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *lora_w;
  int r;
  int nkb;           // weight K-steps
  int nls;           // adapter K-steps
  uint16_t *out;
  int *status;
  uint64_t wait_limit;
};

struct Smem {
  uint64_t full[STAGES];
  uint64_t decoded[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, const Params &p, Smem *sm) {
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

template <bool DGRAD>
__global__ void __launch_bounds__(THREADS, 1)
    qgemm_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
                 const __grid_constant__ CUtensorMap tm_lact, const Params p, const Nf4Table tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem *sm = reinterpret_cast<Smem *>(smem + STAGES * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int nsteps = p.nkb + p.nls;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->decoded[s], NUM_DEC_WARPS);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->acc_full, 1);
    sm->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_lact);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (i >= STAGES && !wait_or_abort(&sm->empty[s], ph ^ 1, p, sm)) break;
        uint8_t *st = smem + s * STAGE_BYTES;
        if (i < p.nkb) {
          mbar_arrive_expect_tx(&sm->full[s], A_BYTES + P_BYTES);
          if (DGRAD) {
            tma_load_2d(st, &tm_act, &sm->full[s], i * BK, static_cast<int>(m0));
            tma_load_2d(st + A_BYTES, &tm_codes, &sm->full[s], static_cast<int>(n0 / 2), i * BK);
          } else {
            tma_load_2d(st, &tm_act, &sm->full[s], i * BK, static_cast<int>(m0));
            tma_load_2d(st + A_BYTES, &tm_codes, &sm->full[s], i * (BK / 2), static_cast<int>(n0));
          }
        } else {
          mbar_arrive_expect_tx(&sm->full[s], A_BYTES);
          tma_load_2d(st, &tm_lact, &sm->full[s], (i - p.nkb) * BK, static_cast<int>(m0));
        }
        issued = i + 1;
      }
      // Let every load this thread started land before the CTA can exit.
      for (int j = (issued > STAGES ? issued - STAGES : 0); j < issued; ++j)
        mbar_wait(&sm->full[j % STAGES], (j / STAGES) & 1, kDrainLimit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, 0, DGRAD ? 1 : 0);
      for (int i = 0; i < nsteps; ++i) {
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (!wait_or_abort(&sm->full[s], ph, p, sm)) break;
        if (!wait_or_abort(&sm->decoded[s], ph, p, sm)) break;
        tc_fence_after();
        const uint32_t a_base = smem_addr(smem + s * STAGE_BYTES);
        const uint32_t d_base = a_base + A_BYTES + P_BYTES;
        int nk = BK / 16;
        if (i >= p.nkb) {
          const int rem = p.r - (i - p.nkb) * BK;
          nk = rem >= BK ? BK / 16 : (rem + 15) / 16;
        }
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t adesc = sdesc_sw128(a_base + kk * 32, 16, 1024);
          const uint64_t bdesc = DGRAD ? sdesc_sw128(d_base + kk * 2048, 8192, 1024)
                                       : sdesc_sw128(d_base + kk * 32, 16, 1024);
          tc_mma_bf16(tmem, adesc, bdesc, IDESC, (i | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&sm->empty[s]);
      }
      tc_commit(&sm->acc_full);   // also the drain of every MMA issued above
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int dt = threadIdx.x - 64;      // 0..255
    const int64_t kblocks = p.wK / kBlock;
    // forward: row n0+dt, block i.  dgrad: row i*64 + (dt%64), block n0/64 + dt/64.
    auto block_index = [&](int i, int64_t *idx) -> bool {
      int64_t n, kb;
      if (DGRAD) {
        n = static_cast<int64_t>(i) * BK + (dt & 63);
        kb = n0 / kBlock + (dt >> 6);
      } else {
        n = n0 + dt;
        kb = i;
      }
      *idx = n * kblocks + kb;
      return n < p.wN && kb < kblocks;
    };
    const float mu = dq_offset(tab);
    uint32_t q_next = 0;
    float s_next = 0.0f;
    {
      int64_t idx;
      if (p.nkb > 0 && block_index(0, &idx)) {
        q_next = __ldg(p.absmax_q + idx);
        s_next = __ldg(p.group_scale + (idx >> 8));
      }
    }
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1;
      const float ap = block_constant(q_next, s_next, tab.qx, mu);
      q_next = 0;
      s_next = 0.0f;
      if (i + 1 < p.nkb) {
        int64_t idx;
        if (block_index(i + 1, &idx)) {
          q_next = __ldg(p.absmax_q + idx);
          s_next = __ldg(p.group_scale + (idx >> 8));
        }
      }
      // warp-uniform outcome: the warp-collective steps below need all 32 lanes
      if (!__all_sync(0xffffffffu, wait_or_abort(&sm->full[s], ph, p, sm))) break;
      const uint32_t st = smem_addr(smem + s * STAGE_BYTES);
      const uint32_t pbase = st + A_BYTES;
      const uint32_t dbase = st + A_BYTES + P_BYTES;
      if (i < p.nkb) {
        if (DGRAD) {
          const uint32_t j = dt >> 6, nl = dt & 63, sw = nl & 7;
          const uint32_t prow = pbase + nl * 128;
          nf4_decode_row(prow + (((2 * j) ^ sw) << 4), prow + (((2 * j + 1) ^ sw) << 4), dbase + j * 8192 + nl * 128,
                     sw, ap, tab);
        } else {
          const uint32_t sw32 = (dt >> 2) & 1;
          const uint32_t prow = pbase + dt * 32;
          nf4_decode_row(prow + ((0u ^ sw32) << 4), prow + ((1u ^ sw32) << 4), dbase + dt * 128, dt & 7, ap, tab);
        }
      } else {
        // adapter weight slice, copied into the same operand layout (zero past r / past the matrix)
        const int ls = i - p.nkb;
        if (DGRAD) {
          const uint32_t j = dt >> 6, rl = dt & 63;
          const int64_t rr = static_cast<int64_t>(ls) * BK + rl;
          for (int c = 0; c < 8; ++c) {
            const int64_t kk = n0 + 64 * j + 8 * c;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (rr < p.r && kk < p.wK) v = __ldg(reinterpret_cast<const uint4 *>(p.lora_w + rr * p.wK + kk));
            st_shared_v4(dbase + j * 8192 + rl * 128 + ((static_cast<uint32_t>(c) ^ (rl & 7)) << 4), v.x, v.y, v.z,
                         v.w);
          }
        } else {
          const int64_t n = n0 + dt;
          for (int c = 0; c < 8; ++c) {
            const int64_t rr = static_cast<int64_t>(ls) * BK + 8 * c;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (n < p.wN && rr < p.r) v = __ldg(reinterpret_cast<const uint4 *>(p.lora_w + n * p.r + rr));
            st_shared_v4(dbase + dt * 128 + ((static_cast<uint32_t>(c) ^ (dt & 7)) << 4), v.x, v.y, v.z, v.w);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm->decoded[s]);
    }

    // ------------------------------------------------------------ epilogue
    const bool acc_ok = mbar_wait(&sm->acc_full, 0, kDrainLimit);
    tc_fence_after();
    volatile int *abort_flag = &sm->abort_flag;
    if (__all_sync(0xffffffffu, acc_ok && *abort_flag == 0)) {
      const int quarter = warp & 3;
      const int half = (warp - 2) >> 2;
      const int64_t row = m0 + quarter * 32 + lane;
      uint16_t *orow = p.out + row * p.ldo;
      for (int cc = 0; cc < 4; ++cc) {
        const int col0 = half * 128 + cc * 32;
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + col0, v);
        tmem_ld_wait();
        if (row < p.M) {
          const int64_t c0 = n0 + col0;
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          if (c0 + 32 <= p.n_out && (p.ldo & 7) == 0) {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          } else {
            for (int j = 0; j < 32; ++j)
              if (c0 + j < p.n_out) orow[c0 + j] = static_cast<uint16_t>(pk[j >> 1] >> (16 * (j & 1)));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

qlora_status launch_qgemm(const QGemmArgs &a, cudaStream_t st) {
  if (a.M > kPairMinRows || a.wdense) return launch_qgemm_pair(a, st);
  CUtensorMap tm_act, tm_codes, tm_lact;
  const int64_t kred = a.dgrad ? a.wN : a.wK;      // reduction length of the weight segment
  const int64_t n_out = a.dgrad ? a.wK : a.wN;
  const uint64_t codes_row = static_cast<uint64_t>(a.wK / 2);
  bool ok = make_tmap_2d(&tm_act, a.act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kred, a.M, kred * 2, BK, BM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  if (a.dgrad)
    ok = ok && make_tmap_2d(&tm_codes, a.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_row, a.wN, codes_row, 128, 64,
                            CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_tmap_2d(&tm_codes, a.codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_row, a.wN, codes_row, 32, 256,
                            CU_TENSOR_MAP_SWIZZLE_32B);
  ok = ok && make_tmap_2d(&tm_lact, a.lora_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.r, a.M,
                          static_cast<uint64_t>(a.r) * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return QLORA_ERR_CUDA;

  Params p{};
  p.M = a.M;
  p.n_out = n_out;
  p.ldo = n_out;
  p.wN = a.wN;
  p.wK = a.wK;
  p.absmax_q = a.absmax_q;
  p.group_scale = a.group_scale;
  p.lora_w = a.lora_w;
  p.r = a.r;
  p.nkb = static_cast<int>(ceil_div(kred, BK));
  p.nls = static_cast<int>(ceil_div(a.r, BK));
  p.out = a.out;
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  if (!p.status) return QLORA_ERR_CUDA;

  const dim3 grid(static_cast<unsigned>(ceil_div(n_out, BN)), static_cast<unsigned>(ceil_div(a.M, BM)));
  cudaError_t e;
  const int kind = a.dgrad ? kProfGemmDgrad : kProfGemmFwd;
  if (a.dgrad) {
    e = cudaFuncSetAttribute(qgemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    prof_mark(kind, true, st);
    if (e == cudaSuccess) qgemm_kernel<true><<<grid, THREADS, SMEM_BYTES, st>>>(tm_act, tm_codes, tm_lact, p, a.tab);
  } else {
    e = cudaFuncSetAttribute(qgemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    prof_mark(kind, true, st);
    if (e == cudaSuccess) qgemm_kernel<false><<<grid, THREADS, SMEM_BYTES, st>>>(tm_act, tm_codes, tm_lact, p, a.tab);
  }
  prof_mark(kind, false, st);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
