// Fused NF4 dequant-GEMM over a CTA pair (tcgen05 cta_group::2).
//
// Same computation as qgemm.cu ("Where the memory goes": the 4-bit base is
// dequantized on the fly for each forward and backward pass; the adapter term
// is the last K segment of the same accumulation), on a 256 x 256 output tile
// per accumulator and cluster of two CTAs.  The pair's MMA (M = 256, N = 256,
// K = 16) takes its A rows from both CTAs (128 each) and its B columns from
// both CTAs (128 each), so every CTA decodes only half of the 256-row weight
// tile for the same tensor-core work per SM as the one-CTA kernel; with two
// accumulators per CTA (M > 256: a 512-row pair tile, K-step 64) each decoded
// operand half feeds two MMAs, halving the decode cost per flop again.
//
// Persistent: one cluster per co-resident slot walks its tiles (cid, cid + C,
// ...) as segments, then, when the last round of tiles is split (stream-K),
// its share of the shared tiles' K-steps.  Per CTA (352 threads), with
// separate rings so that neither load latency nor decode sits on the MMA's
// critical path:
//   warp 0      TMA: activation tiles (two 128B-swizzled 64-column boxes per
//               accumulator) into a 4-deep ring, and an L2 prefetch of the
//               tile four steps ahead.
//   warp 1      TMEM allocation for the pair; in the even CTA one lane issues
//               the MMAs of accumulator 0 (of all, with one accumulator); in
//               the odd CTA two lanes, taking the K-steps in turn, forward the
//               readiness of its activation tile and operand half.
//   warps 2-9   decode: thread (row = t % 128, j = t / 128) owns block j of its
//               row.  Its 32 bytes of codes and its 8-bit constant are loaded
//               from global memory into registers two of its K-steps ahead; it
//               builds the block's 16-entry table, looks the codes up with byte
//               permutes and writes 128 swizzled bytes into a 64 KB ring of
//               operand halves (K-major for the forward, MN-major for dgrad;
//               the byte address is the same formula in both).  At a tile's end
//               each group first writes its step of the next tile, then drains
//               its accumulator (TMEM -> bf16 boxes in shared memory -> TMA
//               stores, or fp32 pieces for a shared tile).
//   warp 10     even CTA, two accumulators: the MMA issuer of accumulator 1,
//               so that one issuer's barrier test and commit overlap the
//               other's MMAs.
// In the even CTA a step's inputs (its activation bytes, its decode group, the
// odd CTA's forwarded readiness) all arrive on one barrier per stage, and one
// commit per issuer frees both rings' slots.  Measured per K-step on the
// LLaMA-7B projections, MMA issue takes ~1070 clocks (paced by the tensor
// pipe) against ~150 of barrier testing and ~57 of commits per issuer, and
// late inputs are rare (3-10 % of steps).
// Waits are bounded; on expiry a CTA latches QLORA_ERR_DEVICE_TIMEOUT, lets
// its outstanding loads and the pair's MMAs land, frees TMEM and exits.
#include <algorithm>
#include <atomic>

#include "decode.cuh"
#include "internal.h"

namespace qlora {

namespace {

constexpr int BM = 128;            // rows per CTA
constexpr int BN = 256;            // output columns per pair (128 B-operand columns per CTA)
// Pipeline depths (compile-time tunables): activation stages, KB of decoded
// operand stages, and how many of its own K-steps ahead a decode thread loads
// its codes.
#ifndef QLORA_PAIR_A_STAGES
#define QLORA_PAIR_A_STAGES 4
#endif
#ifndef QLORA_PAIR_D_RING_KB
#define QLORA_PAIR_D_RING_KB 64
#endif
#ifndef QLORA_PAIR_PREFETCH
#define QLORA_PAIR_PREFETCH 2
#endif
constexpr int A_STAGES = QLORA_PAIR_A_STAGES;
constexpr int A_BYTES = 32768;              // one activation stage: NACC x 128 rows x BK bf16
constexpr int HALF = 16384;                 // one 128-row x 64-column swizzled atom column
constexpr int D_RING = QLORA_PAIR_D_RING_KB * 1024;   // decoded-operand stages
constexpr int PREFETCH = QLORA_PAIR_PREFETCH;
constexpr int NUM_DEC_WARPS = 8;
// warp 0 TMA, warp 1 MMA issuer (accumulator 0) / forwarder, warps 2-9 decode,
// warp 10 the second MMA issuer (accumulator 1) when a CTA holds two
constexpr int ISSUER2_WARP = 2 + NUM_DEC_WARPS;
constexpr int THREADS = 32 * (3 + NUM_DEC_WARPS);

// NACC = accumulators per CTA: the pair tile covers 256 * NACC rows.  With
// NACC = 2 every decoded operand half feeds two MMAs (rows 0-255 and 256-511
// of the pair tile), halving the decode work per tensor-core flop again; the
// K-step shrinks to 64 so the activation stage stays 32 KB, and the decode
// warps split into two groups that take alternate K-steps.
template <int NACC>
struct Cfg {
  static constexpr int BK = 128 / NACC;                      // K per stage
  static constexpr int KH = BK / 64;                         // 64-wide halves per stage
  static constexpr int D_BYTES = 128 * BK * 2;               // this CTA's operand half per stage
  static constexpr int D_STAGES = D_RING / D_BYTES;          // 3 or 6
  static constexpr int TMEM_COLS = 256 * NACC;
  static constexpr int GROUP_WARPS = NUM_DEC_WARPS / NACC;   // decode warps per group
};
constexpr int MAX_D_STAGES = 8;
static_assert(Cfg<1>::D_STAGES >= 2 && Cfg<2>::D_STAGES <= MAX_D_STAGES, "operand ring depth");
constexpr uint64_t kDrainLimit = 4000000000ull;
constexpr int kFwdLanes = 2;                // odd CTA: lanes forwarding readiness, steps in turn
constexpr int kGroupM = 8;                  // M-pairs per raster group (default)
// Raster per launch (compile-time switch for comparisons: 0 keeps kGroupM).
#ifndef QLORA_PAIR_RASTER_AUTO
#define QLORA_PAIR_RASTER_AUTO 1
#endif
// Stream-K tail: the tiles left after the last full wave have their K-steps
// split evenly over the cluster slots; a workspace provides for kSkMaxUnits
// such clusters, and none takes fewer than kSkMinSteps K-steps.  Measured on
// the LLaMA-7B projections (0.85 us per K-step), a cluster sharing tiles spends
// about kSkCostSteps K-steps' time beyond its own steps (accumulator drain and
// refill at a tile boundary, writing its 256 KB fp32 piece, the finisher
// reading the others' pieces at ~50 GB/s per SM), and a whole tile about
// kTileCostSteps (fill, drain, epilogue); the automatic mode splits only when
// that comes out shorter.
constexpr int kSkMaxUnits = 80;
constexpr int kSkMinSteps = 16;
constexpr int kSkCostSteps = 33;
constexpr int kTileCostSteps = 8;

struct Params {
  int64_t M;
  int64_t n_out;
  int64_t ldo;
  int64_t wN, wK;
  const uint8_t *codes;
  const uint8_t *absmax_q;
  const float *group_scale;
  const uint16_t *lora_w;
  const uint16_t *wdense;   // DENSE: the bf16 weight [wN, wK]
  int r;
  int nkb;           // weight K-steps (of 128)
  int nls;           // adapter K-steps (of 128)
  int num_m, num_n;  // pair tiles along M and along the output columns
  int group_m;       // M-pairs per raster group
  uint16_t *out;
  int *status;
  uint64_t wait_limit;
  int ns;            // K-steps per tile (nkb + nls)
  int dp_tiles;      // tiles taken whole, one per cluster (the full waves)
  int sk_units;      // clusters sharing the remaining tiles' K-steps (0: none)
  int64_t sk_steps;  // K-steps of the shared tiles
  int *sk_count;     // [shared tile][rank]: CTAs that finished accumulating a piece
  int *sk_ready;     // [shared tile][rank]: pieces written to sk_part
  float *sk_part;    // [unit][first, last piece][rank][NACC x 128 x 256] fp32
};

struct Smem {
  uint64_t afull[A_STAGES];        // activation tile landed (TMA)
  uint64_t aempty[A_STAGES];       // the pair's MMAs reading it completed (multicast commit)
  uint64_t dfree[MAX_D_STAGES];        // the pair's MMAs reading the operand half completed (multicast commit;
                                       // aempty serves both rings when they share their depth)
  uint64_t decoded[MAX_D_STAGES];      // this CTA's decode group wrote the operand half
  uint64_t peer_decoded[MAX_D_STAGES]; // even CTA only: the step's inputs are ready (see kMerged)
  uint64_t acc_full;               // the pair's accumulation completed (multicast commit)
  uint64_t tmem_empty;             // even CTA: both CTAs read the accumulators (next tile may start)
  uint32_t tmem_base;
  int abort_flag;
  int sk_role;                     // this CTA's arrival order on a shared tile
  int sk_ok;                       // the other pieces were written in time
};
constexpr int SMEM_BYTES = A_STAGES * A_BYTES + D_RING + 1024 + static_cast<int>(sizeof(Smem));
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(A_STAGES * A_BYTES >= NUM_DEC_WARPS * 16384, "epilogue staging fits the activation ring");

// Tile t of the grouped raster: consecutive tiles walk group_m M-pairs before
// moving to the next N tile, so a wave reuses both operands from L2.
__device__ __forceinline__ void tile_coords(const Params &p, int t, int &pm, int &pn) {
  const int in_group = p.group_m * p.num_n;
  const int first_m = (t / in_group) * p.group_m;
  const int gsz = min(p.num_m - first_m, p.group_m);
  pm = first_m + (t % in_group) % gsz;
  pn = (t % in_group) / gsz;
}

// Stream-K partition of the shared tiles' K-steps: unit u takes
// [sk_begin(u), sk_begin(u + 1)); sk_unit_of inverts it.
__host__ __device__ __forceinline__ int64_t sk_begin(int64_t steps, int units, int u) {
  return static_cast<int64_t>(u) * steps / units;
}
__device__ __forceinline__ int sk_unit_of(const Params &p, int64_t g) {
  return static_cast<int>(((g + 1) * p.sk_units - 1) / p.sk_steps);
}

template <bool CLUSTER_SCOPE>
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, const Params &p, Smem *sm) {
  const uint32_t a = smem_addr(bar);
  auto poll = [&]() { return CLUSTER_SCOPE ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity); };
  if (poll()) return true;
  const long long t0 = clock64();
  volatile int *abort_flag = &sm->abort_flag;
  while (true) {
    if (poll()) return true;
    if (*abort_flag) return false;
    if (static_cast<uint64_t>(clock64() - t0) > p.wait_limit) {
      *abort_flag = 1;
      latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}

// Registers a decode thread needs for one K-step: its block's 32 code bytes
// and the block constant q * S (zero for blocks outside the weight).
struct BlockLoad {
  uint4 lo, hi;
  uint32_t q;
  float S;
};

// One weight run of a DENSE operand row: 8 x 16 bytes of bf16 W'.
struct DenseLoad {
  uint4 v[8];
};

template <bool DGRAD, int NACC, bool DENSE>
__global__ void __launch_bounds__(THREADS, 1)
    qgemm2_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_lact,
                  const __grid_constant__ CUtensorMap tm_out, const Params p, const Nf4Table tab) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *a_ring = smem;
  using C = Cfg<NACC>;
  constexpr int BK = C::BK;
  constexpr int D_STAGES = C::D_STAGES;
  // When both rings have the same depth, the even CTA's inputs of a step all
  // arrive on one barrier, peer_decoded[s]: its activation TMA (bytes), its
  // decode group's warps and the odd CTA's forwarder, so the MMA issuer tests
  // one barrier per step instead of three (each test costs the issuer time in
  // which the tensor pipe can run dry).  Otherwise peer_decoded carries the
  // forwarder alone and afull / decoded are tested too.
  constexpr bool kMerged = A_STAGES == D_STAGES;
  constexpr int D_BYTES = C::D_BYTES;
  uint8_t *d_ring = smem + A_STAGES * A_BYTES;
  Smem *sm = reinterpret_cast<Smem *>(d_ring + D_RING);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                              // 0 = even (MMA-issuing) CTA
  const bool merged_even = kMerged && rank == 0;
  const int ns = p.ns;
  // The cluster's work, as consecutive segments: whole tiles cid, cid + C,
  // cid + 2C, ... (C = nclus clusters; round i takes tiles iC .. iC + C - 1, in
  // raster order), then, for a stream-K unit, its contiguous share [G0, G1) of the
  // shared tiles' K-steps (tail-linear order: shared tile ts, step k at ts ns + k).
  // Running step j of the cluster counts all its K-steps in that order.
  const int nclus = static_cast<int>(gridDim.x >> 1);
  const int cid = static_cast<int>(blockIdx.x >> 1);
  const int n_dp = cid < p.dp_tiles ? (p.dp_tiles - cid + nclus - 1) / nclus : 0;
  const int unit = cid < p.sk_units ? cid : -1;
  int64_t G0 = 0, G1 = 0;
  int sk_t0 = 0, n_sk = 0;
  if (unit >= 0) {
    G0 = sk_begin(p.sk_steps, p.sk_units, unit);
    G1 = sk_begin(p.sk_steps, p.sk_units, unit + 1);
    sk_t0 = static_cast<int>(G0 / ns);
    n_sk = static_cast<int>((G1 - 1) / ns) - sk_t0 + 1;
  }
  const int nseg = n_dp + n_sk;
  const int nsteps = n_dp * ns + static_cast<int>(G1 - G0);

  // Segment s: K-steps [k_lo, k_hi) of tile t; j0 is the running index of its
  // first step.  This CTA's rows of accumulator a are mbase + 256 a .. + 127,
  // its operand columns nb0 .. + 127.
  struct Seg {
    int t, k_lo, k_hi, j0;
    int mbase, n0, nb0;      // M, N and K are below 2^31
  };
  auto segment = [&](int s) {
    Seg sg;
    if (s < n_dp) {
      sg.t = cid + s * nclus;
      sg.k_lo = 0;
      sg.k_hi = ns;
      sg.j0 = s * ns;
    } else {
      const int ts = sk_t0 + (s - n_dp);
      const int64_t tb = static_cast<int64_t>(ts) * ns;
      sg.t = p.dp_tiles + ts;
      sg.k_lo = static_cast<int>((G0 > tb ? G0 : tb) - tb);
      sg.k_hi = static_cast<int>((G1 < tb + ns ? G1 : tb + ns) - tb);
      sg.j0 = n_dp * ns + static_cast<int>(tb + sg.k_lo - G0);
    }
    int pm, pn;
    tile_coords(p, sg.t, pm, pn);
    sg.mbase = pm * (2 * BM * NACC) + static_cast<int>(rank) * BM;
    sg.n0 = pn * BN;
    sg.nb0 = sg.n0 + static_cast<int>(rank) * 128;
    return sg;
  };
  auto seg_end = [](const Seg &sg) { return sg.j0 + (sg.k_hi - sg.k_lo); };
  // Follows running steps forward (never back) across segments.
  struct Cursor {
    int s;
    Seg sg;
  };
  // tile-local K-step of running step j (j < nsteps), moving the cursor to its segment
  auto cursor_at = [&](Cursor &c, int j) {
    while (j >= seg_end(c.sg)) c.sg = segment(++c.s);
    return c.sg.k_lo + (j - c.sg.j0);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < A_STAGES; ++s) {
      mbar_init(&sm->afull[s], 1);
      mbar_init(&sm->aempty[s], NACC);   // one commit per issuer
    }
    for (int s = 0; s < D_STAGES; ++s) {
      mbar_init(&sm->dfree[s], 1);
      mbar_init(&sm->decoded[s], C::GROUP_WARPS);
      mbar_init(&sm->peer_decoded[s], kMerged ? C::GROUP_WARPS + 2 : 1);
    }
    mbar_init(&sm->acc_full, NACC);
    mbar_init(&sm->tmem_empty, 2 * NUM_DEC_WARPS);
    sm->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_lact);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm->tmem_base, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();        // peer barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  // The next kernel on the stream may be scheduled once every CTA of this grid
  // has passed here (so it never takes a slot one of these still needs); no
  // global memory is touched before the previous kernel's writes are visible.
  griddep_launch_dependents();
  griddep_wait();

  // Pair MMA issuer (even CTA): accumulators [acc_lo, acc_hi) of every step.
  // With two accumulators a second thread (warp ISSUER2_WARP) issues the other
  // one, so one issuer's barrier tests and commits overlap the other's MMAs
  // and the tensor pipe is not left idle between steps; each commits its own
  // MMAs (the slot and accumulator barriers count one arrival per issuer).
  auto run_issuer = [&](int acc_lo, int acc_hi) {
    constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, BN, 0, DGRAD ? 1 : 0);
    int commits = 0;
    bool stop = false;
    for (int seg = 0; seg < nseg && !stop; ++seg) {
      const Seg sg = segment(seg);
      // a later tile overwrites the accumulators: both CTAs must have read them
      if (seg > 0 && !wait_or_abort<true>(&sm->tmem_empty, (seg - 1) & 1, p, sm)) {
        stop = true;
        break;
      }
      for (int k = sg.k_lo; k < sg.k_hi; ++k) {
        const int i = sg.j0 + (k - sg.k_lo);
        const int sa = i % A_STAGES, sd = i % D_STAGES;
        const uint32_t pa = (i / A_STAGES) & 1, pd = (i / D_STAGES) & 1;
        // the three inputs of the step probed together (their latencies overlap);
        // the bounded waits only when one of them is not there yet
        if (kMerged) {
          if (!mbar_test_cluster(smem_addr(&sm->peer_decoded[sd]), pd) &&
              !wait_or_abort<true>(&sm->peer_decoded[sd], pd, p, sm)) {
            stop = true;
            break;
          }
        } else if (!(mbar_test(smem_addr(&sm->afull[sa]), pa) & mbar_test(smem_addr(&sm->decoded[sd]), pd) &
                     mbar_test_cluster(smem_addr(&sm->peer_decoded[sd]), pd))) {
          if ((!mbar_test(smem_addr(&sm->afull[sa]), pa) && !wait_or_abort<false>(&sm->afull[sa], pa, p, sm)) ||
              (!mbar_test(smem_addr(&sm->decoded[sd]), pd) && !wait_or_abort<false>(&sm->decoded[sd], pd, p, sm)) ||
              !wait_or_abort<true>(&sm->peer_decoded[sd], pd, p, sm)) {
            stop = true;
            break;
          }
        }
        tc_fence_after();
        const uint32_t a_base = smem_addr(a_ring + sa * A_BYTES);
        const uint32_t d_base = smem_addr(d_ring + sd * D_BYTES);
        int nk = BK / 16;
        if (k >= p.nkb) {
          const int rem = p.r - (k - p.nkb) * BK;
          nk = rem >= BK ? BK / 16 : (rem + 15) / 16;
        }
        // descriptors of the stage's first slice; a slice's start address adds
        // its byte offset / 16 to the low field (no carry: shared memory < 256 KB)
        const uint64_t adesc0 = sdesc_sw128(a_base, 16, 1024);
        const uint64_t bdesc0 = DGRAD ? sdesc_sw128(d_base, BK * 128, 1024) : sdesc_sw128(d_base, 16, 1024);
        for (int kk = 0; kk < nk; ++kk) {
          const uint32_t koff = (kk >> 2) * HALF + (kk & 3) * 32;
          const uint64_t bdesc = bdesc0 + ((DGRAD ? kk * 2048u : koff) >> 4);
          for (int a = acc_lo; a < acc_hi; ++a) {
            const uint64_t adesc = adesc0 + ((a * C::KH * HALF + koff) >> 4);
            tc_mma_bf16_pair(tmem + 256 * a, adesc, bdesc, IDESC, (k != sg.k_lo || kk != 0) ? 1u : 0u);
          }
        }
        // both rings' slot of the step is free once its MMAs complete: one commit
        // per issuer when they share their depth
        tc_commit_pair_mc(&sm->aempty[sa], 0x3);
        if (!kMerged) tc_commit_pair_mc(&sm->dfree[sd], 0x3);
      }
      if (stop) break;
      tc_commit_pair_mc(&sm->acc_full, 0x3);
      ++commits;
    }
    if (stop) {
      // given up: one more commit, and wait until it (every MMA issued) has
      // completed, so that the accumulators are idle before teardown
      tc_commit_pair_mc(&sm->acc_full, 0x3);
      mbar_wait(&sm->acc_full, commits & 1, kDrainLimit);
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ activation TMA (each CTA)
    if (lane == 0) {
      int issued = 0;
      bool stop = false;
      Cursor pf{0, segment(0)};              // the step A_STAGES ahead, for the L2 prefetch
      for (int s = 0; s < nseg && !stop; ++s) {
        const Seg sg = segment(s);
        for (int k = sg.k_lo; k < sg.k_hi; ++k) {
          const int i = sg.j0 + (k - sg.k_lo);
          const int s = i % A_STAGES;
          const uint32_t ph = (i / A_STAGES) & 1;
          if (i >= A_STAGES && !wait_or_abort<false>(&sm->aempty[s], ph ^ 1, p, sm)) {
            stop = true;
            break;
          }
          uint64_t *full = merged_even ? &sm->peer_decoded[s] : &sm->afull[s];
          uint8_t *st = a_ring + s * A_BYTES;
          // atom column (t, kh) of the stage at (t * KH + kh) * HALF
          if (k < p.nkb) {
            mbar_arrive_expect_tx(full, A_BYTES);
            for (int a = 0; a < NACC; ++a)
              for (int kh = 0; kh < C::KH; ++kh)
                tma_load_2d(st + (a * C::KH + kh) * HALF, &tm_act, full, k * BK + 64 * kh,
                            static_cast<int>(sg.mbase + 256 * a));
          } else {
            const int ls = k - p.nkb;
            const int rem = p.r - ls * BK;
            const int halves = rem > 64 ? C::KH : 1;
            mbar_arrive_expect_tx(full, NACC * halves * HALF);
            for (int a = 0; a < NACC; ++a)
              for (int kh = 0; kh < halves; ++kh)
                tma_load_2d(st + (a * C::KH + kh) * HALF, &tm_lact, full, ls * BK + 64 * kh,
                            static_cast<int>(sg.mbase + 256 * a));
          }
          // the tile A_STAGES steps further on goes to L2 now: its load waits for a free
          // slot, and for the operands read from DRAM the wait would otherwise add the
          // DRAM latency to the step
          const int ipf = i + A_STAGES;
          if (ipf < nsteps) {
            const int kpf = cursor_at(pf, ipf);
            if (kpf < p.nkb)
              for (int a = 0; a < NACC; ++a)
                for (int kh = 0; kh < C::KH; ++kh)
                  tma_prefetch_2d(&tm_act, kpf * BK + 64 * kh, static_cast<int>(pf.sg.mbase + 256 * a));
          }
          issued = i + 1;
        }
      }
      for (int j = (issued > A_STAGES ? issued - A_STAGES : 0); j < issued; ++j)
        mbar_wait(merged_even ? &sm->peer_decoded[j % A_STAGES] : &sm->afull[j % A_STAGES], (j / A_STAGES) & 1,
                  kDrainLimit);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------------- pair MMA issuer (even CTA)
      run_issuer(0, NACC == 2 ? 1 : NACC);
    } else if (rank != 0 && lane < kFwdLanes) {
      // ---------------------------------------------------------- odd CTA: forward readiness
      // The even CTA's MMA reads this CTA's activation tile and operand half:
      // once both are in place, one cluster-scope release per stage.  (The
      // decode warps arrive only locally: a cluster-scope release from them
      // would also wait for the code loads they keep in flight for later steps.)
      // Both barriers are probed together; the bounded waits only for one that
      // is not complete yet.  A cluster-scope release arrive takes about as long
      // as a K-step's MMAs, so kFwdLanes lanes take the steps in turn and their
      // arrives overlap.
      for (int i = lane; i < nsteps; i += kFwdLanes) {
        const int sa = i % A_STAGES, sd = i % D_STAGES;
        const uint32_t pa = (i / A_STAGES) & 1, pd = (i / D_STAGES) & 1;
        const bool ra = mbar_test(smem_addr(&sm->afull[sa]), pa), rd = mbar_test(smem_addr(&sm->decoded[sd]), pd);
        if (!ra && !wait_or_abort<false>(&sm->afull[sa], pa, p, sm)) break;
        if (!rd && !wait_or_abort<false>(&sm->decoded[sd], pd, p, sm)) break;
        mbar_arrive_cluster(mapa_shared(smem_addr(&sm->peer_decoded[sd]), 0));
      }
    }
  } else if (warp == ISSUER2_WARP) {
    if (NACC == 2 && lane == 0 && rank == 0) run_issuer(1, 2);
  } else {
    // ------------------------------------------------------------ decoders (each CTA)
    // NACC groups of decode warps take alternate running steps; within a
    // group, thread u owns block jb of operand row `row` (forward: weight row,
    // 128 per stage; dgrad: reduction row, BK per stage).
    const int dwarp = warp - 2;
    const int grp = dwarp / C::GROUP_WARPS;
    const int u = (threadIdx.x - 64) % (C::GROUP_WARPS * 32);
    constexpr int DROWS = DGRAD ? BK : 128;
    const int row = u % DROWS;
    const int jb = u / DROWS;
    const int64_t kblocks = p.wK / kBlock;
    // Loads for K-step k of the current tile (operand columns nb0 ..) into
    // registers; zero past the tile's weight steps.  The prefetch stays within
    // a segment, so nothing is held across a segment's epilogue.
    auto fetch = [&](int k, bool live, int nb0, BlockLoad &b) {
      b.lo = b.hi = make_uint4(0, 0, 0, 0);
      b.q = 0;
      b.S = 0.0f;
      if (!live || k >= p.nkb) return;
      int64_t n, kb;
      if (DGRAD) {
        n = static_cast<int64_t>(k) * BK + row;
        kb = nb0 / kBlock + jb;
      } else {
        n = nb0 + row;
        kb = static_cast<int64_t>(k) * C::KH + jb;
      }
      if (n < p.wN && kb < kblocks) {
        const int64_t idx = n * kblocks + kb;
        const uint4 *src = reinterpret_cast<const uint4 *>(p.codes + idx * 32);
        b.lo = __ldg(src);
        b.hi = __ldg(src + 1);
        b.q = __ldg(p.absmax_q + idx);
        b.S = __ldg(p.group_scale + (idx >> 8));
      }
    };
    // DENSE: the operand row's 64 weights of this thread's run, 8 x 16 bytes
    // (zero past the matrix), loaded one of the group's K-steps ahead.
    auto fetch_dense = [&](int k, bool live, int nb0, DenseLoad &d) {
#pragma unroll
      for (int c = 0; c < 8; ++c) d.v[c] = make_uint4(0, 0, 0, 0);
      if (!live || k >= p.nkb) return;
      int64_t n, kk;
      if (DGRAD) {
        n = static_cast<int64_t>(k) * BK + row;
        kk = nb0 + 64 * jb;
      } else {
        n = nb0 + row;
        kk = static_cast<int64_t>(k) * BK + 64 * jb;
      }
      if (n < p.wN && kk < p.wK) {
        const uint4 *src = reinterpret_cast<const uint4 *>(p.wdense + n * p.wK + kk);
#pragma unroll
        for (int c = 0; c < 8; ++c) d.v[c] = __ldg(src + c);
      }
    };
    const float mu = DENSE ? 0.0f : dq_offset(tab);
    const uint32_t swz = row & 7;             // 128B swizzle of the operand
    volatile int *abort_flag = &sm->abort_flag;
    volatile int *sk_role = &sm->sk_role;
    volatile int *sk_ok = &sm->sk_ok;
    bool dead = false;                        // warp-uniform: this warp gave up waiting
    // Writes the operand of running step i (K-step k of the tile whose operand
    // columns start at nb0) once its ring slot is free; false if the wait gave up.
    auto emit = [&](int i, int k, int nb0, const BlockLoad &cur, const DenseLoad &dcur) {
      const int sd = i % D_STAGES;
      if (i >= D_STAGES && !__all_sync(0xffffffffu, wait_or_abort<false>(kMerged ? &sm->aempty[sd] : &sm->dfree[sd],
                                                                         ((i / D_STAGES) & 1) ^ 1, p, sm)))
        return false;
      const uint32_t drow = smem_addr(d_ring + sd * D_BYTES) + jb * (DROWS * 128) + row * 128;
      if (DENSE && k < p.nkb) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(drow + ((static_cast<uint32_t>(c) ^ swz) << 4), dcur.v[c].x, dcur.v[c].y, dcur.v[c].z,
                       dcur.v[c].w);
      } else if (k < p.nkb) {
        const float ap = block_constant(cur.q, cur.S, tab.qx, mu);
        uint32_t LO[4], HI[4];
        nf4_block_table(ap, tab, LO, HI);
        const uint32_t words[8] = {cur.lo.x, cur.lo.y, cur.lo.z, cur.lo.w, cur.hi.x, cur.hi.y, cur.hi.z, cur.hi.w};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t o[4];
          nf4_lut8(words[w], LO, HI, o);
          st_shared_v4(drow + ((static_cast<uint32_t>(w) ^ swz) << 4), o[0], o[1], o[2], o[3]);
        }
      } else {
        // adapter weight slice in the same operand layout; zero past r / past the matrix
        const int64_t base_r = static_cast<int64_t>(k - p.nkb) * BK + 64 * jb;
        for (int c = 0; c < 8; ++c) {
          uint4 v = make_uint4(0, 0, 0, 0);
          if (DGRAD) {
            const int64_t rr = static_cast<int64_t>(k - p.nkb) * BK + row;
            const int64_t kk = static_cast<int64_t>(nb0) + 64 * jb + 8 * c;
            if (rr < p.r && kk < p.wK) v = __ldg(reinterpret_cast<const uint4 *>(p.lora_w + rr * p.wK + kk));
          } else {
            const int64_t n = static_cast<int64_t>(nb0) + row;
            const int64_t rr = base_r + 8 * c;
            if (n < p.wN && rr < p.r) v = __ldg(reinterpret_cast<const uint4 *>(p.lora_w + n * p.r + rr));
          }
          st_shared_v4(drow + ((static_cast<uint32_t>(c) ^ swz) << 4), v.x, v.y, v.z, v.w);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(merged_even ? &sm->peer_decoded[sd] : &sm->decoded[sd]);
      return true;
    };
    bool ahead = false;                       // this group's first step of the segment was written early
    for (int seg = 0; seg < nseg; ++seg) {
      const Seg sg = segment(seg);
      const int t = sg.t;
      const int i_end = seg_end(sg);
      const int i_first = sg.j0 + (((grp - sg.j0) % NACC) + NACC) % NACC + (ahead ? NACC : 0);
      // this group's steps i = i_first, i_first + NACC, ... < i_end; K-step k = k_lo + i - j0
      {
        BlockLoad bq[DENSE ? 1 : PREFETCH];   // the group's next PREFETCH K-steps
        DenseLoad dnext;
        if (DENSE) {
          fetch_dense(sg.k_lo + i_first - sg.j0, i_first < i_end, sg.nb0, dnext);
        } else {
#pragma unroll
          for (int j = 0; j < PREFETCH; ++j)
            fetch(sg.k_lo + i_first + j * NACC - sg.j0, i_first + j * NACC < i_end, sg.nb0, bq[j]);
        }
        for (int i = i_first; i < i_end && !dead; i += NACC) {
          const int k = sg.k_lo + (i - sg.j0);
          BlockLoad cur{};
          DenseLoad dcur;
          if (DENSE) {
            dcur = dnext;
            fetch_dense(k + NACC, i + NACC < i_end, sg.nb0, dnext);
          } else {
            cur = bq[0];
#pragma unroll
            for (int j = 0; j + 1 < (DENSE ? 1 : PREFETCH); ++j) bq[j] = bq[j + 1];
            fetch(k + PREFETCH * NACC, i + PREFETCH * NACC < i_end, sg.nb0, bq[(DENSE ? 1 : PREFETCH) - 1]);
          }
          if (!emit(i, k, sg.nb0, cur, dcur)) dead = true;
        }
      }
      // The next tile's first step of this group goes into its slot now, while
      // the tensor cores finish this tile: the next tile's MMAs can start as
      // soon as the accumulators are read.  (The slots of the following
      // D_STAGES - NACC steps hold the epilogue's staging meanwhile.)
      ahead = false;
      if (seg + 1 < nseg && !dead) {
        const Seg nx = segment(seg + 1);
        const int ia = nx.j0 + (((grp - nx.j0) % NACC) + NACC) % NACC;
        if (ia < seg_end(nx)) {
          const int ka = nx.k_lo + (ia - nx.j0);
          BlockLoad b{};
          DenseLoad d;
          if (DENSE)
            fetch_dense(ka, true, nx.nb0, d);
          else
            fetch(ka, true, nx.nb0, b);
          if (emit(ia, ka, nx.nb0, b, d))
            ahead = true;
          else
            dead = true;
        }
      }

      // ---------------------------------------------------------- segment epilogue (each CTA, its rows)
      // Every decode warp passes here once per segment, also after giving up,
      // so that the named barriers below always meet.
      // epilogue geometry: warp quarter q reads TMEM lanes 32 q .. + 31;
      // NACC 1: the two warps of a quarter split the 256 columns;
      // NACC 2: decode group g drains accumulator g (256 columns).
      const int quarter = warp & 3;
      const int acc = NACC == 1 ? 0 : (dwarp >> 2);
      const int col_begin = NACC == 1 ? (dwarp >> 2) * 128 : 0;
      const int nchunk = NACC == 1 ? 4 : 8;
      // A piece is laid out by thread: float4 group g (columns 4g .. 4g + 3) of
      // lane l of warp quarter q of accumulator a at float4 index
      // ((a * 4 + q) * 64 + g) * 32 + l, so that a warp writes and reads 512
      // contiguous bytes per instruction.
      constexpr int64_t kPart = static_cast<int64_t>(NACC) * 128 * 256;   // fp32 of one rank's piece
      auto piece_at = [&](int un, int which) {
        return reinterpret_cast<float4 *>(p.sk_part + (static_cast<int64_t>(un * 2 + which) * 2 + rank) * kPart) +
               (acc * 4 + quarter) * 64 * 32 + lane;
      };
      // The bf16 rows go out through shared memory in 32 x 64 boxes, one TMA
      // store each: after the cluster's last tile all of a warp's boxes fit in
      // the (then idle) activation ring; before that the ring holds the next
      // tile's activations, and each warp takes one 4 KB box in the operand
      // slots of the D_STAGES - NACC steps after the early ones, reused box by box.
      const bool last = seg + 1 == nseg;
      constexpr int kStageSlots = D_STAGES - NACC;
      constexpr int kWarpsPerSlot = (NUM_DEC_WARPS + kStageSlots - 1) / kStageSlots;
      static_assert(kStageSlots >= 1 && kWarpsPerSlot * 4096 <= D_BYTES, "staging boxes fit the free operand slots");
      const uint32_t stage =
          last ? smem_addr(a_ring) + dwarp * (NACC == 1 ? 8192 : 16384)
               : smem_addr(d_ring + ((i_end + NACC + dwarp / kWarpsPerSlot) % D_STAGES) * D_BYTES) +
                     (dwarp % kWarpsPerSlot) * 4096;
      bool ok = false;
      if (!dead) {
        ok = mbar_wait(&sm->acc_full, seg & 1, kDrainLimit);
        if (!ok) latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
      }
      tc_fence_after();
      ok = __all_sync(0xffffffffu, ok) && *abort_flag == 0;
      // A tile shared by P stream-K units: the CTA that finishes its piece last
      // adds the others' fp32 pieces to its own in piece order (the same sum
      // whoever arrives last) and writes the tile; the others write their piece.
      int P = 1, fu = 0;
      int64_t tb_sk = 0;
      if (t >= p.dp_tiles) {
        tb_sk = static_cast<int64_t>(t - p.dp_tiles) * ns;
        fu = sk_unit_of(p, tb_sk);
        P = sk_unit_of(p, tb_sk + ns - 1) - fu + 1;
      }
      int role = 0;                           // 0 whole tile, 1 piece writer, 2 finisher, -1 nothing
      if (P > 1) {
        const int ti = (t - p.dp_tiles) * 2 + static_cast<int>(rank);
        if (threadIdx.x == 64) *sk_role = ok ? atomicAdd(p.sk_count + ti, 1) : -1;
        named_bar_sync(1, 32 * NUM_DEC_WARPS);
        const int arrived = *sk_role;
        role = arrived < 0 ? -1 : (arrived == P - 1 ? 2 : 1);
        if (role == 1) {
          float4 *dst = piece_at(unit, seg == n_dp ? 0 : 1);
          if (ok) {
            for (int cc = 0; cc < nchunk; ++cc) {
              const int col0 = col_begin + cc * 32;
              uint32_t v[32];
              tmem_ld_32x32b_x32(tmem + 256 * acc + (static_cast<uint32_t>(quarter * 32) << 16) + col0, v);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 8; ++j)
                __stcg(dst + (col0 / 4 + j) * 32, make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                              __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
            }
          }
          named_bar_sync(1, 32 * NUM_DEC_WARPS);
          if (threadIdx.x == 64) red_release_gpu_add(p.sk_ready + ti, 1);
        } else if (role == 2) {
          if (threadIdx.x == 64) {
            // the other pieces' CTAs have counted themselves in: they are running and
            // write their pieces now, so this wait is short and cannot depend on a
            // cluster that has not started
            int good = 1;
            if (ld_acquire_gpu(p.sk_ready + ti) < P - 1) {
              const long long t0 = clock64();
              while (ld_acquire_gpu(p.sk_ready + ti) < P - 1) {
                if (static_cast<uint64_t>(clock64() - t0) > p.wait_limit) {
                  latch_status(p.status, QLORA_ERR_DEVICE_TIMEOUT);
                  good = 0;
                  break;
                }
              }
            }
            *sk_ok = good;
          }
          named_bar_sync(1, 32 * NUM_DEC_WARPS);
          if (!*sk_ok) role = -1;
        } else {
          // every path passes two barriers, so that the role word is read by all
          // before the next shared tile's arrival overwrites it
          named_bar_sync(1, 32 * NUM_DEC_WARPS);
        }
      }
      if (ok && (role == 0 || role == 2)) {
        const int own = unit - fu;
        const int64_t orow0 = static_cast<int64_t>(sg.mbase) + 256 * acc + quarter * 32;
        for (int cc = 0; cc < nchunk; ++cc) {
          const int col0 = col_begin + cc * 32;
          uint32_t v[32];
          if (role == 0) {
            tmem_ld_32x32b_x32(tmem + 256 * acc + (static_cast<uint32_t>(quarter * 32) << 16) + col0, v);
            tmem_ld_wait();
          } else {
            // the pieces in order: this CTA's own from TMEM, the others' from the workspace
            float sum[32];
            for (int pc = 0; pc < P; ++pc) {
              if (pc == own) {
                tmem_ld_32x32b_x32(tmem + 256 * acc + (static_cast<uint32_t>(quarter * 32) << 16) + col0, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) sum[j] = pc == 0 ? __uint_as_float(v[j]) : sum[j] + __uint_as_float(v[j]);
              } else {
                const int un = fu + pc;
                const float4 *src = piece_at(un, sk_begin(p.sk_steps, p.sk_units, un) >= tb_sk ? 0 : 1) + (col0 / 4) * 32;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  float4 f[4];
#pragma unroll
                  for (int j = 0; j < 4; ++j) f[j] = __ldcg(src + (4 * h + j) * 32);
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const int e = 16 * h + 4 * j;
                    sum[e] = pc == 0 ? f[j].x : sum[e] + f[j].x;
                    sum[e + 1] = pc == 0 ? f[j].y : sum[e + 1] + f[j].y;
                    sum[e + 2] = pc == 0 ? f[j].z : sum[e + 2] + f[j].z;
                    sum[e + 3] = pc == 0 ? f[j].w : sum[e + 3] + f[j].w;
                  }
                }
              }
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(sum[j]);
          }
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
          {
            // 128B-swizzled rows of a 32 x 64 box; one TMA store per box
            const uint32_t box = last ? stage + (cc >> 1) * 4096 : stage;
            if (!last && cc > 0 && (cc & 1) == 0) {
              if (lane == 0) bulk_wait_read<0>();   // the previous box has been read out
              __syncwarp();
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t c = static_cast<uint32_t>((cc & 1) * 4 + j);
              st_shared_v4(box + lane * 128 + ((c ^ static_cast<uint32_t>(lane & 7)) << 4), pk[4 * j], pk[4 * j + 1],
                           pk[4 * j + 2], pk[4 * j + 3]);
            }
            if (cc & 1) {
              fence_proxy_async_smem();
              __syncwarp();
              const int64_t x = static_cast<int64_t>(sg.n0) + col_begin + (cc >> 1) * 64;
              if (lane == 0 && orow0 < p.M && x < p.n_out) {
                tma_store_2d(&tm_out, box, static_cast<int>(x), static_cast<int>(orow0));
                bulk_commit();
              }
            }
          }
        }
        // the stores have read the staged rows before the shared memory is reused or released
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      if (!last) {
        // every warp's boxes are out of the operand slots before they are decoded into
        named_bar_sync(1, 32 * NUM_DEC_WARPS);
        // the next segment's MMAs overwrite the accumulators once both CTAs have read them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(&sm->tmem_empty);
          else
            mbar_arrive_cluster(mapa_shared(smem_addr(&sm->tmem_empty), 0));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();        // the peer is done with this CTA's shared memory and TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

constexpr size_t kSkCounterBytes = 2 * 2 * kSkMaxUnits * sizeof(int);   // count and ready, per tile and rank

// Clusters of this kernel that fit on the device at once (cached per device).
template <typename Kern>
int cluster_slots(Kern kern, cudaLaunchConfig_t cfg) {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  int v = cache[dev].load();
  if (v == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    v = n > 0 ? n : -1;
    cache[dev].store(v);
  }
  return v > 0 ? v : 0;
}

// Whether a launch splits the K-steps of its last, partial round of tiles over
// all cluster slots (stream-K), and how.
struct SplitPlan {
  bool split = false;
  int tail = 0, units = 0;
  int64_t sk_steps = 0;
};
SplitPlan split_plan(const QGemmArgs &a, int tiles, int ns, int slots) {
  SplitPlan sp;
  const int mode = stream_k_mode();
  sp.tail = slots > 0 && a.sk_ws && mode != QLORA_STREAM_K_OFF ? tiles % slots : 0;
  sp.sk_steps = static_cast<int64_t>(sp.tail) * ns;
  sp.units = static_cast<int>(std::min<int64_t>(slots, std::max<int64_t>(1, sp.sk_steps / kSkMinSteps)));
  sp.split = sp.tail > 0 && (mode == QLORA_STREAM_K_ALWAYS ||
                             ceil_div(sp.sk_steps, sp.units) + kSkCostSteps < ns + kTileCostSteps);
  return sp;
}

// Tiles and K-steps per tile of a pair launch (as launch_qgemm_pair sets them).
void pair_shape(const QGemmArgs &a, int *tiles, int *ns) {
  const int64_t kred = a.dgrad ? a.wN : a.wK;
  const int64_t n_out = a.dgrad ? a.wK : a.wN;
  const int nacc = a.M > 2 * BM ? 2 : 1;
  const int bk = nacc == 2 ? Cfg<2>::BK : Cfg<1>::BK;
  *ns = static_cast<int>(ceil_div(kred, bk) + ceil_div(a.r, bk));
  *tiles = static_cast<int>(ceil_div(a.M, 2 * BM * nacc) * ceil_div(n_out, BN));
}

}  // namespace

qlora_status qgemm_prepare_split(const QGemmArgs &a, cudaStream_t st, bool *zeroed) {
  *zeroed = false;
  if (!(a.M > kPairMinRows || a.wdense) || !a.sk_ws) return QLORA_OK;   // no stream-K tail on this launch
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // every instance of the pair kernel has the same shape of resources; the slot count is cached
  if (cudaFuncSetAttribute(qgemm2_kernel<false, 2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess)
    return QLORA_ERR_CUDA;
  const int slots = std::min(cluster_slots(qgemm2_kernel<false, 2, false>, cfg), kSkMaxUnits);
  int tiles, ns;
  pair_shape(a, &tiles, &ns);
  if (!split_plan(a, tiles, ns, slots).split) return QLORA_OK;
  if (cudaMemsetAsync(a.sk_ws, 0, kSkCounterBytes, st) != cudaSuccess) return QLORA_ERR_CUDA;
  *zeroed = true;
  return QLORA_OK;
}

size_t pair_sk_workspace_bytes(int64_t M) {
  const int64_t nacc = M > 2 * BM ? 2 : 1;
  return kSkCounterBytes + static_cast<size_t>(kSkMaxUnits) * 2 * 2 * nacc * 128 * 256 * sizeof(float);
}

qlora_status launch_qgemm_pair(const QGemmArgs &a, cudaStream_t st) {
  CUtensorMap tm_act, tm_lact, tm_out;
  const int64_t kred = a.dgrad ? a.wN : a.wK;
  const int64_t n_out = a.dgrad ? a.wK : a.wN;
  bool ok = make_tmap_2d(&tm_act, a.act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kred, a.M, kred * 2, 64, BM,
                         CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_tmap_2d(&tm_lact, a.lora_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.r, a.M,
                          static_cast<uint64_t>(a.r) * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  // the output, written from shared memory in 32-row x 64-column boxes
  ok = ok && make_tmap_2d(&tm_out, a.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, n_out, a.M,
                          static_cast<uint64_t>(n_out) * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return QLORA_ERR_CUDA;

  Params p{};
  p.M = a.M;
  p.n_out = n_out;
  p.ldo = n_out;
  p.wN = a.wN;
  p.wK = a.wK;
  p.codes = a.codes;
  p.absmax_q = a.absmax_q;
  p.group_scale = a.group_scale;
  p.lora_w = a.lora_w;
  p.wdense = a.wdense;
  p.r = a.r;
  p.out = a.out;
  p.status = device_status_ptr();
  p.wait_limit = wait_limit();
  if (!p.status) return QLORA_ERR_CUDA;

  // two accumulators per CTA (512-row pair tile) once M fills them
  const int nacc = a.M > 2 * BM ? 2 : 1;
  const int bk = nacc == 2 ? Cfg<2>::BK : Cfg<1>::BK;
  p.nkb = static_cast<int>(ceil_div(kred, bk));
  p.nls = static_cast<int>(ceil_div(a.r, bk));
  p.ns = p.nkb + p.nls;
  p.num_m = static_cast<int>(ceil_div(a.M, 2 * BM * nacc));
  p.num_n = static_cast<int>(ceil_div(n_out, BN));
  const int tiles = p.num_m * p.num_n;
  p.dp_tiles = tiles;
  // Raster: a wave of kGroupM-row groups touches every M-pair, so an activation
  // too large to stay in L2 is read from DRAM once per round of tiles (about
  // 2.6 times for the 90 MB operands at 1.73 rounds), while each weight tile is
  // read about once.  Walking one M-pair's tiles at a time reads the activation
  // about once and the (packed, smaller) weight once per round instead.
  const double act_bytes = static_cast<double>(a.M) * static_cast<double>(kred) * 2.0;
  const double w_bytes = static_cast<double>(a.wN) * static_cast<double>(a.wK) * (a.wdense ? 2.0 : 0.5);
  p.group_m = QLORA_PAIR_RASTER_AUTO && act_bytes >= 64.0 * (1 << 20) && act_bytes > 2.0 * w_bytes ? 1 : kGroupM;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);        // set per launch below (the occupancy query reads the rest)
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;             // the occupancy query sees the cluster shape only
  const Nf4Table tab = a.tab;
  const int kind = a.dgrad ? kProfGemmDgrad : kProfGemmFwd;
  auto go = [&](auto kern) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    // Persistent clusters: as many as fit on the device at once (one per tile
    // when that is not known), each taking tiles cid, cid + C, ...  The tiles
    // of a last, partial round can instead have their K-steps split evenly over
    // all clusters (stream-K), so that no cluster idles while others finish.
    const int slots = std::min(cluster_slots(kern, cfg), kSkMaxUnits);
    int clusters = slots > 0 ? std::min(tiles, slots) : tiles;
    const SplitPlan sp = split_plan(a, tiles, p.ns, slots);
    if (sp.split) {
      p.dp_tiles = tiles - sp.tail;
      p.sk_steps = sp.sk_steps;
      p.sk_units = sp.units;
      p.sk_count = static_cast<int *>(a.sk_ws);
      p.sk_ready = p.sk_count + 2 * kSkMaxUnits;
      p.sk_part = reinterpret_cast<float *>(static_cast<char *>(a.sk_ws) + kSkCounterBytes);
      clusters = p.dp_tiles > 0 ? slots : sp.units;
      if (!a.sk_zeroed) {
        e = cudaMemsetAsync(a.sk_ws, 0, kSkCounterBytes, st);
        if (e != cudaSuccess) return e;
      }
    }
    cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters));
    prof_mark(kind, true, st);
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, tm_act, tm_lact, tm_out, p, tab);
    cfg.numAttrs = 1;
    prof_mark(kind, false, st);
    return e;
  };
  cudaError_t e;
  if (a.wdense) {
    if (a.dgrad)
      e = nacc == 2 ? go(qgemm2_kernel<true, 2, true>) : go(qgemm2_kernel<true, 1, true>);
    else
      e = nacc == 2 ? go(qgemm2_kernel<false, 2, true>) : go(qgemm2_kernel<false, 1, true>);
  } else if (a.dgrad) {
    e = nacc == 2 ? go(qgemm2_kernel<true, 2, false>) : go(qgemm2_kernel<true, 1, false>);
  } else {
    e = nacc == 2 ? go(qgemm2_kernel<false, 2, false>) : go(qgemm2_kernel<false, 1, false>);
  }
  return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

}  // namespace qlora
