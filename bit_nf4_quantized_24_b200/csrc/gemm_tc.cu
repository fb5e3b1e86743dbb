// Fused NF4-dequant GEMM on the sm_100a tensor cores (tcgen05 + TMEM), run by
// pairs of CTAs on two SMs (cta_group::2).
//
// katajob, "NF4: 4-bit NormalFloat": the 4-bit weight is expanded block by
// block to bf16 only for the product and thrown away afterwards.  Here the
// expanded weight tile exists only in shared memory, one pipeline stage at a
// time, as the B operand of tcgen05.mma.
//
//   mode 0, forward:  D[m, n] = sum_k X[m,k] W'[n,k]       (W' K-major)
//   mode 1, dX:       D[m, k] = sum_n dY[m,n] W'[n,k]      (W' MN-major)
// followed by one tail stage that adds the LoRA product from bf16 operands
// loaded by TMA: Hs B^T (forward, Hs = s*H) or dH A (dX).
//
// Tiling.  A cluster of 2 CTAs (one per SM) computes 512 tokens x 256 outputs.
// Each CTA owns 256 tokens (its A tile, two 128-row halves) and expands half of
// the 256-row weight tile (128 rows) into its own shared memory.  The leader
// CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): the MMA
// reads the A rows and the B half of both CTAs and writes 128 x 256 fp32 into
// each CTA's TMEM.  Two such MMAs per k16 step (one per A half) fill all 512
// TMEM columns of both SMs.  Per SM this halves the dequantization work and
// the B-operand shared-memory traffic of a single-CTA tile of the same size.
//
// Warp roles (576 threads per CTA):
//   warp 0       TMA producer: NF4 code tiles into an 8-deep ring, CAHEAD
//                stages ahead of the activation tiles (4-deep ring)
//   warp 1       TMEM allocation (both CTAs); MMA issue (leader only)
//   warps 2..17  dequantizers in four groups of four that take every fourth
//                stage (one 64-weight block per thread per stage: register
//                lookup table -> 128 B of swizzled bf16 in smem); the scale
//                of each block is loaded eight stages ahead.  They signal the
//                leader's barrier (the peer remotely), then run the epilogue.
// Every wait is bounded (kWaitLimitNs); on expiry the kernel records
// kDevTimeout, drains what it issued, frees TMEM and exits.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "internal.h"

namespace qn {

namespace {

constexpr int BM = 256;              // tokens per CTA (two MMA halves of 128)
constexpr int UM = 128;              // rows of A each CTA gives one pair MMA
constexpr int BN = 256;              // outputs per pair (N of the MMA)
constexpr int BNL = BN / 2;          // outputs expanded by each CTA
constexpr int BK = 64;
constexpr int STAGES = 4;             // activation (A) and expanded-weight (B) ring
constexpr int CSTAGES = 8;            // NF4 code ring: codes run CAHEAD stages ahead of A
constexpr int CAHEAD = 4;
constexpr int DQ_GROUPS = 4;         // dequant groups of 4 warps (128 threads)
constexpr int A_BYTES = BM * BK * 2;     // 32 KB
constexpr int B_BYTES = BNL * BK * 2;    // 16 KB
constexpr int C_BYTES = BNL * BK / 2;    // 4 KB of packed codes
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
constexpr int OFF_C = OFF_B + STAGES * B_BYTES;
constexpr int OFF_BAR = OFF_C + CSTAGES * C_BYTES;
constexpr int SMEM_USED = OFF_BAR + 256;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;  // slack for 1024-byte alignment
constexpr int NUM_THREADS = 64 + DQ_GROUPS * 128;
constexpr int TMEM_COLS = 512;  // accumulator h at columns 256h .. 256h+255

static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

struct Bars {
  uint64_t full_tma[STAGES];  // this CTA's activation tile (or tail tiles) landed
  uint64_t full_deq[STAGES];  // leader: both CTAs' A tiles landed and B halves written
  uint64_t empty[STAGES];     // MMAs of the stage completed (multicast by the leader)
  uint64_t full_c[CSTAGES];   // this CTA's code tile landed
  uint64_t empty_c[CSTAGES];  // this CTA's dequantizers finished with a code tile
  uint64_t accum;             // all MMAs completed (multicast by the leader)
  uint64_t drain;             // leader: used only when aborting
  uint64_t dealloc;           // the other CTA finished with the pair's TMEM
  uint32_t tmem_base;
  int abort;
};

// Work items of a launch: whole tiles first, then nsplit pieces of each of
// the last ntail tiles (the tiles that would otherwise form a partial last
// wave on the resident CTA pairs).
struct SplitGrid {
  int npairs, nout_tiles;  // token pairs and output tiles (tiles = npairs * nout_tiles)
  int nwhole, ntail, nsplit;
};

// GEN = false: the default NF4 format (64-weight blocks, double quantization
// over groups of 256 blocks).  GEN = true: 2^lg-weight blocks (lg = 5..8),
// double quantization on or off (dq), chosen at run time; a thread's 64
// consecutive weights then lie in one block, or in two when blocks hold 32.
template <int MODE, bool GEN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_nf4_gemm(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_codes,
               const __grid_constant__ CUtensorMap tm_tail_a, const __grid_constant__ CUtensorMap tm_tail_b,
               const uint8_t* __restrict__ absmax_q, const float* __restrict__ dq_scale, Nf4Levels lv, int M, int N,
               int K, int r, int band_pairs, int lg, int dq, __nv_bfloat16* __restrict__ out, int* status,
               SplitGrid sg, float* __restrict__ part) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  Bars* bars = reinterpret_cast<Bars*>(base_ptr + OFF_BAR);
  const uint32_t bar0 = base + OFF_BAR;
  auto full_tma = [&](int s) { return bar0 + 8u * s; };
  auto full_deq = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto full_c = [&](int c) { return bar0 + 8u * (3 * STAGES + c); };
  auto empty_c = [&](int c) { return bar0 + 8u * (3 * STAGES + CSTAGES + c); };
  const uint32_t accum_bar = bar0 + 8u * (3 * STAGES + 2 * CSTAGES);
  const uint32_t drain_bar = accum_bar + 8u;
  const uint32_t dealloc_bar = accum_bar + 16u;
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  // mode 0: contraction K, outputs N.  mode 1: contraction N, outputs K.
  const int Kc = MODE == 0 ? K : N;
  const int Nout = MODE == 0 ? N : K;
  const int numK = (Kc + BK - 1) / BK;
  // Work item blockIdx.x / 2: items below sg.nwhole are whole tiles (tile L =
  // item); the rest are pieces of the last sg.ntail tiles, sg.nsplit per tile,
  // piece z taking the z-th of nsplit contiguous ranges of K stages (the last
  // piece also the LoRA stage) and leaving fp32 partial sums for the reduction
  // kernel.  Tiles are handed out band by band: a band of `band_pairs` token
  // pairs sweeps every output tile before the next band starts, so the band's
  // activations stay in L2 while the weight tiles stream past them.
  int pair, otile, zpiece = 0, nsplit = 1, tail_idx = 0;
  {
    const int item = blockIdx.x >> 1;
    int L = item;
    if (item >= sg.nwhole) {
      const int j = item - sg.nwhole;
      nsplit = sg.nsplit;
      tail_idx = j / nsplit;
      zpiece = j - tail_idx * nsplit;
      L = sg.nwhole + tail_idx;
    }
    const int npx = sg.npairs, nout = sg.nout_tiles;
    const int per_band = band_pairs * nout;
    const int band = L / per_band, rem = L - band * per_band;
    const int in_band = min(band_pairs, npx - band * band_pairs);
    otile = rem / in_band;
    pair = band * band_pairs + (rem - otile * in_band);
  }
  const int kbeg = (zpiece * numK) / nsplit, kend = ((zpiece + 1) * numK) / nsplit;
  const int nloc = kend - kbeg;                  // K stages of this item
  const bool has_tail = zpiece == nsplit - 1;    // it also runs the LoRA stage
  const int nstage = nloc + (has_tail ? 1 : 0);  // ring iterations
  const int n0 = otile * BN;                            // first output of the pair's tile
  const int nl0 = n0 + BNL * static_cast<int>(rank);    // first output this CTA expands
  const int m0 = (2 * pair + static_cast<int>(rank)) * BM;  // first token of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_tma(s), 1);
      mbar_init(full_deq(s), 2 * 4);  // the stage group's 4 warps in each CTA
      mbar_init(empty(s), 1);
    }
    for (int c = 0; c < CSTAGES; ++c) {
      mbar_init(full_c(c), 1);
      mbar_init(empty_c(c), 4);  // the 4 warps of the iteration's dequant group
    }
    mbar_init(accum_bar, 1);
    mbar_init(drain_bar, 1);
    mbar_init(dealloc_bar, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_tail_a);
    tma_prefetch_desc(&tm_tail_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(base + OFF_BAR + static_cast<uint32_t>(offsetof(Bars, tmem_base)), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer
    // Code tiles run CAHEAD iterations ahead of the activation tiles, so the
    // expansion of a stage overlaps the latency of its activation tile.
    if (lane == 0) {
      int a_issued = 0, c_issued = 0;
      bool ok = true;
      // it: the item's ring iteration; the K stage it loads is kbeg + it
      auto issue_codes = [&](int it) {
        const int c = it % CSTAGES;
        if (!(ok = wait_bounded(empty_c(c), ((it / CSTAGES) & 1) ^ 1, abort, status))) return;
        mbar_arrive_expect_tx(full_c(c), C_BYTES);
        if (MODE == 0)
          tma_load_2d(base + OFF_C + c * C_BYTES, &tm_codes, full_c(c), (kbeg + it) * (BK / 2), nl0);
        else
          tma_load_2d(base + OFF_C + c * C_BYTES, &tm_codes, full_c(c), nl0 / 2, (kbeg + it) * BK);
        ++c_issued;
      };
      for (int it = 0; it < CAHEAD && it < nloc && ok; ++it) issue_codes(it);
      for (int it = 0; it < nloc && ok; ++it) {
        if (it + CAHEAD < nloc) {
          issue_codes(it + CAHEAD);
          if (!ok) break;
        }
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!(ok = wait_bounded(empty(s), ph ^ 1, abort, status))) break;
        mbar_arrive_expect_tx(full_tma(s), A_BYTES);
        tma_load_2d(base + OFF_A + s * A_BYTES, &tm_act, full_tma(s), (kbeg + it) * BK, m0);
        ++a_issued;
      }
      // The tail operands come from the previous kernel of the stream, which
      // may still be running (programmatic dependent launch); every other
      // input of this kernel predates it.  Waited for on every path, so that
      // this grid completes only after its predecessor.
      pdl_wait();
      if (ok && has_tail) {  // tail stage: LoRA operands
        const int it = nloc, s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if ((ok = wait_bounded(empty(s), ph ^ 1, abort, status))) {
          mbar_arrive_expect_tx(full_tma(s), A_BYTES + B_BYTES);
          tma_load_2d(base + OFF_A + s * A_BYTES, &tm_tail_a, full_tma(s), 0, m0);
          if (MODE == 0) {
            tma_load_2d(base + OFF_B + s * B_BYTES, &tm_tail_b, full_tma(s), 0, nl0);
          } else {
#pragma unroll
            for (int j = 0; j < BNL / 64; ++j)
              tma_load_2d(base + OFF_B + s * B_BYTES + j * 8192, &tm_tail_b, full_tma(s), nl0 + 64 * j, 0);
          }
          ++a_issued;
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (int it = (a_issued > STAGES ? a_issued - STAGES : 0); it < a_issued; ++it)
          wait_drain(full_tma(it % STAGES), (it / STAGES) & 1);
        for (int it = (c_issued > CSTAGES ? c_issued - CSTAGES : 0); it < c_issued; ++it)
          wait_drain(full_c(it % CSTAGES), (it / CSTAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (leader && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * UM, BN, false, MODE == 1);
      bool ok = true;
      int committed = 0;
      for (int it = 0; it < nstage; ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const bool tail = (it == nloc);
        // full_deq gathers both CTAs: their tiles landed and their B halves are written
        if (!(ok = wait_bounded_cluster(full_deq(s), ph, abort, status))) break;
        tc_fence_after();
        const uint32_t a_s = base + OFF_A + s * A_BYTES;
        const uint32_t b_s = base + OFF_B + s * B_BYTES;
        const int nk = tail ? (r + 15) / 16 : BK / 16;
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t bd = MODE == 0 ? desc_sw128(b_s + kk * 32, 16, 1024)
                                        : desc_sw128(b_s + kk * 2048, 8192, 1024);
          const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
          tc_mma_f16_pair(tmem, desc_sw128(a_s + kk * 32, 16, 1024), bd, idesc, acc);
          tc_mma_f16_pair(tmem + 256, desc_sw128(a_s + UM * 128 + kk * 32, 16, 1024), bd, idesc, acc);
        }
        tc_commit_pair(empty(s));
        committed = 1;
      }
      if (ok) {
        tc_commit_pair(accum_bar);
      } else if (committed) {  // wait for MMAs in flight before TMEM is freed
        tc_commit_pair(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
  } else {
    // ------------------------------------------- dequantizers, then epilogue
    const int e = warp - 2;             // 0..15
    const int grp = e >> 2;             // stages it = grp, grp + 4, ...
    const int t = (e & 3) * 32 + lane;  // item of the stage: 0..127
    const uint32_t deq_bar_leader0 = mapa_shared(full_deq(0), 0);
    bool ok = true;
    const int KB = K / 64;              // 64-blocks per weight row
    // which (row, 64-block) of W this thread expands at iteration it; its
    // expansion goes to row t of this CTA's B stage
    auto item_of = [&](int it, int& wrow, int& kcol0) {
      if (MODE == 0) {
        wrow = nl0 + t;
        kcol0 = it * BK;
      } else {
        wrow = it * BK + (t & 63);
        kcol0 = nl0 + 64 * (t >> 6);  // smem row t = 64 * (t >> 6) + (t & 63)
      }
    };
    // Raw scale parts of the (one or two) blocks of a thread's 64 weights,
    // loaded two iterations ahead and combined only when used.
    struct Scale {
      uint32_t q0, q1;
      float s0, s1;
      bool valid;
    };
    auto fetch = [&](int it) {
      Scale sc{0u, 0u, 0.0f, 0.0f, false};
      if (it < nloc) {
        int wrow, kcol0;
        item_of(kbeg + it, wrow, kcol0);
        if (wrow < N && kcol0 < K) {
          if (!GEN) {
            const int64_t blk = static_cast<int64_t>(wrow) * KB + (kcol0 >> 6);
            sc.q0 = __ldg(absmax_q + blk);
            sc.s0 = __ldg(dq_scale + (blk >> 8));
          } else {
            const int64_t blk = (static_cast<int64_t>(wrow) * K + kcol0) >> lg;
            if (dq) {
              sc.q0 = __ldg(absmax_q + blk);
              sc.s0 = __ldg(dq_scale + (blk >> 8));
              if (lg == 5) {
                sc.q1 = __ldg(absmax_q + blk + 1);
                sc.s1 = __ldg(dq_scale + ((blk + 1) >> 8));
              }
            } else {
              sc.s0 = __ldg(dq_scale + blk);
              if (lg == 5) sc.s1 = __ldg(dq_scale + blk + 1);
            }
          }
          sc.valid = true;
        }
      }
      return sc;
    };
    Scale p0 = fetch(grp), p1 = fetch(grp + DQ_GROUPS);
    for (int it = grp; it < nstage; it += DQ_GROUPS) {  // it == nloc: the tail stage
      const Scale p2 = fetch(it + 2 * DQ_GROUPS);
      const int s = it % STAGES;
      const uint32_t ph = (it / STAGES) & 1;
      if (it < nloc) {
        const int cs = it % CSTAGES;
        if (!(ok = wait_bounded(full_c(cs), (it / CSTAGES) & 1, abort, status))) break;
        const uint32_t c_s = base + OFF_C + cs * C_BYTES;
        uint4 q0, q1;
        if (MODE == 0) {  // code tile [128 rows][32 B], 32-byte swizzle
          const uint32_t sw = (static_cast<uint32_t>(t) >> 2) & 1u;
          q0 = ld_shared_v4(c_s + t * 32 + ((0u ^ sw) << 4));
          q1 = ld_shared_v4(c_s + t * 32 + ((1u ^ sw) << 4));
        } else {          // code tile [64 rows][64 B], 64-byte swizzle
          const uint32_t row = t & 63, j = t >> 6, sw = (row >> 1) & 3u;
          q0 = ld_shared_v4(c_s + row * 64 + (((2 * j) ^ sw) << 4));
          q1 = ld_shared_v4(c_s + row * 64 + (((2 * j + 1) ^ sw) << 4));
        }
        // the B slot is free once the MMAs of iteration it - STAGES completed
        if (!(ok = wait_bounded(empty(s), ph ^ 1, abort, status))) break;
        const uint32_t b_row = base + OFF_B + s * B_BYTES + t * 128;
        const uint32_t sw = t & 7;
        if (p0.valid) {
          const float a0 = (GEN && !dq) ? p0.s0 : __fmul_rn(static_cast<float>(p0.q0), p0.s0);
          const Nf4Lut lut = make_lut(lv, a0);
          const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          if (GEN && lg == 5) {  // two 32-weight blocks: words 0-3 and 4-7
            const float a1 = dq ? __fmul_rn(static_cast<float>(p0.q1), p0.s1) : p0.s1;
            const Nf4Lut lut1 = make_lut(lv, a1);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o0, o1, o2, o3;
              deq8(w[c], c < 4 ? lut : lut1, o0, o1, o2, o3);
              st_shared_v4(b_row + ((c ^ sw) << 4), o0, o1, o2, o3);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o0, o1, o2, o3;
              deq8(w[c], lut, o0, o1, o2, o3);
              st_shared_v4(b_row + ((c ^ sw) << 4), o0, o1, o2, o3);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) st_shared_v4(b_row + (c << 4), 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_c(cs));  // code tile consumed (values are in registers)
      }
      // the stage's activation tile (or the tail tiles) must have landed too
      if (!(ok = wait_bounded(full_tma(s), ph, abort, status))) break;
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(full_deq(s));
        else mbar_arrive_remote(deq_bar_leader0 + 8u * s);
      }
      p0 = p1;
      p1 = p2;
    }

    // -------------------------------------------------------- epilogue
    if (ok) ok = wait_bounded(accum_bar, 0, abort, status);
    if (ok) {
      tc_fence_after();
      const int quad = warp & 3;                 // TMEM lanes 32*quad .. +31
      const int h = (e >> 2) & 1;                // accumulator: tokens 128h .. 128h+127
      const int ch = e >> 3;                     // column half of the accumulator
      const int m = m0 + h * UM + quad * 32 + lane;
#pragma unroll 1
      for (int col = ch * (BN / 2); col < (ch + 1) * (BN / 2); col += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(h * 256 + col),
                           v);
        tmem_ld_wait();
        const int n = n0 + col;
        if (nsplit > 1) {  // a piece of a split tile: fp32 partial sums, the whole CTA tile
          float4* dst = reinterpret_cast<float4*>(
              part + ((static_cast<int64_t>(tail_idx) * nsplit + zpiece) * 2 + rank) * (BM * BN) +
              (h * UM + quad * 32 + lane) * BN + col);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
        } else if (m < M && n < Nout) {
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(m) * Nout + n);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (n + 8 * q < Nout) {
              uint4 o;
              o.x = bf16x2_bits(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
              o.y = bf16x2_bits(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
              o.z = bf16x2_bits(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
              o.w = bf16x2_bits(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
              dst[q] = o;
            }
          }
        }
      }
    }
  }

  // Both CTAs must be done with the pair's TMEM before it is freed: each tells
  // the other (remote arrive) and waits for the other's word (bounded).
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      mbar_arrive_remote(mapa_shared(dealloc_bar, rank ^ 1u));
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait_cluster(dealloc_bar, 0)) {
        if (global_timer_ns() - t0 > kWaitLimitNs) {
          atomicExch(status, kDevTimeout);
          break;
        }
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Sum of the split pieces of the last sg.ntail tiles in piece order (fp32),
// rounded once to bf16.  Thread: 8 consecutive outputs of one token row.
// Waits for the GEMM grid (programmatic dependent launch) before reading.
__global__ void __launch_bounds__(256) k_split_reduce(const float* __restrict__ part, SplitGrid sg, int band_pairs,
                                                      int M, int Nout, __nv_bfloat16* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_tile = 2 * BM * (BN / 8);  // 512 rows x 32 groups of 8 outputs
  const int t = static_cast<int>(g / per_tile), w = static_cast<int>(g - static_cast<int64_t>(t) * per_tile);
  if (t >= sg.ntail) return;
  const int row = w / (BN / 8), c8 = (w - row * (BN / 8)) * 8;  // row of the pair tile, first column
  const int L = sg.nwhole + t;
  const int per_band = band_pairs * sg.nout_tiles;
  const int band = L / per_band, rem = L - band * per_band;
  const int in_band = min(band_pairs, sg.npairs - band * band_pairs);
  const int otile = rem / in_band, pair = band * band_pairs + (rem - otile * in_band);
  const int m = pair * 2 * BM + row, n = otile * BN + c8;
  if (m >= M || n >= Nout) return;
  // the partial of piece z: [z][rank = row / 256][row % 256][col]
  const float* src = part + static_cast<int64_t>(t) * sg.nsplit * 2 * (BM * BN) + (row / BM) * (BM * BN) +
                     (row % BM) * BN + c8;
  float4 a = *reinterpret_cast<const float4*>(src), b = *reinterpret_cast<const float4*>(src + 4);
  for (int z = 1; z < sg.nsplit; ++z) {
    const float* q = src + static_cast<int64_t>(z) * 2 * (BM * BN);
    const float4 c = *reinterpret_cast<const float4*>(q), d = *reinterpret_cast<const float4*>(q + 4);
    a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
    b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
  }
  uint4 o;
  o.x = bf16x2_bits(a.x, a.y);
  o.y = bf16x2_bits(a.z, a.w);
  o.z = bf16x2_bits(b.x, b.y);
  o.w = bf16x2_bits(b.z, b.w);
  if (n + 8 <= Nout) {
    *reinterpret_cast<uint4*>(out + static_cast<int64_t>(m) * Nout + n) = o;
  } else {  // ragged last columns (Nout % 8 == 0 keeps this branch unused for valid shapes)
    const uint32_t wv[4] = {o.x, o.y, o.z, o.w};
    for (int i = 0; i < 8 && n + i < Nout; ++i)
      reinterpret_cast<uint16_t*>(out)[static_cast<int64_t>(m) * Nout + n + i] =
          static_cast<uint16_t>(wv[i / 2] >> (16 * (i & 1)));
  }
}

// ------------------------------------------------------------ host side

template <int MODE, bool GEN>
cudaError_t launch_mode(const GemmArgs& a, cudaStream_t st) {
  int lg = 0;
  while ((1 << lg) < a.block) ++lg;
  const int64_t Kc = MODE == 0 ? a.K : a.N;
  const int64_t Nout = MODE == 0 ? a.N : a.K;
  CUtensorMap tm_act, tm_codes, tm_ta, tm_tb;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const auto U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
  bool ok = make_map(&tm_act, BF16, a.act, Kc, a.M, Kc * 2, BK, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (MODE == 0)
    ok = ok && make_map(&tm_codes, U8, a.codes, a.K / 2, a.N, a.K / 2, BK / 2, BNL, CU_TENSOR_MAP_SWIZZLE_32B);
  else
    ok = ok && make_map(&tm_codes, U8, a.codes, a.K / 2, a.N, a.K / 2, BNL / 2, BK, CU_TENSOR_MAP_SWIZZLE_64B);
  ok = ok && make_map(&tm_ta, BF16, a.tail_a, a.r, a.M, a.r * 2, 64, BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (MODE == 0)
    ok = ok && make_map(&tm_tb, BF16, a.tail_b, a.r, a.N, a.r * 2, 64, BNL, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tm_tb, BF16, a.tail_b, a.K, a.r, a.K * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;

  cudaError_t e = smem_limit_once<k_nf4_gemm<MODE, GEN>>(SMEM_ALLOC);
  if (e != cudaSuccess) return e;

  // Token tiles are rounded up to whole pairs: a CTA past the last token
  // feeds zeros (TMA fills out-of-range rows) to its half and stores nothing.
  const SplitPlan plan = gemm_split_plan(MODE, a.M, a.N, a.K);
  const bool split = plan.nsplit > 1 && a.part && a.part_bytes >= plan.part_bytes;
  SplitGrid sg;
  sg.npairs = static_cast<int>(plan.npairs);
  sg.nout_tiles = static_cast<int>(plan.nout_tiles);
  sg.nwhole = static_cast<int>(split ? plan.nwhole : plan.npairs * plan.nout_tiles);
  sg.ntail = split ? static_cast<int>(plan.ntail) : 0;
  sg.nsplit = split ? plan.nsplit : 1;
  const int64_t items = int64_t(sg.nwhole) + int64_t(sg.ntail) * sg.nsplit;
  const dim3 grid(static_cast<unsigned>(2 * items), 1, 1);
  // token pairs per band: keep a band's activations (512 tokens x Kc per pair) near 48 MB
  const int64_t pair_bytes = int64_t(2) * BM * Kc * 2;
  const int band_pairs =
      static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(plan.npairs, (48ll << 20) / pair_bytes)));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;  // the two CTAs of a pair hold consecutive token tiles
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = a.pdl ? 2 : 1;
  trace_before(st);
  e = cudaLaunchKernelEx(&cfg, k_nf4_gemm<MODE, GEN>, tm_act, tm_codes, tm_ta, tm_tb, a.absmax_q, a.dq_scale,
                         host_codebook().levels, static_cast<int>(a.M), static_cast<int>(a.N), static_cast<int>(a.K),
                         a.r, band_pairs, lg, a.dq_block ? 1 : 0, reinterpret_cast<__nv_bfloat16*>(a.out),
                         device_status_ptr(), sg, split ? a.part : nullptr);
  if (e == cudaSuccess && split) {
    const int64_t threads = int64_t(sg.ntail) * 2 * BM * (BN / 8);
    e = launch_ex(k_split_reduce, dim3(static_cast<unsigned>((threads + 255) / 256)), dim3(256), 0, st, true,
                  static_cast<const float*>(a.part), sg, band_pairs, static_cast<int>(a.M), static_cast<int>(Nout),
                  reinterpret_cast<__nv_bfloat16*>(a.out));
  }
  trace_after(st);  // the traced interval covers the reduction of split tiles too
  return e;
}

template <int MODE>
int max_active_pairs() {
  if (smem_limit_once<k_nf4_gemm<MODE, false>>(SMEM_ALLOC) != cudaSuccess) return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_nf4_gemm<MODE, false>, &cfg) != cudaSuccess) return -2;
  return n;
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2D row-major map: inner dimension `inner` elements, `outer` rows, row
// pitch `pitch_bytes`; box {box_inner, box_outer}.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_nf4_gemm(const GemmArgs& a, cudaStream_t st) {
  const bool gen = !(a.block == 64 && a.dq_block == 256);
  if (a.mode == 0) return gen ? launch_mode<0, true>(a, st) : launch_mode<0, false>(a, st);
  return gen ? launch_mode<1, true>(a, st) : launch_mode<1, false>(a, st);
}

int nf4_gemm_max_active_pairs(int mode) { return mode == 0 ? max_active_pairs<0>() : max_active_pairs<1>(); }

// Resident CTA pairs of the current device (cached per device and mode; 0
// when unknown, e.g. without a device).
static int resident_pairs_cached(int mode) {
  constexpr int kDev = 64;
  static std::atomic<int> cache[kDev][2];  // 0: not yet asked; -1: unknown
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kDev) {
    cudaGetLastError();
    return 0;
  }
  int v = cache[d][mode].load(std::memory_order_relaxed);
  if (v == 0) {
    v = nf4_gemm_max_active_pairs(mode);
    if (v <= 0) {
      cudaGetLastError();
      v = -1;
    }
    cache[d][mode].store(v, std::memory_order_relaxed);
  }
  return v > 0 ? v : 0;
}

SplitPlan gemm_split_plan(int mode, int64_t M, int64_t N, int64_t K) {
  SplitPlan p{};
  const int64_t Kc = mode == 0 ? K : N, Nout = mode == 0 ? N : K;
  p.npairs = ((M + BM - 1) / BM + 1) / 2;
  p.nout_tiles = (Nout + BN - 1) / BN;
  const int64_t tiles = p.npairs * p.nout_tiles, numK = (Kc + BK - 1) / BK;
  p.nwhole = tiles;
  p.nsplit = 1;
  const int P = resident_pairs_cached(mode);
  if (P <= 0 || M <= 0) return p;
  const int64_t w = tiles % P;  // tiles of the partial last wave
  if (w == 0) return p;
  // Pieces of S-th of a tile run in ceil(w S / P) rounds after the whole
  // tiles, so the tail takes ceil(w S / P) / S of a tile's numK stages
  // instead of all of them; each piece costs its fp32 partial sums (1 MB
  // written, then read back by the reduction), about 0.16 of a stage's time
  // (a pair runs a 64-deep stage of a 512 x 256 tile in ~1 us at ~1.2 PFLOP/s
  // over 74 pairs; 1 MB moves in ~0.16 us at ~6.4 TB/s).  S maximises the
  // saving, and must save at least 5 % of a tile.  A piece keeps at least 16
  // stages: shorter pieces lose more to the tile's set-up and epilogue than the
  // split gains (measured on the dX of a 1024-output projection, 16 stages per
  // tile: split in two it ran 11 % slower).
  const int64_t smax = std::min<int64_t>(numK / 16, 16);
  int64_t S = 1;
  double best = 0.05 * static_cast<double>(numK);
  for (int64_t c = 2; c <= smax; ++c) {
    const double rounds = static_cast<double>((w * c + P - 1) / P);
    const double save = (1.0 - rounds / static_cast<double>(c)) * static_cast<double>(numK) - 0.16 * w * c;
    if (save > best) {
      best = save;
      S = c;
    }
  }
  if (S < 2) return p;
  p.nsplit = static_cast<int>(S);
  p.ntail = w;
  p.nwhole = tiles - w;
  p.part_bytes = static_cast<size_t>(w * S) * 2 * BM * BN * 4;
  return p;
}

}  // namespace qn
