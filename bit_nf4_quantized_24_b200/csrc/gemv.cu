// Decode-sized forward (M <= 16 tokens): Y = X deq(W)^T + Hs B^T, Hs = bf16(s X A^T).
// Bound by streaming the NF4 weight once (katajob, "NF4: 4-bit NormalFloat":
// the weight is read in 4-bit and expanded per block only inside the product).
//
// Data movement.  One persistent CTA per SM owns a contiguous run of 16-row
// weight tiles.  A producer thread streams each tile's code bytes through a
// ring in shared memory with 2D TMA copies (16 rows x 128 bytes per box,
// 128-byte swizzle), one stage = 16 rows x 32 blocks of 64 weights.
//
// Expansion.  A code byte holds two weights; a 256-entry table maps it to the
// two levels as a bf16 pair.  The table is replicated once per lane (entry e
// of lane l at T + 256 e + 4 l, T aligned to 64 KB), so a warp's lookups never
// share a bank and one prmt builds the lookup address from the code byte and
// the lane's base.  The weights are the A operand of m16n8k16 (16 rows x 16
// k per step, tokens in n), and the four steps of one 64-weight block
// accumulate into a fresh fragment that is then added with the block's scale
// absmax(q) * dq_scale.  Each step stays inside one block: lane t holds the
// block's code bytes 8t .. 8t+7 and covers k = 16t + 4s + 0..3 at step s; the
// activation fragments are read in the same order.
//
// Work split.  16 consumer warps take two blocks of every stage each (a
// K-split), keep per-row partial sums in registers across the tile, and hand
// them to an epilogue warp through a double-buffered shared array.  The
// epilogue warp adds the 16 partials in a fixed order (deterministic), adds
// the LoRA term with one more MMA over r, and stores bf16 Y.
#include <algorithm>

#include "internal.h"

namespace qn {

namespace {

constexpr int G_CW = 16;                            // consumer warps
constexpr int G_THREADS = (G_CW + 2) * 32;          // + TMA producer warp + epilogue warp
constexpr int G_ROWS = 16;                          // weight rows per tile
constexpr int G_SBLK = 2 * G_CW;                    // 64-weight blocks per stage
constexpr int G_BOX = 128 * G_ROWS;                 // one TMA box: 16 rows x 128 code bytes
constexpr int G_STAGE = (G_SBLK / 4) * G_BOX;       // 16 KB of codes per stage
constexpr int G_TABLE = 65536;                      // 256 entries x 256 B (128 B used)
constexpr int G_SDEPTH = 4;                         // stages the block-scale loads run ahead

// Shared memory, from the 64 KB-aligned table T: the table (entry e of lane
// l at T + 256 e + 4 l) fills the lower half of each 256-byte row; the upper
// halves (T + 256 e + 128) are 32-float rows that hold the partial sums
// handed to the epilogue warp.  The code ring, the warps' scale buffers and
// the barriers follow the table.
template <int NTILE>
struct GemvSmem {
  static constexpr int NS = 5;                                        // ring stages
  static constexpr int RED_ROWS = G_CW * NTILE * 4;                   // 32-float rows per partial-sum buffer
  static constexpr int OFF_RING = G_TABLE;
  static constexpr int OFF_SCALE = OFF_RING + NS * G_STAGE;           // [warp][2][32] fp32 block scales
  static constexpr int OFF_BAR = OFF_SCALE + G_CW * 2 * 32 * 4;
  static constexpr int USED = OFF_BAR + 8 * (2 * NS + 4);
  static constexpr int BYTES = USED + 65536;                          // room to align the table
};
static_assert(2 * GemvSmem<2>::RED_ROWS <= 256, "partial sums fit the table rows");
static_assert(GemvSmem<1>::BYTES <= 232448 && GemvSmem<2>::BYTES <= 232448, "shared memory");

// The MMA and the table loads are plain register functions for the compiler
// (no volatile), so it can schedule the lookups of a block ahead of its MMAs.
// Loads from the TMA ring stay volatile: they must not move above the wait.
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {  // the level table: written once, before any use
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// bf16x2 pair of the levels of a code byte, from the lane's table copy:
// address = [lane base byte 0, code byte, table base bytes 2-3].
template <int BYTE>
__device__ __forceinline__ uint32_t lut_pair(uint32_t word, uint32_t lane_base) {
  return lds32(prmt(word, lane_base, 0x7604u | (BYTE << 4)));
}

// What one consumer lane preloads for one block: its activation fragment
// X[8nt + g][64b + 16t .. +15].
template <int NTILE>
struct BlockIn {
  uint32_t x[NTILE][8];
};

// NB (1 or 2) consecutive 64-weight blocks of a 16-row tile, as one
// straight-line sequence so that the lookups and the two MMA chains of the
// blocks interleave: the lane's code bytes of its two rows (8 box rows apart)
// from the staged boxes, all table lookups, four MMA steps per block into a
// fresh fragment, then the scaled add into acc.
template <int NTILE, int NB>
__device__ __forceinline__ void blocks_mma(float (&acc)[NTILE][4], const BlockIn<NTILE> (&in)[2],
                                           const uint32_t (&code_addr)[2], uint32_t lane_base,
                                           const float2 (&sc)[2]) {
  uint2 cg[NB], ch[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    cg[b] = lds64(code_addr[b]);
    ch[b] = lds64(code_addr[b] + 1024u);
  }
  uint32_t a[NB][4][4];  // A fragments of the four k16 steps of each block
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const uint32_t wg = s < 2 ? cg[b].x : cg[b].y, wh = s < 2 ? ch[b].x : ch[b].y;
      if ((s & 1) == 0) {
        a[b][s][0] = lut_pair<0>(wg, lane_base); a[b][s][2] = lut_pair<1>(wg, lane_base);
        a[b][s][1] = lut_pair<0>(wh, lane_base); a[b][s][3] = lut_pair<1>(wh, lane_base);
      } else {
        a[b][s][0] = lut_pair<2>(wg, lane_base); a[b][s][2] = lut_pair<3>(wg, lane_base);
        a[b][s][1] = lut_pair<2>(wh, lane_base); a[b][s][3] = lut_pair<3>(wh, lane_base);
      }
    }
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < 4; ++s)
        mma16816(p, a[b][s][0], a[b][s][1], a[b][s][2], a[b][s][3], in[b].x[nt][2 * s], in[b].x[nt][2 * s + 1]);
      acc[nt][0] = fmaf(sc[b].x, p[0], acc[nt][0]);
      acc[nt][1] = fmaf(sc[b].x, p[1], acc[nt][1]);
      acc[nt][2] = fmaf(sc[b].y, p[2], acc[nt][2]);
      acc[nt][3] = fmaf(sc[b].y, p[3], acc[nt][3]);
    }
}

// MULTI: token m uses adapter aidx[m] of a stack (Bl = B_all [na, N, r]; Hs
// already holds that adapter's scaled H); the epilogue then adds the LoRA
// term per output with FMAs instead of one MMA shared by all tokens.  A
// token whose index is outside [0, na) gets no LoRA term.
//
// Bounded waits.  Every wait gives up after `wait_ns` (or once another warp of
// the CTA has given up) and records kDevTimeout.  `withhold` >= 0 is a testing
// aid: the producer then skips the copy of that code stage (no arrival, no
// copy), so the consumers' wait for it runs out; the producer stops at its next
// wait, lets the copies it did issue land and returns, the consumers and the
// epilogue warp leave their loops, and the CTA exits (no cluster, no barrier
// across the roles after the split).  Normal launches pass -1.
template <int NTILE, bool MULTI>
__global__ void __launch_bounds__(G_THREADS, 1)
    k_gemv(const __grid_constant__ CUtensorMap tm_codes, const uint16_t* __restrict__ X, int M,
           const uint8_t* __restrict__ absmax_q, const float* __restrict__ dq_scale, int N, int K,
           const uint16_t* __restrict__ Hs, const uint16_t* __restrict__ Bl, int r, Nf4Levels lv,
           const int32_t* __restrict__ aidx, int na, uint16_t* __restrict__ Y, int* status,
           unsigned long long wait_ns, int withhold, int lgs, int dq) {
  using S = GemvSmem<NTILE>;
  constexpr int NS = S::NS;
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t table = (raw + 65535u) & ~65535u;
  if (table + S::USED > raw + S::BYTES) {  // cannot happen with S::BYTES; never index past it
    if (threadIdx.x == 0) atomicExch(status, kDevTimeout);
    return;
  }
  const uint32_t ring = table + S::OFF_RING;
  // partial-sum row `row` of buffer `buf`, lane l: upper half of table row buf * RED_ROWS + row
  auto red_addr = [&](int buf, int row, int l) -> uint32_t {
    return table + (buf * S::RED_ROWS + row) * 256 + 128 + l * 4;
  };
  const uint32_t full0 = table + S::OFF_BAR, empty0 = full0 + 8u * NS;
  // rfull: an mbarrier per partial-sum buffer; rempty: a count of the buffer's
  // uses the epilogue has read (a count cannot be taken for one two uses older)
  const uint32_t rfull0 = empty0 + 8u * NS, rempty0 = rfull0 + 16u;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int pg = ((g & 3) << 1) | (g >> 2);  // tile row of MMA row g

  // table: entry e -> {bf16(L[e & 15]), bf16(L[e >> 4])}, one copy per lane
  for (int idx = tid; idx < 256 * 32; idx += G_THREADS) {
    const int e = idx >> 5, l = idx & 31;
    const uint32_t v = bf16x2_bits(lv.v[e & 15], lv.v[e >> 4]);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(table + e * 256 + l * 4), "r"(v) : "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, G_CW);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(rfull0 + 8u * b, G_CW);
      asm volatile("st.shared.s32 [%0], 0;" ::"r"(rempty0 + 4u * b) : "memory");  // uses of buffer b read
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int KB = K / 64;
  const int spt = (KB + G_SBLK - 1) / G_SBLK;  // stages per tile
  const int ntiles = (N + G_ROWS - 1) / G_ROWS;
  const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * ntiles / gridDim.x);
  const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nit = (t1 - t0) * spt;

  if (warp == G_CW) {  // producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_codes);
      int issued = 0, s = 0, tile = t0;
      for (int it = 0; it < nit; ++it) {
        const int slot = it % NS;
        if (!wait_bounded(empty0 + 8u * slot, ((it / NS) & 1) ^ 1, &abort_flag, status, wait_ns)) break;
        const int b0 = s * G_SBLK;
        const int nbox = min(G_SBLK / 4, (KB - b0 + 3) / 4);  // boxes that start inside the row
        if (it != withhold) {
          mbar_arrive_expect_tx(full0 + 8u * slot, nbox * G_BOX);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(ring + slot * G_STAGE + bx * G_BOX, &tm_codes, full0 + 8u * slot, (b0 + 4 * bx) * 32,
                        tile * G_ROWS);
        }
        ++issued;
        if (++s == spt) { s = 0; ++tile; }
      }
      // all copies land before exit (the withheld stage has none)
      for (int it = (issued > NS ? issued - NS : 0); it < issued; ++it)
        if (it != withhold) wait_drain(full0 + 8u * (it % NS), (it / NS) & 1);
    }
    return;
  }

  if (warp == G_CW + 1) {  // epilogue: sum the K-split partials, add the LoRA term, store
    // Hs comes from the previous kernel of the stream, which may still be
    // running (programmatic dependent launch): wait for it to complete
    pdl_wait();
    for (int ti = 0; ti < t1 - t0; ++ti) {
      const int n0 = (t0 + ti) * G_ROWS;
      const int buf = ti & 1;
      // LoRA operands first; their latency hides behind the wait
      auto ld2 = [&](const uint16_t* p, int row, int rows, int j) -> uint32_t {
        if (row >= rows || j >= r) return 0u;
        return __ldg(reinterpret_cast<const uint32_t*>(p + static_cast<int64_t>(row) * r + j));
      };
      uint32_t la[4][4], lb[4][NTILE][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (MULTI) break;
        const int j0 = 16 * k;
        la[k][0] = ld2(Bl, n0 + pg, N, j0 + 2 * t);
        la[k][1] = ld2(Bl, n0 + pg + 8, N, j0 + 2 * t);
        la[k][2] = ld2(Bl, n0 + pg, N, j0 + 2 * t + 8);
        la[k][3] = ld2(Bl, n0 + pg + 8, N, j0 + 2 * t + 8);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
          lb[k][nt][0] = ld2(Hs, 8 * nt + g, M, j0 + 2 * t);
          lb[k][nt][1] = ld2(Hs, 8 * nt + g, M, j0 + 2 * t + 8);
        }
      }
      if (!wait_bounded(rfull0 + 8u * buf, (ti >> 1) & 1, &abort_flag, status, wait_ns)) break;
      float v[NTILE][4];
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float sum = 0.f;
#pragma unroll 4
          for (int w = 0; w < G_CW; ++w) sum += lds_f32(red_addr(buf, (w * NTILE + nt) * 4 + c, lane));
          v[nt][c] = sum;
        }
      __syncwarp();
      if (lane == 0) set_count(rempty0 + 4u * buf, (ti >> 1) + 1);  // partial sums read: the buffer is free
      if (MULTI) {  // per-token adapters: sum_j Hs[m, j] B_a[n, j] with 8-wide loads
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = 8 * nt + 2 * t + (c & 1), n = n0 + pg + 8 * (c >> 1);
            if (m >= M || n >= N) continue;
            const int a = __ldg(aidx + m);
            if (a < 0 || a >= na) continue;
            const uint4* hp = reinterpret_cast<const uint4*>(Hs + static_cast<int64_t>(m) * r);
            const uint4* bp = reinterpret_cast<const uint4*>(Bl + (static_cast<int64_t>(a) * N + n) * r);
            float lora = 0.f;
            for (int j8 = 0; j8 < r / 8; ++j8) {
              const uint4 h = __ldg(hp + j8), b = __ldg(bp + j8);
              const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                lora = fmaf(__uint_as_float(hw[q] << 16), __uint_as_float(bw[q] << 16), lora);
                lora = fmaf(__uint_as_float(hw[q] & 0xffff0000u), __uint_as_float(bw[q] & 0xffff0000u), lora);
              }
            }
            v[nt][c] += lora;
          }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (16 * k >= r) break;
#pragma unroll
          for (int nt = 0; nt < NTILE; ++nt)
            mma16816(v[nt], la[k][0], la[k][1], la[k][2], la[k][3], lb[k][nt][0], lb[k][nt][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt) {
        const int m = 8 * nt + 2 * t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + pg + 8 * h;
          if (n >= N) continue;
          if (m < M) Y[static_cast<int64_t>(m) * N + n] = static_cast<uint16_t>(bf16x2_bits(v[nt][2 * h], 0.f));
          if (m + 1 < M)
            Y[static_cast<int64_t>(m + 1) * N + n] = static_cast<uint16_t>(bf16x2_bits(v[nt][2 * h + 1], 0.f));
        }
      }
    }
    return;
  }

  // consumers: warp w takes blocks 2w and 2w + 1 of every stage.  MMA row g
  // is tile row pg (and g + 8 is pg + 8): with this order the 16 lanes of a
  // half-warp read 8 different 16-byte chunks of the swizzled box, so the
  // 64-bit code loads are conflict-free.
  const uint32_t lane_base = table + lane * 4;
  uint32_t coff[2];  // byte offset of this lane's 8 code bytes (row pg) inside a stage
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int bb = 2 * warp + q;
    const int chunk = 2 * (bb & 3) + (t >> 1);
    coff[q] = (bb >> 2) * G_BOX + pg * 128 + ((chunk ^ pg) << 4) + ((t & 1) << 3);
  }
  // Token rows >= M read row M - 1 and weight rows >= N read row N - 1: those
  // columns and rows of the product are computed but never stored.
  const uint16_t* xrow[NTILE];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt)
    xrow[nt] = X + static_cast<int64_t>(min(8 * nt + g, M - 1)) * K + 16 * t + 128 * warp;
  float acc[NTILE][4];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  // Activation fragments are loaded one stage ahead of the MMAs into
  // registers (ls: the stage they fetch; they do not depend on the tile).  The block
  // scales come from HBM, so they run G_SDEPTH stages ahead in a register
  // shift ring: one per lane (tile row lane & 15, block 2w + (lane >> 4));
  // at its stage the lane stores absmax * dq_scale to the warp's scale
  // buffer, where rows pg and pg + 8 of a block sit side by side.
  const uint32_t wscale = table + S::OFF_SCALE + warp * (2 * 32 * 4);
  const int srow = lane & 15, sq = lane >> 4;
  const uint32_t sput = ((sq * 16 + (srow & 7) * 2 + (srow >> 3)) << 2);
  const uint32_t sget = pg * 8;  // + q * 64 for block q
  BlockIn<NTILE> in[2];
  int ls = 0;
  auto load_q = [&](int q) {
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      const uint4* p = reinterpret_cast<const uint4*>(xrow[nt] + ls * (64 * G_SBLK) + 64 * q);
      const uint4 lo = __ldg(p), hi = __ldg(p + 1);
      in[q].x[nt][0] = lo.x; in[q].x[nt][1] = lo.y; in[q].x[nt][2] = lo.z; in[q].x[nt][3] = lo.w;
      in[q].x[nt][4] = hi.x; in[q].x[nt][5] = hi.y; in[q].x[nt][6] = hi.z; in[q].x[nt][7] = hi.w;
    }
  };
  auto load_next = [&]() {  // both blocks of stage ls, or the one inside the row (warp-uniform)
    const int nv = KB - ls * G_SBLK - 2 * warp;
    if (nv >= 2) {
      load_q(0);
      load_q(1);
    } else if (nv == 1) {
      load_q(0);
    }
    if (++ls == spt) ls = 0;
  };
  uint32_t rq[G_SDEPTH];
  float rd[G_SDEPTH];
  int ss = 0, sn0 = t0 * G_ROWS;  // stage and tile row of the next scale load
  int sidx = min(sn0 + srow, N - 1) * KB + 2 * warp + sq;
  auto load_scale = [&](uint32_t& q, float& d) {
    q = 0u;
    d = 0.f;
    if (ss * G_SBLK + 2 * warp + sq < KB) {
      const int j = sidx + ss * G_SBLK;
      const int blk = j >> lgs;  // the format's block of this 64-weight block
      if (dq) {
        q = __ldg(absmax_q + blk);
        d = __ldg(dq_scale + (blk >> 8));
      } else {  // the exact fp32 absmax: q * d = 1 * d
        q = 1u;
        d = __ldg(dq_scale + blk);
      }
    }
    if (++ss == spt) {
      ss = 0;
      sn0 += G_ROWS;
      sidx = min(sn0 + srow, N - 1) * KB + 2 * warp + sq;
    }
  };
  load_next();
#pragma unroll
  for (int i = 0; i < G_SDEPTH; ++i) load_scale(rq[i], rd[i]);  // loads past the last stage read clamped rows

  int s = 0, ti = 0, slot = 0;
  uint32_t ph = 0;
  for (int it = 0; it < nit; ++it) {
    if (!wait_bounded(full0 + 8u * slot, ph, &abort_flag, status, wait_ns)) break;
    const bool more = it + 1 < nit;
    const int nvalid = KB - s * G_SBLK - 2 * warp;  // blocks of this warp inside the row
    const uint32_t sbuf = wscale + ((it & 1) << 7);
    sts_f32(sbuf + sput, __fmul_rn(static_cast<float>(rq[0]), rd[0]));
    __syncwarp();
#pragma unroll
    for (int i = 0; i + 1 < G_SDEPTH; ++i) {
      rq[i] = rq[i + 1];
      rd[i] = rd[i + 1];
    }
    load_scale(rq[G_SDEPTH - 1], rd[G_SDEPTH - 1]);
    {
      const uint32_t sb = ring + slot * G_STAGE;
      const uint32_t ca[2] = {sb + coff[0], sb + coff[1]};
      const float2 sc[2] = {lds_f2(sbuf + sget), lds_f2(sbuf + sget + 64)};
      if (nvalid >= 2)
        blocks_mma<NTILE, 2>(acc, in, ca, lane_base, sc);
      else if (nvalid == 1)
        blocks_mma<NTILE, 1>(acc, in, ca, lane_base, sc);
    }
    if (more) load_next();
    // the stage is refilled by TMA (async proxy): order this warp's reads of
    // it before the release
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8u * slot);
    if (++slot == NS) {
      slot = 0;
      ph ^= 1u;
    }
    if (++s == spt) {  // tile done: hand the partial sums to the epilogue warp
      const int buf = ti & 1;
      if (!wait_count_bounded(rempty0 + 4u * buf, ti >> 1, &abort_flag, status, wait_ns)) break;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          sts_f32(red_addr(buf, (warp * NTILE + nt) * 4 + c, lane), acc[nt][c]);
          acc[nt][c] = 0.f;
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(rfull0 + 8u * buf);
      s = 0;
      ++ti;
    }
  }
}

template <int NTILE, bool MULTI>
cudaError_t gemv_launch(const CUtensorMap& tm, const uint16_t* X, int64_t M, const uint8_t* absmax_q,
                        const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B, int r,
                        const int32_t* aidx, int na, uint16_t* Y, cudaStream_t st, unsigned long long wait_ns,
                        int withhold, int lgs, int dq) {
  using S = GemvSmem<NTILE>;
  cudaError_t e = smem_limit_once<k_gemv<NTILE, MULTI>>(S::BYTES);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  const int64_t ntiles = (N + G_ROWS - 1) / G_ROWS;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntiles, sms));
  // Programmatic dependent launch: the weight stream starts while the kernel
  // that computes Hs finishes; only the epilogue warp waits for it.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(G_THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemv<NTILE, MULTI>, tm, static_cast<const uint16_t*>(X), int(M), absmax_q,
                            dq_scale, int(N), int(K), Hs, B, r, host_codebook().levels, aidx, na, Y,
                            device_status_ptr(), wait_ns, withhold, lgs, dq);
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* X, int64_t M, const uint8_t* codes, const uint8_t* absmax_q,
                        const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B, int r,
                        uint16_t* Y, cudaStream_t st, const int32_t* aidx, int na, bool withhold_one_stage,
                        int block, int dq_block) {
  if (M == 0 || N == 0) return cudaSuccess;
  // the testing aid: a 1 ms wait limit and the second code stage of every CTA withheld
  const unsigned long long wait_ns = withhold_one_stage ? 1000000ull : kWaitLimitNs;
  const int withhold = withhold_one_stage ? 1 : -1;
  if (block != 64 && block != 128 && block != 256) return cudaErrorInvalidValue;  // a 64-weight block has one scale
  const int lgs = block == 64 ? 0 : block == 128 ? 1 : 2;
  const int dq = dq_block ? 1 : 0;
  if (M > 16 || r > 64 || N * (K / 64) >= (int64_t(1) << 31)) return cudaErrorInvalidValue;  // 32-bit block index
  CUtensorMap tm;
  if (!make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, K / 2, N, K / 2, 128, G_ROWS,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (aidx)
    return M <= 8 ? gemv_launch<1, true>(tm, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st, wait_ns,
                                         withhold, lgs, dq)
                  : gemv_launch<2, true>(tm, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st, wait_ns,
                                         withhold, lgs, dq);
  return M <= 8 ? gemv_launch<1, false>(tm, X, M, absmax_q, dq_scale, N, K, Hs, B, r, nullptr, 0, Y, st, wait_ns,
                                        withhold, lgs, dq)
                : gemv_launch<2, false>(tm, X, M, absmax_q, dq_scale, N, K, Hs, B, r, nullptr, 0, Y, st, wait_ns,
                                        withhold, lgs, dq);
}

namespace {

// ---------------------------------------------------------------------------
// Decode tiles: a serving layout of the codes, made once when the weight is
// loaded.  Unit (tile tau, block kb) is 512 contiguous bytes in which lane
// L = 4g + t of a warp owns bytes 16L .. 16L+15: the code bytes 8t .. 8t+7 of
// block kb in row 16 tau + g, then the same bytes of row 16 tau + g + 8 (rows
// past N hold zeros).  The units of a tile follow in kb order, so a tile is
// one contiguous run of 8 * K bytes, a warp reads a unit with one 128-bit load
// per lane, and the bytes land in exactly the registers the lookups of the
// row-major kernel above build from shared memory.
//
// Work split.  A CTA owns a run of tiles; a work item is 16 blocks (8 KB) of
// one tile, and consumer warp w takes items w, w + 15, w + 30, ... of the
// CTA's run, so the 15 warps read 120 KB of consecutive codes at a time.
// Each warp prefetches its next item into L2 with a bulk prefetch and keeps
// four units of loads in flight in registers.  A warp hands the item's
// per-row partial sums to the epilogue warp through a slot of shared memory;
// the epilogue adds a tile's items in item order (deterministic), adds the
// LoRA term and stores Y.
//
// Block scales.  With K % 1024 == 0 the 16 blocks of an item lie in one
// double-quantization group for every row, so a lane loads its two rows' 16
// absmax bytes and group scales once per item; the scale of unit u is then
// fl32(q * d) = fma(2^23 + q, d, -2^23 d) with 2^23 + q built by one prmt.

constexpr int T_CW = 15;                      // consumer warps (+ 1: four warps per SM sub-partition)
constexpr int T_THREADS = (T_CW + 1) * 32;    // + epilogue warp
constexpr int T_UNIT = 512;                   // bytes of one (tile, block) unit
constexpr int T_ITEM = 16;                    // blocks per work item
constexpr int T_GU = 4;                       // units per group of code loads (two groups in flight)
constexpr int T_SLOTS_MAX = 4;                // tiles whose partial sums can wait for the epilogue
constexpr int T_SMEM_LIMIT = 231424;          // dynamic shared memory cap (227 KB less 1 KB of static)
constexpr int T_HS_SMS = 8;                   // SMs of the kernel before this one (the Hs cluster)

__host__ __device__ constexpr int tiles_slot_bytes(int nch, int ntile) { return nch * ntile * 4 * 32 * 4; }
__host__ __device__ constexpr int tiles_smem_bytes(int nch, int ntile, int ts) {
  return 65536 /* table alignment */ + G_TABLE + ts * tiles_slot_bytes(nch, ntile) + 16 * ts + 64;
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(p));
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {  // activations and absmax bytes: keep them in L1
  return __ldg(reinterpret_cast<const uint4*>(p));
}
// The same load issued only by lanes with `on` set; the other lanes keep
// their registers (zeros, set once).  The predicate is explicit so the
// compiler cannot turn it into a load by every lane.
__device__ __forceinline__ void ldg_v4_if(const void* p, int on, uint32_t& a, uint32_t& b, uint32_t& c,
                                          uint32_t& d) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
      : "+r"(a), "+r"(b), "+r"(c), "+r"(d)
      : "l"(p), "r"(on));
}

// fl32(q * d) for the absmax byte at byte position `byte` of `word`: 2^23 + q
// is exact in fp32, so one fused multiply-add with c = -2^23 d rounds q * d once.
__device__ __forceinline__ float block_scale(uint32_t word, int byte, float d, float c) {
  return fmaf(__uint_as_float(prmt(word, 0x4B000000u, 0x7540u | byte)), d, c);
}

template <int NTILE>
struct UnitX {
  uint32_t x[NTILE][8];
};

// One unit: the A fragments of four MMA steps from the lane's four code
// words by 16 lookups (word i = cw.x, .y: row g bytes 0-3, 4-7; cw.z, .w:
// row g + 8; it fills steps 2(i & 1) and 2(i & 1) + 1), four MMA steps into a
// fresh fragment per token tile, then the scaled add (rows g: sa, rows g + 8:
// sb).
template <int NTILE>
__device__ __forceinline__ void unit_mma(float (&acc)[NTILE][4], const uint4& cw, const UnitX<NTILE>& in,
                                         uint32_t lane_base, float sa, float sb) {
  uint32_t a[4][4];
  const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int s0 = 2 * (i & 1), h = i >> 1;
    a[s0][h] = lut_pair<0>(w[i], lane_base);
    a[s0][h + 2] = lut_pair<1>(w[i], lane_base);
    a[s0 + 1][h] = lut_pair<2>(w[i], lane_base);
    a[s0 + 1][h + 2] = lut_pair<3>(w[i], lane_base);
  }
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) {
    float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < 4; ++s) mma16816(p, a[s][0], a[s][1], a[s][2], a[s][3], in.x[nt][2 * s], in.x[nt][2 * s + 1]);
    acc[nt][0] = fmaf(sa, p[0], acc[nt][0]);
    acc[nt][1] = fmaf(sa, p[1], acc[nt][1]);
    acc[nt][2] = fmaf(sb, p[2], acc[nt][2]);
    acc[nt][3] = fmaf(sb, p[3], acc[nt][3]);
  }
}

// GEN: a non-default format (blocks of 2^(6 + lgs) weights, double
// quantization on or off: dq); the scale of each unit is then loaded per unit
// instead of 16 absmax bytes per item.
template <int NTILE, bool MULTI, bool GEN>
__global__ void __launch_bounds__(T_THREADS, 1)
    k_gemv_tiles(const uint8_t* __restrict__ tiles, const uint16_t* __restrict__ X, int M,
                 const uint8_t* __restrict__ absmax_q, const float* __restrict__ dq_scale, int N, int K,
                 const uint16_t* __restrict__ Hs, const uint16_t* __restrict__ Bl, int r, Nf4Levels lv,
                 const int32_t* __restrict__ aidx, int na, int ts, int pf, uint16_t* __restrict__ Y, int* status,
                 int lgs, int dq) {
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag;
  const int KB = K / 64, NCH = KB / T_ITEM;
  const int bytes = tiles_smem_bytes(NCH, NTILE, ts);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t table = (raw + 65535u) & ~65535u;
  const uint32_t part0 = table + G_TABLE;
  const uint32_t slot_bytes = tiles_slot_bytes(NCH, NTILE);
  // full: an mbarrier per slot (NCH hand-overs per use); freed: how many uses
  // of the slot the epilogue has read (a count, so a warp may run any number
  // of tiles ahead of the epilogue without mistaking an old release for a new one)
  const uint32_t full0 = part0 + ts * slot_bytes, freed0 = full0 + 8u * ts;
  if (freed0 + 8u * ts > raw + bytes) {  // cannot happen with the launch's size; never index past it
    if (threadIdx.x == 0) atomicExch(status, kDevTimeout);
    return;
  }
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  for (int idx = tid; idx < 256 * 32; idx += T_THREADS) {
    const int e = idx >> 5, l = idx & 31;
    const uint32_t v = bf16x2_bits(lv.v[e & 15], lv.v[e >> 4]);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(table + e * 256 + l * 4), "r"(v) : "memory");
  }
  if (tid == 0) {
    for (int s = 0; s < ts; ++s) {
      mbar_init(full0 + 8u * s, NCH);
      asm volatile("st.shared.s32 [%0], 0;" ::"r"(freed0 + 4u * s) : "memory");
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int ntiles = (N + G_ROWS - 1) / G_ROWS;
  const int t0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * ntiles / gridDim.x);
  const int t1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * ntiles / gridDim.x);
  const int nitems = (t1 - t0) * NCH;
  // partial-sum word (chunk ch, tile nt, element c) of slot `slot`, lane l
  auto part_addr = [&](int slot, int ch, int nt, int c, int l) -> uint32_t {
    return part0 + slot * slot_bytes + ((((ch * NTILE + nt) * 4 + c) * 32 + l) << 2);
  };

  if (warp == T_CW) {  // epilogue: sum the items of each tile in order, add the LoRA term, store
    pdl_wait();  // Hs comes from the previous kernel of the stream
    for (int ti = 0; ti < t1 - t0; ++ti) {
      const int n0 = (t0 + ti) * G_ROWS;
      const int slot = ti % ts, use = ti / ts;
      auto ld2 = [&](const uint16_t* p, int row, int rows, int j) -> uint32_t {
        if (row >= rows || j >= r) return 0u;
        return __ldg(reinterpret_cast<const uint32_t*>(p + static_cast<int64_t>(row) * r + j));
      };
      uint32_t la[4][4], lb[4][NTILE][2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (MULTI) break;
        const int j0 = 16 * k;
        la[k][0] = ld2(Bl, n0 + g, N, j0 + 2 * t);
        la[k][1] = ld2(Bl, n0 + g + 8, N, j0 + 2 * t);
        la[k][2] = ld2(Bl, n0 + g, N, j0 + 2 * t + 8);
        la[k][3] = ld2(Bl, n0 + g + 8, N, j0 + 2 * t + 8);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
          lb[k][nt][0] = ld2(Hs, 8 * nt + g, M, j0 + 2 * t);
          lb[k][nt][1] = ld2(Hs, 8 * nt + g, M, j0 + 2 * t + 8);
        }
      }
      if (!wait_bounded(full0 + 8u * slot, use & 1, &abort_flag, status)) break;
      float v[NTILE][4];
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) v[nt][c] = 0.f;
      for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) v[nt][c] += lds_f32(part_addr(slot, ch, nt, c, lane));
      __syncwarp();
      if (lane == 0) set_count(freed0 + 4u * slot, use + 1);  // partial sums read: the slot is free
      if (MULTI) {
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int m = 8 * nt + 2 * t + (c & 1), n = n0 + g + 8 * (c >> 1);
            if (m >= M || n >= N) continue;
            const int a = __ldg(aidx + m);
            if (a < 0 || a >= na) continue;
            const uint4* hp = reinterpret_cast<const uint4*>(Hs + static_cast<int64_t>(m) * r);
            const uint4* bp = reinterpret_cast<const uint4*>(Bl + (static_cast<int64_t>(a) * N + n) * r);
            float lora = 0.f;
            for (int j8 = 0; j8 < r / 8; ++j8) {
              const uint4 h = __ldg(hp + j8), b = __ldg(bp + j8);
              const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                lora = fmaf(__uint_as_float(hw[q] << 16), __uint_as_float(bw[q] << 16), lora);
                lora = fmaf(__uint_as_float(hw[q] & 0xffff0000u), __uint_as_float(bw[q] & 0xffff0000u), lora);
              }
            }
            v[nt][c] += lora;
          }
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (16 * k >= r) break;
#pragma unroll
          for (int nt = 0; nt < NTILE; ++nt)
            mma16816(v[nt], la[k][0], la[k][1], la[k][2], la[k][3], lb[k][nt][0], lb[k][nt][1]);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt) {
        const int m = 8 * nt + 2 * t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + g + 8 * h;
          if (n >= N) continue;
          if (m < M) Y[static_cast<int64_t>(m) * N + n] = static_cast<uint16_t>(bf16x2_bits(v[nt][2 * h], 0.f));
          if (m + 1 < M)
            Y[static_cast<int64_t>(m + 1) * N + n] = static_cast<uint16_t>(bf16x2_bits(v[nt][2 * h + 1], 0.f));
        }
      }
    }
    return;
  }

  // consumers
  const uint32_t lane_base = table + lane * 4;
  const int64_t tile_bytes = static_cast<int64_t>(KB) * T_UNIT;
  auto item_codes = [&](int j) -> const uint8_t* {  // this lane's 16 bytes of the item's first unit
    const int ti = j / NCH, ch = j - ti * NCH;
    return tiles + static_cast<int64_t>(t0 + ti) * tile_bytes + static_cast<int64_t>(ch) * (T_ITEM * T_UNIT) + lane * 16;
  };
  // Lanes of token rows >= M load nothing and hold zeros (those columns are
  // never stored).
  const uint16_t* xrow[NTILE];
  int xon[NTILE];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) {
    xon[nt] = 8 * nt + g < M;
    xrow[nt] = X + static_cast<int64_t>(min(8 * nt + g, M - 1)) * K + 16 * t;
  }
  auto load_x = [&](UnitX<NTILE>& in, int kb) {
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      const uint16_t* p = xrow[nt] + kb * 64;
      ldg_v4_if(p, xon[nt], in.x[nt][0], in.x[nt][1], in.x[nt][2], in.x[nt][3]);
      ldg_v4_if(p + 8, xon[nt], in.x[nt][4], in.x[nt][5], in.x[nt][6], in.x[nt][7]);
    }
  };
  // the two rows' absmax bytes of item j start at this lane's index (dq group: index >> 8)
  auto absmax_index = [&](int j, int h) -> int64_t {
    const int ti = j / NCH, ch = j - ti * NCH;
    return static_cast<int64_t>(min((t0 + ti) * G_ROWS + g + 8 * h, N - 1)) * KB + ch * T_ITEM;
  };

  if (lane == 0)
    for (int q = 0; q < pf; ++q) {
      const int j = warp + q * T_CW;
      if (j < nitems) prefetch_l2(item_codes(j), T_ITEM * T_UNIT);
    }
  constexpr int NG = T_ITEM / T_GU;  // code groups per item (even: the next item's first group goes to cw[0])
  static_assert(NG % 2 == 0, "group count");
  uint4 cw[2][T_GU];  // codes of the current and the next group of units
  if (warp < nitems) {
    const uint8_t* c0 = item_codes(warp);
#pragma unroll
    for (int u = 0; u < T_GU; ++u) cw[0][u] = ldg_nc_v4(c0 + u * T_UNIT);
  }
  float acc[NTILE][4];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

  for (int j = warp; j < nitems; j += T_CW) {
    const int ti = j / NCH, ch = j - ti * NCH;
    const uint8_t* cbase = item_codes(j);
    if (lane == 0 && pf > 0) {
      const int jp = j + pf * T_CW;
      if (jp < nitems) prefetch_l2(item_codes(jp), T_ITEM * T_UNIT);
    }
    // the two rows' absmax bytes and group scales of the item; the next
    // item's lines go to L1 now, so its loads do not wait on L2
    const int kb0 = ch * T_ITEM;
    const int64_t ia = absmax_index(j, 0), ib = absmax_index(j, 1);
    const uint4 qa = GEN ? make_uint4(0u, 0u, 0u, 0u) : ldg_v4(absmax_q + ia);
    const uint4 qb = GEN ? make_uint4(0u, 0u, 0u, 0u) : ldg_v4(absmax_q + ib);
    const float da = GEN ? 0.f : __ldg(dq_scale + (ia >> 8)), db = GEN ? 0.f : __ldg(dq_scale + (ib >> 8));
    if (!GEN && j + T_CW < nitems) {
      const int64_t pa = absmax_index(j + T_CW, 0), pb = absmax_index(j + T_CW, 1);
      prefetch_l1(absmax_q + pa);
      prefetch_l1(absmax_q + pb);
      prefetch_l1(dq_scale + (pa >> 8));
      prefetch_l1(dq_scale + (pb >> 8));
    }
    const float ca = -8388608.0f * da, cb = -8388608.0f * db;
    const uint32_t qaw[4] = {qa.x, qa.y, qa.z, qa.w}, qbw[4] = {qb.x, qb.y, qb.z, qb.w};
    UnitX<NTILE> xin[2];
#pragma unroll
    for (int b = 0; b < 2; ++b)
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int i = 0; i < 8; ++i) xin[b].x[nt][i] = 0u;  // lanes of absent tokens keep zeros
    load_x(xin[0], kb0);
#pragma unroll
    for (int grp = 0; grp < NG; ++grp) {
      // loads of the next group: this item's, or the first of the next item
      if (grp + 1 < NG) {
#pragma unroll
        for (int u = 0; u < T_GU; ++u)
          cw[(grp + 1) & 1][u] = ldg_nc_v4(cbase + (T_GU * (grp + 1) + u) * T_UNIT);
      } else if (j + T_CW < nitems) {
        const uint8_t* cn = item_codes(j + T_CW);
#pragma unroll
        for (int u = 0; u < T_GU; ++u) cw[0][u] = ldg_nc_v4(cn + u * T_UNIT);
      }
#pragma unroll
      for (int u = 0; u < T_GU; ++u) {
        const int uu = T_GU * grp + u;
        if (uu + 1 < T_ITEM) load_x(xin[(uu + 1) & 1], kb0 + uu + 1);
        float sa, sb;
        if (!GEN) {
          sa = block_scale(qaw[uu >> 2], uu & 3, da, ca);
          sb = block_scale(qbw[uu >> 2], uu & 3, db, cb);
        } else {  // the format's blocks of this unit's 64-weight blocks (2^lgs of them per scale)
          const int64_t ga = (ia + uu) >> lgs, gb = (ib + uu) >> lgs;
          sa = dq ? __fmul_rn(static_cast<float>(__ldg(absmax_q + ga)), __ldg(dq_scale + (ga >> 8)))
                  : __ldg(dq_scale + ga);
          sb = dq ? __fmul_rn(static_cast<float>(__ldg(absmax_q + gb)), __ldg(dq_scale + (gb >> 8)))
                  : __ldg(dq_scale + gb);
        }
        unit_mma<NTILE>(acc, cw[grp & 1][u], xin[uu & 1], lane_base, sa, sb);
      }
    }
    // hand the item's partial sums to the epilogue warp
    const int slot = ti % ts, use = ti / ts;
    if (!wait_count_bounded(freed0 + 4u * slot, use, &abort_flag, status)) break;
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        sts_f32(part_addr(slot, ch, nt, c, lane), acc[nt][c]);
        acc[nt][c] = 0.f;
      }
    __syncwarp();
    if (lane == 0) mbar_arrive(full0 + 8u * slot);
  }
}

// one thread per 16-byte chunk of the tiles: chunk (tau * KB + kb) * 32 + L
__global__ void k_pack_tiles(const uint8_t* __restrict__ codes, int N, int K, uint8_t* __restrict__ tiles,
                             int64_t nchunks) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= nchunks) return;
  const int KB = K / 64;
  const int L = static_cast<int>(idx & 31);
  const int64_t rest = idx >> 5;
  const int kb = static_cast<int>(rest % KB);
  const int64_t tau = rest / KB;
  const int g = L >> 2, t = L & 3;
  const int64_t ra = tau * G_ROWS + g, rb = ra + 8;
  const int64_t off = static_cast<int64_t>(kb) * 32 + 8 * t;
  uint2 a = make_uint2(0u, 0u), b = make_uint2(0u, 0u);
  if (ra < N) a = __ldg(reinterpret_cast<const uint2*>(codes + ra * (K / 2) + off));
  if (rb < N) b = __ldg(reinterpret_cast<const uint2*>(codes + rb * (K / 2) + off));
  reinterpret_cast<uint4*>(tiles)[idx] = make_uint4(a.x, a.y, b.x, b.y);
}

template <int NTILE, bool MULTI, bool GEN>
cudaError_t gemv_tiles_launch_t(const uint8_t* tiles, const uint16_t* X, int64_t M, const uint8_t* absmax_q,
                                const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B,
                                int r, const int32_t* aidx, int na, uint16_t* Y, cudaStream_t st, int lgs, int dq) {
  const int nch = static_cast<int>(K / 64 / T_ITEM);
  const int avail = T_SMEM_LIMIT - tiles_smem_bytes(nch, NTILE, 0);
  const int ts = std::min(T_SLOTS_MAX, avail / (tiles_slot_bytes(nch, NTILE) + 16));
  if (ts < 1) return cudaErrorInvalidValue;  // K too large for one slot of partial sums
  cudaError_t e = smem_limit_once<k_gemv_tiles<NTILE, MULTI, GEN>>(T_SMEM_LIMIT);
  if (e != cudaSuccess) return e;
  // The kernel that computes Hs runs on T_HS_SMS SMs while this one starts
  // (programmatic dependent launch), and a CTA of this kernel cannot share an
  // SM with it (it holds the whole register file).  Use the fewest CTAs that
  // keep the largest per-CTA tile count of a launch that avoids those SMs: the
  // slowest CTA is as fast as with one CTA per SM, and no CTA waits for the
  // Hs kernel to leave its SM.
  const int64_t sms = std::max(1, device_sm_count() - T_HS_SMS);
  const int64_t ntiles = (N + G_ROWS - 1) / G_ROWS;
  const int64_t per_cta = (ntiles + sms - 1) / sms;
  const unsigned grid = static_cast<unsigned>((ntiles + per_cta - 1) / per_cta);
  return launch_ex(k_gemv_tiles<NTILE, MULTI, GEN>, dim3(grid), dim3(T_THREADS), tiles_smem_bytes(nch, NTILE, ts),
                   st, true, tiles, X, int(M), absmax_q, dq_scale, int(N), int(K), Hs, B, r, host_codebook().levels,
                   aidx, na, ts, 1, Y, device_status_ptr(), lgs, dq);
}

template <int NTILE, bool MULTI>
cudaError_t gemv_tiles_launch(const uint8_t* tiles, const uint16_t* X, int64_t M, const uint8_t* absmax_q,
                              const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B,
                              int r, const int32_t* aidx, int na, uint16_t* Y, cudaStream_t st, int lgs, int dq) {
  if (lgs == 0 && dq)
    return gemv_tiles_launch_t<NTILE, MULTI, false>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st,
                                                    lgs, dq);
  return gemv_tiles_launch_t<NTILE, MULTI, true>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st, lgs,
                                                 dq);
}

}  // namespace

int64_t decode_tiles_bytes(int64_t N, int64_t K) { return (N + G_ROWS - 1) / G_ROWS * (K / 64) * T_UNIT; }

cudaError_t launch_pack_tiles(const uint8_t* codes, int64_t N, int64_t K, uint8_t* tiles, cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  if (K % 1024 || N >= (int64_t(1) << 31) || K >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  const int64_t nchunks = decode_tiles_bytes(N, K) / 16;
  const unsigned grid = static_cast<unsigned>((nchunks + 255) / 256);
  k_pack_tiles<<<grid, 256, 0, st>>>(codes, int(N), int(K), tiles, nchunks);
  return cudaGetLastError();
}

cudaError_t launch_gemv_tiles(const uint16_t* X, int64_t M, const uint8_t* tiles, const uint8_t* absmax_q,
                              const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B,
                              int r, uint16_t* Y, cudaStream_t st, const int32_t* aidx, int na, int block,
                              int dq_block) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (M > 16 || r > 64 || K % 1024 || N * (K / 64) >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  if (block != 64 && block != 128 && block != 256) return cudaErrorInvalidValue;  // a 64-weight block has one scale
  const int lgs = block == 64 ? 0 : block == 128 ? 1 : 2;
  const int dq = dq_block ? 1 : 0;
  if (aidx)
    return M <= 8
               ? gemv_tiles_launch<1, true>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st, lgs, dq)
               : gemv_tiles_launch<2, true>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, aidx, na, Y, st, lgs, dq);
  return M <= 8
             ? gemv_tiles_launch<1, false>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, nullptr, 0, Y, st, lgs, dq)
             : gemv_tiles_launch<2, false>(tiles, X, M, absmax_q, dq_scale, N, K, Hs, B, r, nullptr, 0, Y, st, lgs, dq);
}

}  // namespace qn
