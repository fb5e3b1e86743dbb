// LoRA adapter kernels ("QLoRA: fine-tuning a large model on one GPU",
// "LoRA, stated once": h = W0 x + (alpha/r) B A x).  With H = X A^T:
//   forward     H = X A^T                   (rowdot, contraction over K)
//   backward    dH = s dY B                 (rowdot over N, B read in place)
//               dA = dH^T X, dB = s dY^T H  (coldot, contraction over tokens)
// These are skinny (r <= 64 outputs per token) and meant to be bound by
// reading X or dY once: a single thread streams tiles with TMA through a
// shared-memory ring.  For r = 64 (64 FLOP per byte streamed) the products
// run on tcgen05 (k_rows_tc, k_cols_tc: 128 tokens or columns as the UMMA M,
// r as N, the accumulator in TMEM); for smaller r, and for the dropout's
// masked inputs, consumer warps run ldmatrix + mma.sync on the swizzled tiles
// (k_rows, k_cols).
#include <algorithm>

#include "internal.h"

namespace qn {

namespace {

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// A narrow tile [rows][NT * 8] bf16 loaded by TMA with the swizzle that
// matches its row pitch (NT = 2, 4, 8 -> 32, 64, 128 bytes).  Byte address of
// the 16-byte chunk holding columns j .. j+7 of row `row`.
template <int NT>
__device__ __forceinline__ uint32_t narrow_addr(uint32_t tile, int row, int j) {
  constexpr int PITCH = NT * 16;
  const int chunk = j >> 3;
  const int sw = ((row * PITCH) >> 7) & (PITCH / 16 - 1);
  return tile + row * PITCH + ((chunk ^ sw) << 4);
}
template <int NT>
constexpr CUtensorMapSwizzle narrow_swizzle() {
  return NT == 2 ? CU_TENSOR_MAP_SWIZZLE_32B : NT == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
}

// ------------------------------------------------------------- rows, M <= 16
//
// The same product for at most 16 tokens (decode).  There is a single token
// tile, so the contraction is split instead: RS_CTAS CTAs of one cluster x
// RS_WARPS warps each take whole 64-wide k groups.  The warps of a CTA meet
// in shared memory, the CTAs through distributed shared memory, where CTA 0
// adds the cluster's partials in a fixed order and writes the outputs.  Each
// CTA lets the next kernel of the stream launch at once (programmatic
// dependent launch); that kernel waits for this grid to finish before it
// reads the outputs.
constexpr int RS_CTAS = 8, RS_WARPS = 8;

__device__ __forceinline__ uint32_t ldg32(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint32_t*>(p));
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}

template <int NT>
__global__ void __cluster_dims__(RS_CTAS, 1, 1) __launch_bounds__(RS_WARPS * 32)
    k_rows_small(const uint16_t* __restrict__ P, const uint16_t* __restrict__ Q, int M, int Kc, int R, float sa,
                 uint16_t* __restrict__ out16a, float sb, uint16_t* __restrict__ out16b,
                 float* __restrict__ out32) {
  __shared__ float wpart[RS_WARPS][16 * 64];
  __shared__ float cpart[16 * 64];
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int rank = static_cast<int>(cluster_ctarank());
  const int worker = rank * RS_WARPS + warp;
  const int ngroups = Kc / 64;
  const int gl = static_cast<int>(static_cast<int64_t>(worker) * ngroups / (RS_CTAS * RS_WARPS));
  const int gh = static_cast<int>(static_cast<int64_t>(worker + 1) * ngroups / (RS_CTAS * RS_WARPS));
  // token rows >= M and output columns >= R read clamped rows; those results are never stored
  const uint16_t* p0 = P + static_cast<int64_t>(min(g, M - 1)) * Kc + 2 * t;
  const uint16_t* p1 = P + static_cast<int64_t>(min(g + 8, M - 1)) * Kc + 2 * t;
  const uint16_t* qr[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) qr[nt] = Q + static_cast<int64_t>(min(8 * nt + g, R - 1)) * Kc + 2 * t;
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  for (int grp = gl; grp < gh; ++grp) {
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int k = grp * 64 + 16 * s;
      const uint32_t a0 = ldg32(p0 + k), a1 = ldg32(p1 + k), a2 = ldg32(p0 + k + 8), a3 = ldg32(p1 + k + 8);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[nt], a0, a1, a2, a3, ldg32(qr[nt] + k), ldg32(qr[nt] + k + 8));
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) wpart[warp][(g + 8 * (c >> 1)) * 64 + 8 * nt + 2 * t + (c & 1)] = acc[nt][c];
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * 64; idx += RS_WARPS * 32) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < RS_WARPS; ++w) v += wpart[w][idx];
    cpart[idx] = v;
  }
  cluster_sync_all();  // every CTA's partial is in its shared memory
  if (rank == 0) {
    const uint32_t base = smem_u32(cpart);
    for (int idx = threadIdx.x; idx < M * R; idx += RS_WARPS * 32) {
      const int m = idx / R, j = idx - m * R;
      float v = 0.f;
#pragma unroll
      for (int c = 0; c < RS_CTAS; ++c) v += ld_dsmem_f32(mapa_shared(base + 4u * (m * 64 + j), c));
      out16a[idx] = static_cast<uint16_t>(bf16x2_bits(sa * v, 0.f));
      if (out16b) out16b[idx] = static_cast<uint16_t>(bf16x2_bits(sb * v, 0.f));
      if (out32) out32[idx] = sb * v;
    }
  }
  cluster_sync_all();  // peers keep their shared memory until CTA 0 has read it
}

// ------------------------------------------------------------ LoRA dropout
//
// The adapter branch reads dropout(X) (the random draw is an input: mask,
// 1 = keep, and keep = 1 / (1 - p)):  Xd = mask ? bf16(fl32(x * keep)) : 0.
// Eight elements per thread (16-byte loads).
// Xd = mask ? bf16(fl32(x * keep)) : 0 for the eight bf16 values of x, mask
// bytes mk (nonzero = keep).  One definition for the materialised Xd and for
// the adapter kernels that apply the mask to their X tiles in shared memory.
__device__ __forceinline__ uint32_t dropout_pair(uint32_t xw, uint32_t mw, int sh, float keep) {
  const float lo = ((mw >> sh) & 0xffu) ? __fmul_rn(__uint_as_float(xw << 16), keep) : 0.f;
  const float hi = ((mw >> (sh + 8)) & 0xffu) ? __fmul_rn(__uint_as_float(xw & 0xffff0000u), keep) : 0.f;
  return bf16x2_bits(lo, hi);
}
__device__ __forceinline__ uint4 dropout8(uint4 x, uint2 mk, float keep) {
  return make_uint4(dropout_pair(x.x, mk.x, 0, keep), dropout_pair(x.y, mk.x, 16, keep),
                    dropout_pair(x.z, mk.y, 0, keep), dropout_pair(x.w, mk.y, 16, keep));
}
__device__ __forceinline__ uint2 ld_shared_v2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__global__ void __launch_bounds__(256) k_dropout_input(const uint16_t* __restrict__ X,
                                                       const uint8_t* __restrict__ mask, float keep, int64_t n8,
                                                       uint16_t* __restrict__ Xd) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 x = __ldg(reinterpret_cast<const uint4*>(X) + i);
  const uint2 mk = __ldg(reinterpret_cast<const uint2*>(mask) + i);
  reinterpret_cast<uint4*>(Xd)[i] = dropout8(x, mk, keep);
}

// dX += mask * keep * (dH A): the adapter's part of the input gradient under
// dropout, added to the base gradient dY deq(W) the GEMM left in dX.  Per
// element: t = fl32(sum_j dH[m, j] A[j, k]) (j in order), then
// dX = bf16(fl32(dX) + fl32(t * keep)) where the mask keeps k.  Eight
// consecutive k of one row per thread.
__global__ void __launch_bounds__(256) k_dx_add_masked(uint16_t* __restrict__ dX, const uint16_t* __restrict__ dH,
                                                       const uint16_t* __restrict__ A,
                                                       const uint8_t* __restrict__ mask, float keep, int64_t M,
                                                       int64_t K, int r) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;  // 8-element chunk
  if (i >= M * K / 8) return;
  const int64_t m = (8 * i) / K, k0 = 8 * i - m * K;
  float t[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const uint16_t* hr = dH + m * r;
  for (int j = 0; j < r; ++j) {
    const float h = __uint_as_float(static_cast<uint32_t>(hr[j]) << 16);
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(j) * K + k0));
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      t[2 * q] = fmaf(h, __uint_as_float(aw[q] << 16), t[2 * q]);
      t[2 * q + 1] = fmaf(h, __uint_as_float(aw[q] & 0xffff0000u), t[2 * q + 1]);
    }
  }
  uint4 d = reinterpret_cast<const uint4*>(dX)[i];
  const uint2 mk = __ldg(reinterpret_cast<const uint2*>(mask) + i);
  uint32_t dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t mw = q < 2 ? mk.x : mk.y;
    const int sh = 16 * (q & 1);
    float lo = __uint_as_float(dw[q] << 16), hi = __uint_as_float(dw[q] & 0xffff0000u);
    if ((mw >> sh) & 0xffu) lo = __fadd_rn(lo, __fmul_rn(t[2 * q], keep));
    if ((mw >> (sh + 8)) & 0xffu) hi = __fadd_rn(hi, __fmul_rn(t[2 * q + 1], keep));
    dw[q] = bf16x2_bits(lo, hi);
  }
  reinterpret_cast<uint4*>(dX)[i] = make_uint4(dw[0], dw[1], dw[2], dw[3]);
}

// ------------------------------------------------ rows, one adapter per token
//
// Hs[m, j] = bf16(scales[a] * sum_k X[m, k] A_all[a, j, k]), a = aidx[m], for
// the multi-adapter decode: every token may use a different A, so there is no
// shared operand for an MMA.  CTA (m, 8 consecutive j): its 256 threads split
// the contraction in 8-wide chunks (16-byte loads), then the CTA adds the
// threads' sums in a fixed order.  An index outside [0, na) gives zeros.
__global__ void __launch_bounds__(256) k_rows_multi(const uint16_t* __restrict__ X, int K,
                                                    const uint16_t* __restrict__ A_all, int na, int r,
                                                    const float* __restrict__ scales,
                                                    const int32_t* __restrict__ aidx, uint16_t* __restrict__ Hs) {
  __shared__ float red[8][8];
  pdl_trigger();
  pdl_wait();
  const int m = blockIdx.x, j0 = blockIdx.y * 8;
  const int a = aidx[m];
  const bool ok = a >= 0 && a < na;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (ok) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(m) * K);
    const uint16_t* ab = A_all + static_cast<int64_t>(a) * r * K;
    for (int c = threadIdx.x; c < K / 8; c += 256) {
      const uint4 x = __ldg(xr + c);
      const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj >= r) break;
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(ab + static_cast<int64_t>(j0 + jj) * K) + c);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[jj] = fmaf(__uint_as_float(xw[q] << 16), __uint_as_float(ww[q] << 16), acc[jj]);
          acc[jj] = fmaf(__uint_as_float(xw[q] & 0xffff0000u), __uint_as_float(ww[q] & 0xffff0000u), acc[jj]);
        }
      }
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int jj = 0; jj < 8; ++jj)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc[jj] += __shfl_xor_sync(0xffffffffu, acc[jj], off);
  if (lane == 0)
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) red[warp][jj] = acc[jj];
  __syncthreads();
  if (threadIdx.x < 8 && j0 + static_cast<int>(threadIdx.x) < r) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w][threadIdx.x];
    const float sc = ok ? scales[a] : 0.f;
    Hs[static_cast<int64_t>(m) * r + j0 + threadIdx.x] = static_cast<uint16_t>(bf16x2_bits(sc * v, 0.f));
  }
}

// ------------------------------------------------------------------ rows
//
// out[m, j] = sum_k P[m, k] Q(j, k) for 16 * CW tokens per CTA.  P is bf16
// [M, Kc]; Q is either [R, Kc] (QT = false: A) or [Kc, R] (QT = true: lora_B,
// read in place for dH = dY B).  Two groups of CW = NT / 2 consumer warps (16
// tokens each) take alternate stages and run ldmatrix + m16n8k16 (the second
// group doubles the warps that hide the MMA latency), the last warp's lane 0
// produces: per stage a
// (16 CW) x 64 tile of P (128-byte swizzle) and the 64-wide slice of Q (as
// many bytes as the P tile, so Q costs no more L2 traffic than P), four
// stages in flight.  When the token tiles alone do not fill the GPU, the
// contraction is split too: a cluster of `nsplit` CTAs (consecutive along
// grid x) shares a token tile, each CTA takes a contiguous range of the
// 64-wide stages, leaves its fp32 sums in shared memory, and after a cluster
// barrier each CTA adds one share of the outputs over the cluster's partials
// in rank order (distributed shared memory): deterministic, no scratch.
// MASK (LoRA dropout, H = Xd A^T without Xd in memory): each stage also
// brings the (16 CW) x 64 tile of the keep mask, and each consumer warp turns
// its 16 rows of the P tile into Xd in place before reading them.
template <int NT, bool MASK = false>
struct RowsSmem {
  // stages in flight; even, so that every slot of the ring belongs to one
  // consumer group (stage it goes to slot it % ST and group it % 2): a group
  // then uses its slots in order and can never wait on a slot two phases
  // ahead of the one it last released (an mbarrier parity cannot tell those
  // apart)
  static constexpr int ST = 4;
  static constexpr int CW = NT / 2;
  static constexpr int P_BYTES = 16 * CW * 64 * 2;
  static constexpr int Q_BYTES = NT * 8 * 64 * 2;
  static constexpr int M_BYTES = MASK ? 16 * CW * 64 : 0;
  static constexpr int OFF_Q = ST * P_BYTES;
  static constexpr int OFF_M = OFF_Q + ST * Q_BYTES;
  static constexpr int OFF_PART = OFF_M + ST * M_BYTES;  // fp32 [16 CW m][NT * 8 j]
  static constexpr int OFF_BAR = OFF_PART + 16 * CW * NT * 8 * 4;
  static constexpr int BYTES = OFF_BAR + 2 * ST * 8 + 1024;
};

// Sum over the cluster's ranks 0 .. n-1 (n <= 8) of the fp32 word at shared
// address `off` of each rank, in rank order; the remote loads are all issued
// before the first add.
__device__ __forceinline__ float cluster_sum_ranks(uint32_t off, int n) {
  float x[8];
#pragma unroll
  for (int rk = 0; rk < 8; ++rk) {
    x[rk] = 0.f;
    if (rk < n) asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x[rk]) : "r"(mapa_shared(off, rk)) : "memory");
  }
  float sum = x[0];
#pragma unroll
  for (int rk = 1; rk < 8; ++rk)
    if (rk < n) sum += x[rk];
  return sum;
}

// The same for four consecutive fp32 words (16-byte aligned) per rank.
__device__ __forceinline__ float4 cluster_sum_ranks4(uint32_t off, int n) {
  float4 x[8];
#pragma unroll
  for (int rk = 0; rk < 8; ++rk) {
    x[rk] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (rk < n)
      asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                   : "=f"(x[rk].x), "=f"(x[rk].y), "=f"(x[rk].z), "=f"(x[rk].w)
                   : "r"(mapa_shared(off, rk))
                   : "memory");
  }
  float4 sum = x[0];
#pragma unroll
  for (int rk = 1; rk < 8; ++rk)
    if (rk < n) {
      sum.x += x[rk].x;
      sum.y += x[rk].y;
      sum.z += x[rk].z;
      sum.w += x[rk].w;
    }
  return sum;
}

// The cluster's reduction of k_rows with a split contraction: every thread of
// every CTA arrives (the producer warp too); then CTA `split` writes outputs
// [V split / nsplit, V (split + 1) / nsplit) of the tile's V = 16 CW x R, each
// the sum of the ranks' partials in rank order.
template <int NT, int CW>
__device__ __forceinline__ void rows_reduce(uint32_t part, int M, int R, int m0, int split, int nsplit, float sa,
                                            uint16_t* out16a, float sb, uint16_t* out16b, float* out32) {
  constexpr int RJ = NT * 8;
  cluster_sync_all();  // every CTA's partial sums are in its shared memory
  const int V = 16 * CW * R;
  const int v0 = static_cast<int>(static_cast<int64_t>(V) * split / nsplit);
  const int v1 = static_cast<int>(static_cast<int64_t>(V) * (split + 1) / nsplit);
  for (int v = v0 + static_cast<int>(threadIdx.x); v < v1; v += blockDim.x) {
    const int ml = v / R, j = v - ml * R;
    const int m = m0 + ml;
    const float sum = cluster_sum_ranks(part + (ml * RJ + j) * 4, nsplit);
    if (m >= M) continue;
    const int64_t o = static_cast<int64_t>(m) * R + j;
    out16a[o] = static_cast<uint16_t>(bf16x2_bits(sa * sum, 0.f));
    if (out16b) out16b[o] = static_cast<uint16_t>(bf16x2_bits(sb * sum, 0.f));
    if (out32) out32[o] = sb * sum;
  }
  cluster_sync_all();  // peers keep their shared memory until every read is done
}

template <int NT, bool QT, bool MASK>
__global__ void __launch_bounds__(32 * (NT + 1)) k_rows(const __grid_constant__ CUtensorMap tmP,
                                                            const __grid_constant__ CUtensorMap tmQ,
                                                            const __grid_constant__ CUtensorMap tmM, float keep,
                                                            int M, int Kc, int R, float sa,
                                                            uint16_t* __restrict__ out16a, float sb,
                                                            uint16_t* __restrict__ out16b, float* __restrict__ out32,
                                                            int nsplit, int* status) {
  using S = RowsSmem<NT, MASK>;
  constexpr int RW_ST = S::ST;
  constexpr int CW = S::CW;
  constexpr int RJ = NT * 8;  // j extent of the partial buffer
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t full0 = base + S::OFF_BAR, empty0 = full0 + 8u * RW_ST;
  const uint32_t part = base + S::OFF_PART;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = nsplit > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int m0 = (blockIdx.x / nsplit) * 16 * CW;
  const int nk_all = (Kc + 63) / 64;
  const int it0 = static_cast<int>(static_cast<int64_t>(nk_all) * split / nsplit);
  const int nk = static_cast<int>(static_cast<int64_t>(nk_all) * (split + 1) / nsplit) - it0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RW_ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, CW);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 2 * CW) {  // producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % RW_ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / RW_ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, S::P_BYTES + S::Q_BYTES + S::M_BYTES);
        const int kx = (it0 + it) * 64;
        tma_load_2d(base + s * S::P_BYTES, &tmP, full0 + 8u * s, kx, m0);
        if (MASK) tma_load_2d(base + S::OFF_M + s * S::M_BYTES, &tmM, full0 + 8u * s, kx, m0);
        if (QT)
          tma_load_2d(base + S::OFF_Q + s * S::Q_BYTES, &tmQ, full0 + 8u * s, 0, kx);
        else
          tma_load_2d(base + S::OFF_Q + s * S::Q_BYTES, &tmQ, full0 + 8u * s, kx, 0);
        ++issued;
      }
      for (int it = (issued > RW_ST ? issued - RW_ST : 0); it < issued; ++it)  // all copies land before exit
        wait_drain(full0 + 8u * (it % RW_ST), (it / RW_ST) & 1);
    }
    __syncwarp();  // lane 0 rejoins the warp before the cluster barriers
    if (nsplit > 1) rows_reduce<NT, CW>(part, M, R, m0, split, nsplit, sa, out16a, sb, out16b, out32);
    return;
  }

  // Two groups of CW consumer warps take alternate stages (group grp the
  // stages it with it % 2 == grp); warp rw of a group owns rows 16 rw .. +15.
  const int rw = warp % CW, grp = warp / CW;
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const int q = lane >> 3, l7 = lane & 7;
  for (int it = grp; it < nk; it += 2) {
    const int s = it % RW_ST;
    if (!wait_bounded(full0 + 8u * s, (it / RW_ST) & 1, &abort_flag, status)) break;
    const uint32_t pt = base + s * S::P_BYTES;
    const uint32_t qt = base + S::OFF_Q + s * S::Q_BYTES;
    if (MASK) {  // this warp's 16 rows of the tile become Xd (16-byte chunks, 128-byte swizzle)
      const uint32_t mt = base + S::OFF_M + s * S::M_BYTES;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int ci = lane + 32 * u, row = 16 * rw + (ci >> 3), lc = ci & 7;
        const uint32_t xa = pt + row * 128 + ((lc ^ (row & 7)) << 4);
        const uint4 y = dropout8(ld_shared_v4(xa), ld_shared_v2(mt + row * 64 + lc * 8), keep);
        st_shared_v4(xa, y.x, y.y, y.z, y.w);
      }
      __syncwarp();
    }
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16) {
      // A: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
      uint32_t a0, a1, a2, a3;
      {
        const int row = 16 * rw + l7 + (q & 1) * 8, chunk = 2 * k16 + (q >> 1);
        ldsm_x4(pt + row * 128 + ((chunk ^ (row & 7)) << 4), a0, a1, a2, a3);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;  // (tile 2np: k 0-7, k 8-15), (tile 2np+1: k 0-7, k 8-15)
        if (QT) {  // Q tile [64 k][NT*8 j], rows = contraction
          const int kr = 16 * k16 + l7 + (q & 1) * 8, j = (2 * np + (q >> 1)) * 8;
          ldsm_x4_trans(narrow_addr<NT>(qt, kr, j), b0, b1, b2, b3);
        } else {   // Q tile [NT*8 j][64 k], 128-byte swizzle
          const int j = (2 * np + (q >> 1)) * 8 + l7, chunk = 2 * k16 + (q & 1);
          ldsm_x4(qt + j * 128 + ((chunk ^ (j & 7)) << 4), b0, b1, b2, b3);
        }
        mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // the stage is refilled by TMA (async proxy): order this warp's reads of
    // it before the release
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8u * s);
  }

  const int g = lane >> 2, t = lane & 3;
  // The groups' sums meet in part[m_local][j]: group 1 leaves its sums there,
  // group 0 adds them to its own (stage order does not matter for a sum of
  // disjoint stages, and the pairing is fixed, so the result is deterministic).
  auto part_addr = [&](int nt, int h) { return part + ((16 * rw + g + 8 * h) * RJ + nt * 8 + 2 * t) * 4; };
  if (grp == 1) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(part_addr(nt, h)), "f"(acc[nt][2 * h]),
                     "f"(acc[nt][2 * h + 1])
                     : "memory");
  }
  asm volatile("bar.sync 1, %0;" ::"r"(2 * CW * 32) : "memory");  // the consumer warps only
  if (grp == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float2 o;
        asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(o.x), "=f"(o.y) : "r"(part_addr(nt, h)) : "memory");
        acc[nt][2 * h] += o.x;
        acc[nt][2 * h + 1] += o.y;
      }
  }
  if (nsplit > 1) {  // this CTA's sums part[m_local][j], then the cluster's reduction
    if (grp == 0) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(part_addr(nt, h)), "f"(acc[nt][2 * h]),
                       "f"(acc[nt][2 * h + 1])
                       : "memory");
    }
    __syncwarp();
    rows_reduce<NT, CW>(part, M, R, m0, split, nsplit, sa, out16a, sb, out16b, out32);
    return;
  }
  if (grp == 1) return;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + 16 * rw + g + 8 * h;
      const int j = nt * 8 + 2 * t;
      if (m >= M || j >= R) continue;
      const float v0 = acc[nt][2 * h], v1 = acc[nt][2 * h + 1];
      const int64_t o = static_cast<int64_t>(m) * R + j;
      *reinterpret_cast<uint32_t*>(out16a + o) = bf16x2_bits(sa * v0, sa * v1);
      if (out16b) *reinterpret_cast<uint32_t*>(out16b + o) = bf16x2_bits(sb * v0, sb * v1);
      if (out32) *reinterpret_cast<float2*>(out32 + o) = make_float2(sb * v0, sb * v1);
    }
  }
}

// ---------------------------------------------------- rows on tcgen05, r = 64
//
// The same products for r = 64 on the 5th-generation tensor cores: with
// r = 64 each token row of X (or dY) meets 64 outputs, 64 FLOP per byte
// streamed, more than mma.sync sustains at HBM speed.  A CTA owns 128 tokens
// (the UMMA M) and a contiguous range of the 64-wide K stages; warp 0's lane 0
// streams the 128 x 64 tile of X and the 64 x 64 tile of A (K-major) or of B
// (QT: [Kc, 64] read in place, MN-major) through a 3-deep TMA ring (two CTAs
// per SM);
// warp 1 allocates 64 TMEM columns and its lane 0 issues
// tcgen05.mma.cta_group::1 (M = 128, N = 64, K = 16, four per stage) and
// commits each stage's release; warps 2-5 read the 128 x 64 fp32 accumulator
// back (one TMEM lane quarter each).  When the token tiles do not fill the
// GPU, the contraction is split over a cluster as in k_rows: the CTAs' fp32
// sums meet in distributed shared memory and are added in rank order.
constexpr int RT_BM = 128, RT_N = 64, RT_ST = 3;  // two CTAs fit an SM
constexpr int RT_P = RT_BM * 64 * 2;                    // X tile, 16 KB
constexpr int RT_Q = RT_N * 64 * 2;                     // A or B tile, 8 KB
constexpr int RT_OFF_Q = RT_ST * RT_P;
constexpr int RT_OFF_PART = RT_OFF_Q + RT_ST * RT_Q;    // fp32 [128][64], 16-byte chunks XOR-swizzled by row
constexpr int RT_OFF_BAR = RT_OFF_PART + RT_BM * RT_N * 4;
constexpr int RT_BYTES = RT_OFF_BAR + (2 * RT_ST + 3) * 8 + 1024;
constexpr int RT_THREADS = 192;

// part[ml][j]: chunk j / 4 of row ml stored at chunk (j / 4) ^ (ml & 15), so that
// a quarter-warp's 16-byte stores (8 rows, one chunk) and a warp's reads of 32
// consecutive j of one row both touch distinct banks.
__device__ __forceinline__ uint32_t rt_part(uint32_t part, int ml, int j) {
  return part + ml * 256 + ((((j >> 2) ^ (ml & 15))) << 4) + (j & 3) * 4;
}

__device__ __forceinline__ void rows_tc_reduce(uint32_t part, int M, int m0, int split, int nsplit, float sa,
                                               uint16_t* out16a, float sb, uint16_t* out16b, float* out32) {
  cluster_sync_all();  // every CTA's partial sums are in its shared memory
  // four consecutive outputs (one 16-byte chunk of a row) per thread and step
  const int V4 = RT_BM * RT_N / 4;
  const int v0 = V4 * split / nsplit, v1 = V4 * (split + 1) / nsplit;
  for (int v = v0 + static_cast<int>(threadIdx.x); v < v1; v += blockDim.x) {
    const int ml = v >> 4, j = (v & 15) * 4, m = m0 + ml;
    const float4 sum = cluster_sum_ranks4(rt_part(part, ml, j), nsplit);
    if (m >= M) continue;
    const int64_t o = static_cast<int64_t>(m) * RT_N + j;
    *reinterpret_cast<uint2*>(out16a + o) =
        make_uint2(bf16x2_bits(sa * sum.x, sa * sum.y), bf16x2_bits(sa * sum.z, sa * sum.w));
    if (out16b)
      *reinterpret_cast<uint2*>(out16b + o) =
          make_uint2(bf16x2_bits(sb * sum.x, sb * sum.y), bf16x2_bits(sb * sum.z, sb * sum.w));
    if (out32) *reinterpret_cast<float4*>(out32 + o) = make_float4(sb * sum.x, sb * sum.y, sb * sum.z, sb * sum.w);
  }
  cluster_sync_all();  // peers keep their shared memory until every read is done
}

template <bool QT>
__global__ void __launch_bounds__(RT_THREADS, 2) k_rows_tc(const __grid_constant__ CUtensorMap tmP,
                                                          const __grid_constant__ CUtensorMap tmQ, int M, int Kc,
                                                          float sa, uint16_t* __restrict__ out16a, float sb,
                                                          uint16_t* __restrict__ out16b, float* __restrict__ out32,
                                                          int nsplit, int* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t full0 = base + RT_OFF_BAR, empty0 = full0 + 8u * RT_ST;
  const uint32_t accum_bar = empty0 + 8u * RT_ST, drain_bar = accum_bar + 8u, tmem_slot = drain_bar + 8u;
  const uint32_t part = base + RT_OFF_PART;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = nsplit > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int m0 = (blockIdx.x / nsplit) * RT_BM;
  const int nk_all = (Kc + 63) / 64;
  const int it0 = static_cast<int>(static_cast<int64_t>(nk_all) * split / nsplit);
  const int nk = static_cast<int>(static_cast<int64_t>(nk_all) * (split + 1) / nsplit) - it0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RT_ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, RT_N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + (tmem_slot - raw));

  if (warp == 0) {  // TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % RT_ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / RT_ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, RT_P + RT_Q);
        const int kx = (it0 + it) * 64;
        tma_load_2d(base + s * RT_P, &tmP, full0 + 8u * s, kx, m0);
        if (QT)
          tma_load_2d(base + RT_OFF_Q + s * RT_Q, &tmQ, full0 + 8u * s, 0, kx);
        else
          tma_load_2d(base + RT_OFF_Q + s * RT_Q, &tmQ, full0 + 8u * s, kx, 0);
        ++issued;
      }
      for (int it = (issued > RT_ST ? issued - RT_ST : 0); it < issued; ++it)  // all copies land before exit
        wait_drain(full0 + 8u * (it % RT_ST), (it / RT_ST) & 1);
    }
  } else if (warp == 1) {  // MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(RT_BM, RT_N, false, QT);
      bool ok = true, committed = false;
      for (int it = 0; it < nk; ++it) {
        const int s = it % RT_ST;
        if (!(ok = wait_bounded(full0 + 8u * s, (it / RT_ST) & 1, &abort_flag, status))) break;
        tc_fence_after();
        const uint32_t p_s = base + s * RT_P, q_s = base + RT_OFF_Q + s * RT_Q;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = QT ? desc_sw128(q_s + kk * 2048, 8192, 1024) : desc_sw128(q_s + kk * 32, 16, 1024);
          tc_mma_f16(tmem, desc_sw128(p_s + kk * 32, 16, 1024), bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty0 + 8u * s);  // the slot is free once these MMAs have read it
        committed = true;
      }
      if (ok) {
        tc_commit(accum_bar);
      } else if (committed) {  // MMAs in flight finish before TMEM is freed
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
  } else {  // warps 2-5: the accumulator back from TMEM (lanes 32 (warp % 4) ..)
    if (wait_bounded(accum_bar, 0, &abort_flag, status)) {
      tc_fence_after();
      const int qd = warp & 3, ml = 32 * qd + lane;
      uint32_t v[2][32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * qd) << 16), v[0]);
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + 32u, v[1]);
      tmem_ld_wait();
      if (nsplit > 1) {
#pragma unroll
        for (int c = 0; c < 16; ++c)
          st_shared_v4(rt_part(part, ml, 4 * c), v[c >> 3][(c & 7) * 4], v[c >> 3][(c & 7) * 4 + 1],
                       v[c >> 3][(c & 7) * 4 + 2], v[c >> 3][(c & 7) * 4 + 3]);
      } else if (m0 + ml < M) {
        const int64_t o = static_cast<int64_t>(m0 + ml) * RT_N;
        auto f = [&](int j) { return __uint_as_float(v[j >> 5][j & 31]); };
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 a, b;
          a.x = bf16x2_bits(sa * f(8 * c), sa * f(8 * c + 1));
          a.y = bf16x2_bits(sa * f(8 * c + 2), sa * f(8 * c + 3));
          a.z = bf16x2_bits(sa * f(8 * c + 4), sa * f(8 * c + 5));
          a.w = bf16x2_bits(sa * f(8 * c + 6), sa * f(8 * c + 7));
          reinterpret_cast<uint4*>(out16a + o)[c] = a;
          if (out16b) {
            b.x = bf16x2_bits(sb * f(8 * c), sb * f(8 * c + 1));
            b.y = bf16x2_bits(sb * f(8 * c + 2), sb * f(8 * c + 3));
            b.z = bf16x2_bits(sb * f(8 * c + 4), sb * f(8 * c + 5));
            b.w = bf16x2_bits(sb * f(8 * c + 6), sb * f(8 * c + 7));
            reinterpret_cast<uint4*>(out16b + o)[c] = b;
          }
          if (out32) {
            reinterpret_cast<float4*>(out32 + o)[2 * c] =
                make_float4(sb * f(8 * c), sb * f(8 * c + 1), sb * f(8 * c + 2), sb * f(8 * c + 3));
            reinterpret_cast<float4*>(out32 + o)[2 * c + 1] =
                make_float4(sb * f(8 * c + 4), sb * f(8 * c + 5), sb * f(8 * c + 6), sb * f(8 * c + 7));
          }
        }
      }
    }
  }
  // every TMEM read is done before the columns are freed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, RT_N);
  }
  if (nsplit > 1) rows_tc_reduce(part, M, m0, split, nsplit, sa, out16a, sb, out16b, out32);
}

// ---------------------------------------------------- cols on tcgen05, r = 64
//
// dA = dH^T X (out [64, C]) and dB = s dY^T H (transpose: out [C, 64]) for
// r = 64 on the tensor cores: D[c][j] = sum_m P[m][c] G[m][j] with the
// columns c as the UMMA M (128 per CTA) and j as N = 64.  Per stage 64 tokens:
// P arrives as two 64 x 64 boxes (the A operand, MN-major: c contiguous) and
// G as one 64 x 64 box (the B operand, MN-major: j contiguous).  Roles as in
// k_rows_tc; the tokens are split over a cluster and the fp32 sums meet in
// distributed shared memory, laid out so that the reduction reads runs of
// consecutive words in the output's order: [c][j] (row-swizzled) for the
// transposed dB, [j][c] for dA.
constexpr int CT_BN = 128, CT_ST = 3;
constexpr int CT_P = 64 * CT_BN * 2;                    // 64 tokens x 128 columns, 16 KB
constexpr int CT_G = 64 * RT_N * 2;                     // 64 tokens x 64, 8 KB
constexpr int CT_OFF_G = CT_ST * CT_P;
constexpr int CT_OFF_PART = CT_OFF_G + CT_ST * CT_G;   // fp32, 128 x 64
constexpr int CT_OFF_BAR = CT_OFF_PART + CT_BN * RT_N * 4;
constexpr int CT_BYTES = CT_OFF_BAR + (2 * CT_ST + 3) * 8 + 1024;

__global__ void __launch_bounds__(RT_THREADS, 2) k_cols_tc(const __grid_constant__ CUtensorMap tmP,
                                                          const __grid_constant__ CUtensorMap tmG, int M, int C,
                                                          float scale, int transpose, uint16_t* __restrict__ out,
                                                          int nsplit, int* status) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t full0 = base + CT_OFF_BAR, empty0 = full0 + 8u * CT_ST;
  const uint32_t accum_bar = empty0 + 8u * CT_ST, drain_bar = accum_bar + 8u, tmem_slot = drain_bar + 8u;
  const uint32_t part = base + CT_OFF_PART;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = nsplit > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const int c0 = (blockIdx.x / nsplit) * CT_BN;
  const int ns_all = (M + 63) / 64;  // 64-token slabs
  const int it0 = static_cast<int>(static_cast<int64_t>(ns_all) * split / nsplit);
  const int nk = static_cast<int>(static_cast<int64_t>(ns_all) * (split + 1) / nsplit) - it0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < CT_ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, RT_N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem_raw + (tmem_slot - raw));

  if (warp == 0) {  // TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % CT_ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / CT_ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, CT_P + CT_G);
        const int m = (it0 + it) * 64;
        tma_load_2d(base + s * CT_P, &tmP, full0 + 8u * s, c0, m);
        tma_load_2d(base + s * CT_P + 8192, &tmP, full0 + 8u * s, c0 + 64, m);
        tma_load_2d(base + CT_OFF_G + s * CT_G, &tmG, full0 + 8u * s, 0, m);
        ++issued;
      }
      for (int it = (issued > CT_ST ? issued - CT_ST : 0); it < issued; ++it)  // all copies land before exit
        wait_drain(full0 + 8u * (it % CT_ST), (it / CT_ST) & 1);
    }
  } else if (warp == 1) {  // MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(CT_BN, RT_N, true, true);
      bool ok = true, committed = false;
      for (int it = 0; it < nk; ++it) {
        const int s = it % CT_ST;
        if (!(ok = wait_bounded(full0 + 8u * s, (it / CT_ST) & 1, &abort_flag, status))) break;
        tc_fence_after();
        const uint32_t p_s = base + s * CT_P, g_s = base + CT_OFF_G + s * CT_G;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 tokens per MMA
          tc_mma_f16(tmem, desc_sw128(p_s + kk * 2048, 8192, 1024), desc_sw128(g_s + kk * 2048, 8192, 1024), idesc,
                     (it > 0 || kk > 0) ? 1u : 0u);
        tc_commit(empty0 + 8u * s);
        committed = true;
      }
      if (ok) {
        tc_commit(accum_bar);
      } else if (committed) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0);
      }
    }
  } else {  // warps 2-5: TMEM lane (column) 32 (warp % 4) + lane
    if (wait_bounded(accum_bar, 0, &abort_flag, status)) {
      tc_fence_after();
      const int qd = warp & 3, cl = 32 * qd + lane, c = c0 + cl;
      uint32_t v[2][32];
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * qd) << 16), v[0]);
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + 32u, v[1]);
      tmem_ld_wait();
      auto f = [&](int j) { return __uint_as_float(v[j >> 5][j & 31]); };
      if (nsplit > 1) {
        if (transpose) {
#pragma unroll
          for (int q = 0; q < 16; ++q)
            st_shared_v4(rt_part(part, cl, 4 * q), v[q >> 3][(q & 7) * 4], v[q >> 3][(q & 7) * 4 + 1],
                         v[q >> 3][(q & 7) * 4 + 2], v[q >> 3][(q & 7) * 4 + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < RT_N; ++j)
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(part + (j * CT_BN + cl) * 4), "f"(f(j)) : "memory");
        }
      } else if (c < C) {
        if (transpose) {
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(c) * RT_N);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_uint4(bf16x2_bits(scale * f(8 * q), scale * f(8 * q + 1)),
                                bf16x2_bits(scale * f(8 * q + 2), scale * f(8 * q + 3)),
                                bf16x2_bits(scale * f(8 * q + 4), scale * f(8 * q + 5)),
                                bf16x2_bits(scale * f(8 * q + 6), scale * f(8 * q + 7)));
        } else {
#pragma unroll
          for (int j = 0; j < RT_N; ++j)
            out[static_cast<int64_t>(j) * C + c] = static_cast<uint16_t>(bf16x2_bits(scale * f(j), 0.f));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, RT_N);
  }
  if (nsplit > 1) {
    cluster_sync_all();  // every CTA's partial sums are in its shared memory
    // four consecutive outputs per thread and step: j .. j + 3 of one column (dB)
    // or columns cl .. cl + 3 of one j (dA)
    const int V4 = CT_BN * RT_N / 4;
    const int v0 = V4 * split / nsplit, v1 = V4 * (split + 1) / nsplit;
    for (int v = v0 + static_cast<int>(threadIdx.x); v < v1; v += blockDim.x) {
      if (transpose) {
        const int cl = v >> 4, j = (v & 15) * 4, c = c0 + cl;
        const float4 sum = cluster_sum_ranks4(rt_part(part, cl, j), nsplit);
        if (c >= C) continue;
        *reinterpret_cast<uint2*>(out + static_cast<int64_t>(c) * RT_N + j) =
            make_uint2(bf16x2_bits(scale * sum.x, scale * sum.y), bf16x2_bits(scale * sum.z, scale * sum.w));
      } else {
        const int j = v >> 5, cl = (v & 31) * 4, c = c0 + cl;
        const float4 sum = cluster_sum_ranks4(part + (j * CT_BN + cl) * 4, nsplit);
        const float w[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (c + q < C) out[static_cast<int64_t>(j) * C + c + q] = static_cast<uint16_t>(bf16x2_bits(scale * w[q], 0.f));
      }
    }
    cluster_sync_all();  // peers keep their shared memory until every read is done
  }
}

// ------------------------------------------------------------------ cols
//
// out = bf16(scale * D), D[c, j] = sum_m P[m, c] G[m, j] (contraction over
// tokens), written as [R, C] or transposed [C, R].  A cluster of up to
// CL_SPLIT_MAX CTAs (consecutive along grid x) owns 64 CB columns c x all R;
// its CTAs split the tokens into ranges of whole 32-token slabs.  In a CTA,
// the last warp's lane 0 streams 32-token slabs of P (CB boxes of 32 x 64,
// 128-byte swizzle) and G (32 x NT*8) through the stages, and the consumer
// warps (16 MT columns each) run ldmatrix.trans + mma.sync.  CB = 4 (256
// columns) reads G a quarter as often as CB = 1 and gives each TMA row four
// boxes; CB = 1 serves narrow outputs, where 256-column tiles would leave
// SMs idle.  The CTAs then leave their fp32 partial sums in shared memory (the
// ring, no longer in use) and, after a cluster barrier, each CTA adds one
// share of the outputs over the cluster's partials (distributed shared memory,
// fixed order) and stores it: no global scratch, no second kernel,
// deterministic.  Rows past M and columns past C arrive as zeros from TMA.
constexpr int CL_SPLIT_MAX = 8;  // portable cluster size

// MASK (LoRA dropout, dA = dH^T Xd without Xd in memory): each stage also
// brings the 32 x 64 CB tile of the keep mask, and each consumer warp turns
// its columns of the P tile into Xd in place before reading them.
template <int NT, int CB, bool MASK = false>
struct ColsCfg {
  static constexpr int MT = CB == 1 ? 1 : 2;          // 16-column MMA tiles per consumer warp
  static constexpr int CWC = CB * 4 / MT;             // consumer warps
  static constexpr int THREADS = 32 * (CWC + 1);
  static constexpr int ST = CB == 1 ? 8 : MASK ? 3 : 4;  // ring stages (two CTAs fit an SM)
  static constexpr int P_BYTES = CB * 32 * 64 * 2;    // CB boxes of 32 tokens x 64 columns
  static constexpr int G_BYTES = 32 * NT * 8 * 2;
  static constexpr int M_BYTES = MASK ? 32 * 64 * CB : 0;
  static constexpr int OFF_G = ST * P_BYTES;
  static constexpr int OFF_M = OFF_G + ST * G_BYTES;
  static constexpr int RING = OFF_M + ST * M_BYTES;
  static constexpr int PART = CB * 64 * NT * 8 * 4;   // fp32 [64 CB c][NT * 8 j], over the ring
  static constexpr int OFF_BAR = RING > PART ? RING : PART;
  static constexpr int BYTES = OFF_BAR + 2 * ST * 8 + 1024;
};

template <int NT, int CB, bool MASK>
__global__ void __launch_bounds__(ColsCfg<NT, CB, MASK>::THREADS) k_cols(const __grid_constant__ CUtensorMap tmP,
                                                                        const __grid_constant__ CUtensorMap tmG,
                                                                        const __grid_constant__ CUtensorMap tmM,
                                                                        float keep, int M, int C, int R,
                                                                        int rows_per_split, float scale, int transpose,
                                                                        uint16_t* __restrict__ out, int* status) {
  using S = ColsCfg<NT, CB, MASK>;
  constexpr int RJ = NT * 8;  // j extent of the partial buffer
  // The partial sums sit where the cluster's reduction reads them in runs of
  // consecutive words (a warp's remote loads then form few requests): for the
  // transposed output (consecutive threads take consecutive j) at
  // part[cl][j ^ pswz(cl)] (pairs j, j + 1 adjacent, the consumers' paired
  // stores spread over banks), for the untransposed one (consecutive cl) at
  // part[j][cl].
  auto pswz = [](int cl) { return (cl << 1) & (RJ - 1); };
  constexpr int MT = S::MT, CWC = S::CWC, ST = S::ST;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t full0 = base + S::OFF_BAR, empty0 = full0 + 8u * ST;
  const uint32_t part = base;  // the ring, once every stage is consumed
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t nsplit;
  asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(nsplit));
  const int split = static_cast<int>(cluster_ctarank());
  const int c0 = (blockIdx.x / nsplit) * 64 * CB;
  const int mb0 = split * rows_per_split;
  const int mb1 = min(M, mb0 + rows_per_split);
  const int nslab = mb1 > mb0 ? (mb1 - mb0 + 31) / 32 : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, CWC);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  float acc[MT][NT][4];
  if (warp == CWC) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nslab; ++it) {
        const int s = it % ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, S::P_BYTES + S::G_BYTES + S::M_BYTES);
#pragma unroll
        for (int b = 0; b < CB; ++b)
          tma_load_2d(base + s * S::P_BYTES + b * 4096, &tmP, full0 + 8u * s, c0 + 64 * b, mb0 + 32 * it);
        tma_load_2d(base + S::OFF_G + s * S::G_BYTES, &tmG, full0 + 8u * s, 0, mb0 + 32 * it);
        if (MASK) tma_load_2d(base + S::OFF_M + s * S::M_BYTES, &tmM, full0 + 8u * s, c0, mb0 + 32 * it);
        ++issued;
      }
      for (int it = (issued > ST ? issued - ST : 0); it < issued; ++it)
        wait_drain(full0 + 8u * (it % ST), (it / ST) & 1);
    }
    __syncwarp();
  } else {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < NT; ++i) acc[mt][i][0] = acc[mt][i][1] = acc[mt][i][2] = acc[mt][i][3] = 0.f;
    const int q = lane >> 3, l7 = lane & 7;
    const int cw0 = warp * 16 * MT;                  // first column of this warp in the CTA's tile
    const uint32_t box_off = (cw0 >> 6) * 4096;     // its box (a warp's columns stay in one box)
    const int cchunk0 = (cw0 & 63) >> 3;             // first 8-column chunk inside the box
    for (int it = 0; it < nslab; ++it) {
      const int s = it % ST;
      if (!wait_bounded(full0 + 8u * s, (it / ST) & 1, &abort_flag, status)) break;
      const uint32_t pt = base + s * S::P_BYTES + box_off;
      const uint32_t gt = base + S::OFF_G + s * S::G_BYTES;
      if (MASK) {  // this warp's 16 MT columns of the 32 tokens become Xd (128-byte swizzled box)
        constexpr int CPR = 2 * MT;  // 16-byte chunks of a token row in this warp's columns
        const uint32_t mt = base + S::OFF_M + s * S::M_BYTES;
#pragma unroll
        for (int u = 0; u < CPR; ++u) {
          const int ci = lane + 32 * u, row = ci / CPR, cc = ci % CPR, lc = cchunk0 + cc;
          const uint32_t xa = pt + row * 128 + ((lc ^ (row & 7)) << 4);
          const uint4 y = dropout8(ld_shared_v4(xa), ld_shared_v2(mt + row * (64 * CB) + cw0 + 8 * cc), keep);
          st_shared_v4(xa, y.x, y.y, y.z, y.w);
        }
        __syncwarp();
      }
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t a[MT][4];  // P^T per 16 columns: (c 0-7, m 0-7), (c 8-15, m 0-7), (c 0-7, m 8-15), (c 8-15, m 8-15)
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          const int m = 16 * ks + (q >> 1) * 8 + l7, chunk = cchunk0 + 2 * mt + (q & 1);
          ldsm_x4_trans(pt + m * 128 + ((chunk ^ (m & 7)) << 4), a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
        }
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          uint32_t b0, b1, b2, b3;  // G: (m 0-7, tile 2np), (m 8-15, tile 2np), (m 0-7, tile 2np+1), (m 8-15, ...)
          const int m = 16 * ks + (q & 1) * 8 + l7, j = (2 * np + (q >> 1)) * 8;
          ldsm_x4_trans(narrow_addr<NT>(gt, m, j), b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            mma_bf16_16816(acc[mt][2 * np], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b0, b1);
            mma_bf16_16816(acc[mt][2 * np + 1], a[mt][0], a[mt][1], a[mt][2], a[mt][3], b2, b3);
          }
        }
      }
      // the stage is refilled by TMA (async proxy): order this warp's reads
      // of it before the release
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * s);
    }
  }
  // Every stage is consumed and every copy has landed (the producer drains):
  // the ring now holds this CTA's partial sums part[c_local][j].
  __syncthreads();
  if (warp < CWC) {
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int cl = warp * 16 * MT + mt * 16 + g + 8 * h, j = nt * 8 + 2 * t;
          if (transpose) {
            asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(part + (cl * RJ + (j ^ pswz(cl))) * 4),
                         "f"(acc[mt][nt][2 * h]), "f"(acc[mt][nt][2 * h + 1])
                         : "memory");
          } else {
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(part + (j * (64 * CB) + cl) * 4), "f"(acc[mt][nt][2 * h])
                         : "memory");
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(part + ((j + 1) * (64 * CB) + cl) * 4),
                         "f"(acc[mt][nt][2 * h + 1])
                         : "memory");
          }
        }
  }
  cluster_sync_all();  // every CTA's partial sums are in its shared memory

  // This CTA's share of the 64 CB x R outputs, each the sum of the cluster's
  // partials in rank order.  Consecutive threads take consecutive output
  // addresses (c for [R, C], j for [C, R]).
  const int V = 64 * CB * R;
  const int v0 = static_cast<int>((static_cast<int64_t>(V) * split) / nsplit);
  const int v1 = static_cast<int>((static_cast<int64_t>(V) * (split + 1)) / nsplit);
  for (int v = v0 + static_cast<int>(threadIdx.x); v < v1; v += blockDim.x) {
    int cl, j;
    if (transpose) {
      cl = v / R;
      j = v - cl * R;
    } else {
      j = v / (64 * CB);
      cl = v - j * (64 * CB);
    }
    const int c = c0 + cl;
    if (c >= C) continue;
    const uint32_t off = transpose ? part + (cl * RJ + (j ^ pswz(cl))) * 4 : part + (j * (64 * CB) + cl) * 4;
    const float sum = cluster_sum_ranks(off, static_cast<int>(nsplit));
    const int64_t o = transpose ? static_cast<int64_t>(c) * R + j : static_cast<int64_t>(j) * C + c;
    out[o] = static_cast<uint16_t>(bf16x2_bits(scale * sum, 0.f));
  }
  cluster_sync_all();  // peers keep their shared memory until every read is done
}

int nt_for(int R) { return R <= 16 ? 2 : R <= 32 ? 4 : 8; }

// Token splits per column tile: one cluster of up to CL_SPLIT_MAX CTAs, at
// least 256 tokens each.
int cols_splits(int64_t M) {
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(CL_SPLIT_MAX, (M + 255) / 256)));
}

template <int NT, bool QT, bool MASK = false>
cudaError_t rows_launch(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                        uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl,
                        const uint8_t* mask = nullptr, float keep = 1.0f) {
  using S = RowsSmem<NT, MASK>;
  CUtensorMap tmP, tmQ, tmM;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, Kc, M, Kc * 2, 64, 16 * S::CW, CU_TENSOR_MAP_SWIZZLE_128B);
  if (QT)
    ok = ok && make_map(&tmQ, BF16, Q, R, Kc, R * 2, NT * 8, 64, narrow_swizzle<NT>());
  else
    ok = ok && make_map(&tmQ, BF16, Q, Kc, R, Kc * 2, 64, NT * 8, CU_TENSOR_MAP_SWIZZLE_128B);
  if (MASK)  // keep mask u8 [M, Kc], 64-byte rows of the (16 CW) x 64 tile
    ok = ok && make_map(&tmM, CU_TENSOR_MAP_DATA_TYPE_UINT8, mask, Kc, M, Kc, 64, 16 * S::CW,
                        CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    tmM = tmP;  // unused
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_rows<NT, QT, MASK>>(S::BYTES);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (M + 16 * S::CW - 1) / (16 * S::CW);
  // split the contraction when the token tiles give fewer than two CTAs per
  // SM (two fit by shared memory), keeping at least 4 stages per split
  const int64_t nk = (Kc + 63) / 64;
  const int64_t want = (2 * device_sm_count()) / std::max<int64_t>(1, tiles);
  const int nsplit = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({8, want, nk / 4})));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * nsplit), 1, 1);
  cfg.blockDim = dim3(32 * (2 * S::CW + 1), 1, 1);
  cfg.dynamicSmemBytes = S::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (nsplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(nsplit);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, k_rows<NT, QT, MASK>, tmP, tmQ, tmM, keep, int(M), int(Kc), R, sa, out16a, sb,
                            out16b, out32, nsplit, device_status_ptr());
}

template <bool QT>
cudaError_t rows_tc_launch(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, float sa, uint16_t* out16a,
                           float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  CUtensorMap tmP, tmQ;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, Kc, M, Kc * 2, 64, RT_BM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (QT)
    ok = ok && make_map(&tmQ, BF16, Q, RT_N, Kc, RT_N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok = ok && make_map(&tmQ, BF16, Q, Kc, RT_N, Kc * 2, 64, RT_N, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_rows_tc<QT>>(RT_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (M + RT_BM - 1) / RT_BM;
  // split the contraction over a cluster while the token tiles leave SMs idle
  // (two CTAs per SM), keeping at least 4 stages per split
  const int64_t nk = (Kc + 63) / 64;
  const int64_t want = 2 * device_sm_count() / std::max<int64_t>(1, tiles);
  const int nsplit = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({8, want, nk / 4})));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * nsplit), 1, 1);
  cfg.blockDim = dim3(RT_THREADS, 1, 1);
  cfg.dynamicSmemBytes = RT_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (nsplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(nsplit);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, k_rows_tc<QT>, tmP, tmQ, int(M), int(Kc), sa, out16a, sb, out16b, out32, nsplit,
                            device_status_ptr());
}

template <bool QT>
cudaError_t rows_dispatch(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  if (R == RT_N) return rows_tc_launch<QT>(P, Q, M, Kc, sa, out16a, sb, out16b, out32, st, pdl);
  switch (nt_for(R)) {
    case 2: return rows_launch<2, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
    case 4: return rows_launch<4, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
    default: return rows_launch<8, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
  }
}

template <int NT, int CB, bool MASK = false>
cudaError_t cols_launch_cb(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                           int transpose, uint16_t* out, cudaStream_t st, bool pdl, const uint8_t* mask = nullptr,
                           float keep = 1.0f) {
  using S = ColsCfg<NT, CB, MASK>;
  CUtensorMap tmP, tmG, tmM;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, C, M, C * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&tmG, BF16, G, R, M, R * 2, NT * 8, 32, narrow_swizzle<NT>());
  if (MASK)  // keep mask u8 [M, C], the 32 x 64 CB tile
    ok = ok && make_map(&tmM, CU_TENSOR_MAP_DATA_TYPE_UINT8, mask, C, M, C, 64 * CB, 32, CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    tmM = tmP;  // unused
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_cols<NT, CB, MASK>>(S::BYTES);
  if (e != cudaSuccess) return e;
  const int splits = cols_splits(M);
  // token ranges are whole 32-token slabs, so a slab never straddles two splits
  const int rows_per_split = static_cast<int>(((M + splits - 1) / splits + 31) / 32 * 32);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((C + 64 * CB - 1) / (64 * CB) * splits), 1, 1);
  cfg.blockDim = dim3(S::THREADS, 1, 1);
  cfg.dynamicSmemBytes = S::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(splits);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_cols<NT, CB, MASK>, tmP, tmG, tmM, keep, int(M), int(C), R, rows_per_split, scale,
                            transpose, out, device_status_ptr());
}

// 256-column tiles when they still give most SMs a CTA, else 64-column tiles.
template <int NT, bool MASK = false>
cudaError_t cols_launch(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                        int transpose, uint16_t* out, cudaStream_t st, bool pdl, const uint8_t* mask = nullptr,
                        float keep = 1.0f) {
  if ((C + 255) / 256 * cols_splits(M) >= device_sm_count() * 3 / 4)
    return cols_launch_cb<NT, 4, MASK>(G, P, M, C, R, scale, transpose, out, st, pdl, mask, keep);
  return cols_launch_cb<NT, 1, MASK>(G, P, M, C, R, scale, transpose, out, st, pdl, mask, keep);
}

}  // namespace

cudaError_t launch_rowdot(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  if (M == 0) return cudaSuccess;
  if (M <= 16) {
    const int iM = static_cast<int>(M), iK = static_cast<int>(Kc);
    const dim3 g(RS_CTAS), b(RS_WARPS * 32);
    switch (nt_for(R)) {
      case 2: return launch_ex(k_rows_small<2>, g, b, 0, st, pdl, P, Q, iM, iK, R, sa, out16a, sb, out16b, out32);
      case 4: return launch_ex(k_rows_small<4>, g, b, 0, st, pdl, P, Q, iM, iK, R, sa, out16a, sb, out16b, out32);
      default: return launch_ex(k_rows_small<8>, g, b, 0, st, pdl, P, Q, iM, iK, R, sa, out16a, sb, out16b, out32);
    }
  }
  return rows_dispatch<false>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
}

cudaError_t launch_dropout_input(const uint16_t* X, const uint8_t* mask, float keep, int64_t n, uint16_t* Xd,
                                 cudaStream_t st, bool pdl) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  return launch_ex(k_dropout_input, dim3(static_cast<unsigned>((n8 + 255) / 256)), dim3(256), 0, st, pdl, X, mask,
                   keep, n8, Xd);
}

cudaError_t launch_dx_add_masked(uint16_t* dX, const uint16_t* dH, const uint16_t* A, const uint8_t* mask, float keep,
                                 int64_t M, int64_t K, int r, cudaStream_t st, bool pdl) {
  const int64_t n8 = M * K / 8;
  if (n8 == 0) return cudaSuccess;
  return launch_ex(k_dx_add_masked, dim3(static_cast<unsigned>((n8 + 255) / 256)), dim3(256), 0, st, pdl, dX, dH, A,
                   mask, keep, M, K, r);
}

cudaError_t launch_rows_multi(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A_all, int na, int r,
                              const float* scales, const int32_t* aidx, uint16_t* Hs, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  return launch_ex(k_rows_multi, dim3(static_cast<unsigned>(M), static_cast<unsigned>((r + 7) / 8)), dim3(256), 0,
                   st, false, X, static_cast<int>(K), A_all, na, r, scales, aidx, Hs);
}

cudaError_t launch_rowdot_qt(const uint16_t* P, const uint16_t* Qt, int64_t M, int64_t Kc, int R, float sa,
                             uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  if (M == 0) return cudaSuccess;
  return rows_dispatch<true>(P, Qt, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
}

static cudaError_t cols_tc_launch(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, float scale, int transpose,
                           uint16_t* out, cudaStream_t st, bool pdl) {
  CUtensorMap tmP, tmG;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, C, M, C * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&tmG, BF16, G, RT_N, M, RT_N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_cols_tc>(CT_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (C + CT_BN - 1) / CT_BN, nslab = (M + 63) / 64;
  // split the tokens over a cluster while the column tiles leave SMs idle
  // (two CTAs per SM), keeping at least 4 slabs per split
  const int64_t want = 2 * device_sm_count() / std::max<int64_t>(1, tiles);
  const int nsplit = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>({8, want, nslab / 4})));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * nsplit), 1, 1);
  cfg.blockDim = dim3(RT_THREADS, 1, 1);
  cfg.dynamicSmemBytes = CT_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (nsplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = static_cast<unsigned>(nsplit);
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, k_cols_tc, tmP, tmG, int(M), int(C), scale, transpose, out, nsplit,
                            device_status_ptr());
}

cudaError_t launch_coldot(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                          int transpose, uint16_t* out, cudaStream_t st, bool pdl) {
  if (M == 0) return cudaMemsetAsync(out, 0, sizeof(uint16_t) * static_cast<size_t>(R) * C, st);
  if (R == RT_N) return cols_tc_launch(G, P, M, C, scale, transpose, out, st, pdl);
  switch (nt_for(R)) {
    case 2: return cols_launch<2>(G, P, M, C, R, scale, transpose, out, st, pdl);
    case 4: return cols_launch<4>(G, P, M, C, R, scale, transpose, out, st, pdl);
    default: return cols_launch<8>(G, P, M, C, R, scale, transpose, out, st, pdl);
  }
}

cudaError_t launch_rowdot_masked(const uint16_t* X, const uint8_t* mask, float keep, const uint16_t* Q, int64_t M,
                                 int64_t Kc, int R, float sa, uint16_t* out16a, float sb, uint16_t* out16b,
                                 cudaStream_t st, bool pdl) {
  if (M <= 16) return cudaErrorInvalidValue;  // the caller materialises Xd for the small kernel
  switch (nt_for(R)) {
    case 2: return rows_launch<2, false, true>(X, Q, M, Kc, R, sa, out16a, sb, out16b, nullptr, st, pdl, mask, keep);
    case 4: return rows_launch<4, false, true>(X, Q, M, Kc, R, sa, out16a, sb, out16b, nullptr, st, pdl, mask, keep);
    default: return rows_launch<8, false, true>(X, Q, M, Kc, R, sa, out16a, sb, out16b, nullptr, st, pdl, mask, keep);
  }
}

cudaError_t launch_coldot_masked(const uint16_t* G, const uint16_t* X, const uint8_t* mask, float keep, int64_t M,
                                 int64_t C, int R, float scale, uint16_t* out, cudaStream_t st, bool pdl) {
  if (M == 0) return cudaMemsetAsync(out, 0, sizeof(uint16_t) * static_cast<size_t>(R) * C, st);
  switch (nt_for(R)) {
    case 2: return cols_launch<2, true>(G, X, M, C, R, scale, 0, out, st, pdl, mask, keep);
    case 4: return cols_launch<4, true>(G, X, M, C, R, scale, 0, out, st, pdl, mask, keep);
    default: return cols_launch<8, true>(G, X, M, C, R, scale, 0, out, st, pdl, mask, keep);
  }
}

}  // namespace qn
