// LoRA adapter kernels ("QLoRA: fine-tuning a large model on one GPU",
// "LoRA, stated once": h = W0 x + (alpha/r) B A x).  With H = X A^T:
//   forward     H = X A^T                   (rowdot, contraction over K)
//   backward    dH = s dY B                 (rowdot over N, B read in place)
//               dA = dH^T X, dB = s dY^T H  (coldot, contraction over tokens)
// These are skinny (r <= 64 outputs per token) and bound by reading X or dY
// once: a single thread streams tiles with TMA through a deep shared-memory
// ring and the consumer warps run ldmatrix + mma.sync on swizzled tiles
// (r is too narrow for a full tcgen05 tile).
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

// ------------------------------------------------------------------ rows
//
// out[m, j] = sum_k P[m, k] Q(j, k) for 16 * CW tokens per CTA over the whole
// contraction.  P is bf16 [M, Kc]; Q is either [R, Kc] (QT = false: A) or
// [Kc, R] (QT = true: lora_B, read in place for dH = dY B).  CW = NT / 2
// consumer warps (16 tokens each) run ldmatrix + m16n8k16, the last warp's
// lane 0 produces: per stage a (16 CW) x 64 tile of P (128-byte swizzle) and
// the 64-wide slice of Q (as many bytes as the P tile, so Q costs no more L2
// traffic than P), RW_ST stages in flight.
constexpr int RW_ST = 8;

template <int NT>
struct RowsSmem {
  static constexpr int CW = NT / 2;
  static constexpr int P_BYTES = 16 * CW * 64 * 2;
  static constexpr int Q_BYTES = NT * 8 * 64 * 2;
  static constexpr int OFF_Q = RW_ST * P_BYTES;
  static constexpr int OFF_BAR = OFF_Q + RW_ST * Q_BYTES;
  static constexpr int BYTES = OFF_BAR + 2 * RW_ST * 8 + 1024;
};

template <int NT, bool QT>
__global__ void __launch_bounds__(32 * (NT / 2 + 1)) k_rows(const __grid_constant__ CUtensorMap tmP,
                                                            const __grid_constant__ CUtensorMap tmQ, int M, int Kc,
                                                            int R, float sa, uint16_t* __restrict__ out16a, float sb,
                                                            uint16_t* __restrict__ out16b, float* __restrict__ out32,
                                                            int* status) {
  using S = RowsSmem<NT>;
  constexpr int CW = S::CW;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t full0 = base + S::OFF_BAR, empty0 = full0 + 8u * RW_ST;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 16 * CW;
  const int nk = (Kc + 63) / 64;
  if (threadIdx.x == 0) {
    for (int s = 0; s < RW_ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, CW);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {  // producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % RW_ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / RW_ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, S::P_BYTES + S::Q_BYTES);
        tma_load_2d(base + s * S::P_BYTES, &tmP, full0 + 8u * s, it * 64, m0);
        if (QT)
          tma_load_2d(base + S::OFF_Q + s * S::Q_BYTES, &tmQ, full0 + 8u * s, 0, it * 64);
        else
          tma_load_2d(base + S::OFF_Q + s * S::Q_BYTES, &tmQ, full0 + 8u * s, it * 64, 0);
        ++issued;
      }
      for (int it = (issued > RW_ST ? issued - RW_ST : 0); it < issued; ++it)  // all copies land before exit
        wait_drain(full0 + 8u * (it % RW_ST), (it / RW_ST) & 1);
    }
    return;
  }

  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const int q = lane >> 3, l7 = lane & 7;
  for (int it = 0; it < nk; ++it) {
    const int s = it % RW_ST;
    if (!wait_bounded(full0 + 8u * s, (it / RW_ST) & 1, &abort_flag, status)) break;
    const uint32_t pt = base + s * S::P_BYTES;
    const uint32_t qt = base + S::OFF_Q + s * S::Q_BYTES;
#pragma unroll
    for (int k16 = 0; k16 < 4; ++k16) {
      // A: (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15), (rows 8-15, k 8-15)
      uint32_t a0, a1, a2, a3;
      {
        const int row = 16 * warp + l7 + (q & 1) * 8, chunk = 2 * k16 + (q >> 1);
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
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8u * s);
  }

  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int m = m0 + 16 * warp + g + 8 * h;
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

// ------------------------------------------------------------------ cols
//
// partial[split][j][c] = sum over this split's tokens m of G[m, j] P[m, c]:
// D[c, j] = sum_m P^T[c, m] G[m, j].  CTA = 64 columns c (4 consumer warps of
// 16) x all R, over one token range (a multiple of 32 tokens); warp 4 lane 0
// streams 32-token slabs of P (32 x 64, 128-byte swizzle) and G (32 x NT*8)
// through CL_ST stages.  Both operands have the contraction as their row and
// are read with ldmatrix.trans.  Rows past M arrive as zeros from TMA.
constexpr int CL_ST = 8;

template <int NT>
struct ColsSmem {
  static constexpr int P_BYTES = 32 * 64 * 2;
  static constexpr int G_BYTES = 32 * NT * 8 * 2;
  static constexpr int OFF_G = CL_ST * P_BYTES;
  static constexpr int OFF_BAR = OFF_G + CL_ST * G_BYTES;
  static constexpr int BYTES = OFF_BAR + 2 * CL_ST * 8 + 1024;
};

template <int NT>
__global__ void __launch_bounds__(160) k_cols(const __grid_constant__ CUtensorMap tmP,
                                              const __grid_constant__ CUtensorMap tmG, int M, int C, int R,
                                              int rows_per_split, float* __restrict__ partial, int* status) {
  using S = ColsSmem<NT>;
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t full0 = base + S::OFF_BAR, empty0 = full0 + 8u * CL_ST;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * 64;
  const int split = blockIdx.y;
  const int mb0 = split * rows_per_split;
  const int mb1 = min(M, mb0 + rows_per_split);
  const int nslab = mb1 > mb0 ? (mb1 - mb0 + 31) / 32 : 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < CL_ST; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, 4);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < nslab; ++it) {
        const int s = it % CL_ST;
        if (!wait_bounded(empty0 + 8u * s, ((it / CL_ST) & 1) ^ 1, &abort_flag, status)) break;
        mbar_arrive_expect_tx(full0 + 8u * s, S::P_BYTES + S::G_BYTES);
        tma_load_2d(base + s * S::P_BYTES, &tmP, full0 + 8u * s, c0, mb0 + 32 * it);
        tma_load_2d(base + S::OFF_G + s * S::G_BYTES, &tmG, full0 + 8u * s, 0, mb0 + 32 * it);
        ++issued;
      }
      for (int it = (issued > CL_ST ? issued - CL_ST : 0); it < issued; ++it)
        wait_drain(full0 + 8u * (it % CL_ST), (it / CL_ST) & 1);
    }
    return;
  }

  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const int q = lane >> 3, l7 = lane & 7;
  for (int it = 0; it < nslab; ++it) {
    const int s = it % CL_ST;
    if (!wait_bounded(full0 + 8u * s, (it / CL_ST) & 1, &abort_flag, status)) break;
    const uint32_t pt = base + s * S::P_BYTES;
    const uint32_t gt = base + S::OFF_G + s * S::G_BYTES;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a0, a1, a2, a3;  // P^T: (c 0-7, m 0-7), (c 8-15, m 0-7), (c 0-7, m 8-15), (c 8-15, m 8-15)
      {
        const int m = 16 * ks + (q >> 1) * 8 + l7, chunk = 2 * warp + (q & 1);
        ldsm_x4_trans(pt + m * 128 + ((chunk ^ (m & 7)) << 4), a0, a1, a2, a3);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;  // G: (m 0-7, tile 2np), (m 8-15, tile 2np), (m 0-7, tile 2np+1), (m 8-15, ...)
        const int m = 16 * ks + (q & 1) * 8 + l7, j = (2 * np + (q >> 1)) * 8;
        ldsm_x4_trans(narrow_addr<NT>(gt, m, j), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * np], a0, a1, a2, a3, b0, b1);
        mma_bf16_16816(acc[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8u * s);
  }

  const int g = lane >> 2, t = lane & 3;
  float* dst = partial + static_cast<int64_t>(split) * R * C;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int j = nt * 8 + 2 * t;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + 16 * warp + g + 8 * h;
      if (c >= C) continue;
      if (j < R) dst[static_cast<int64_t>(j) * C + c] = acc[nt][2 * h];
      if (j + 1 < R) dst[static_cast<int64_t>(j + 1) * C + c] = acc[nt][2 * h + 1];
    }
  }
}

// out = bf16(scale * sum_split partial[split]), as [R, C] or transposed [C, R].
// Thread = one column c and 8 consecutive j (blockIdx.y picks the 8): every
// partial read is coalesced across the warp, and a transposed output row
// segment of 8 values is one 16-byte store.
__global__ void __launch_bounds__(64) k_coldot_reduce(const float* __restrict__ partial, int splits, int R, int C,
                                                      float scale, int transpose, uint16_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int j0 = blockIdx.y * 8;
  if (c >= C) return;
  const int64_t plane = static_cast<int64_t>(R) * C;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll 4
  for (int sp = 0; sp < splits; ++sp) {
    const float* src = partial + sp * plane + static_cast<int64_t>(j0) * C + c;
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += __ldcs(src + static_cast<int64_t>(j) * C);
  }
  if (transpose) {
    uint4 v;
    v.x = bf16x2_bits(scale * acc[0], scale * acc[1]);
    v.y = bf16x2_bits(scale * acc[2], scale * acc[3]);
    v.z = bf16x2_bits(scale * acc[4], scale * acc[5]);
    v.w = bf16x2_bits(scale * acc[6], scale * acc[7]);
    *reinterpret_cast<uint4*>(out + static_cast<int64_t>(c) * R + j0) = v;
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const __nv_bfloat16 h = __float2bfloat16_rn(scale * acc[j]);
      out[static_cast<int64_t>(j0 + j) * C + c] = *reinterpret_cast<const uint16_t*>(&h);
    }
  }
}

int nt_for(int R) { return R <= 16 ? 2 : R <= 32 ? 4 : 8; }

int coldot_splits(int64_t M, int64_t C) {
  const int64_t col_tiles = (C + 63) / 64;
  int64_t s = (3 * 148 + col_tiles - 1) / col_tiles;  // ~3 CTAs per SM
  s = std::max<int64_t>(1, std::min<int64_t>(s, (M + 255) / 256));
  return static_cast<int>(s);
}

template <int NT, bool QT>
cudaError_t rows_launch(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                        uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  using S = RowsSmem<NT>;
  CUtensorMap tmP, tmQ;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, Kc, M, Kc * 2, 64, 16 * S::CW, CU_TENSOR_MAP_SWIZZLE_128B);
  if (QT)
    ok = ok && make_map(&tmQ, BF16, Q, R, Kc, R * 2, NT * 8, 64, narrow_swizzle<NT>());
  else
    ok = ok && make_map(&tmQ, BF16, Q, Kc, R, Kc * 2, 64, NT * 8, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_rows<NT, QT>>(S::BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((M + 16 * S::CW - 1) / (16 * S::CW));
  return launch_ex(k_rows<NT, QT>, dim3(grid), dim3(32 * (S::CW + 1)), S::BYTES, st, pdl, tmP, tmQ, int(M), int(Kc),
                   R, sa, out16a, sb, out16b, out32, device_status_ptr());
}

template <bool QT>
cudaError_t rows_dispatch(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  switch (nt_for(R)) {
    case 2: return rows_launch<2, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
    case 4: return rows_launch<4, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
    default: return rows_launch<8, QT>(P, Q, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
  }
}

template <int NT>
cudaError_t cols_launch(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, int splits,
                        int rows_per_split, float* partial, cudaStream_t st, bool pdl) {
  using S = ColsSmem<NT>;
  CUtensorMap tmP, tmG;
  const auto BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = make_map(&tmP, BF16, P, C, M, C * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&tmG, BF16, G, R, M, R * 2, NT * 8, 32, narrow_swizzle<NT>());
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = smem_limit_once<k_cols<NT>>(S::BYTES);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((C + 63) / 64), static_cast<unsigned>(splits));
  return launch_ex(k_cols<NT>, grid, dim3(160), S::BYTES, st, pdl, tmP, tmG, int(M), int(C), R, rows_per_split,
                   partial, device_status_ptr());
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

cudaError_t launch_rowdot_qt(const uint16_t* P, const uint16_t* Qt, int64_t M, int64_t Kc, int R, float sa,
                             uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st, bool pdl) {
  if (M == 0) return cudaSuccess;
  return rows_dispatch<true>(P, Qt, M, Kc, R, sa, out16a, sb, out16b, out32, st, pdl);
}

size_t coldot_partial_floats(int64_t M, int64_t C, int R) {
  return static_cast<size_t>(coldot_splits(M, C)) * static_cast<size_t>(R) * static_cast<size_t>(C);
}

cudaError_t launch_coldot(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                          int transpose, float* partial, uint16_t* out, cudaStream_t st, bool pdl) {
  const int splits = coldot_splits(M, C);
  // token ranges are whole 32-token slabs, so a slab never straddles two splits
  const int rows_per_split = static_cast<int>(((M + splits - 1) / splits + 31) / 32 * 32);
  cudaError_t e = cudaSuccess;
  if (M > 0) {
    switch (nt_for(R)) {
      case 2: e = cols_launch<2>(G, P, M, C, R, splits, rows_per_split, partial, st, pdl); break;
      case 4: e = cols_launch<4>(G, P, M, C, R, splits, rows_per_split, partial, st, pdl); break;
      default: e = cols_launch<8>(G, P, M, C, R, splits, rows_per_split, partial, st, pdl); break;
    }
  } else {
    e = cudaMemsetAsync(partial, 0, sizeof(float) * R * C, st);
  }
  if (e != cudaSuccess) return e;
  const int sp = M > 0 ? splits : 1;
  const dim3 rgrid(static_cast<unsigned>((C + 63) / 64), static_cast<unsigned>(R / 8));
  // the reduce follows the partial kernel directly (or a memset when M == 0)
  return launch_ex(k_coldot_reduce, rgrid, dim3(64), 0, st, M > 0, static_cast<const float*>(partial), sp, R,
                   int(C), scale, transpose, out);
}

}  // namespace qn
