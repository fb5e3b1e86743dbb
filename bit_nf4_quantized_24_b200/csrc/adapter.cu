// LoRA adapter kernels ("QLoRA: fine-tuning a large model on one GPU",
// "LoRA, stated once": h = W0 x + (alpha/r) B A x).  With H = X A^T:
//   forward     H = X A^T                   (rowdot, contraction over K)
//   backward    dH = s dY B                 (rowdot over N, with B^T)
//               dA = dH^T X, dB = s dY^T H  (coldot, contraction over tokens)
// These are skinny (r <= 64 outputs per token) and bound by reading X / dY.
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

__device__ __forceinline__ uint4 ldg_v4_or_zero(const uint16_t* p, bool ok) {
  return ok ? __ldg(reinterpret_cast<const uint4*>(p)) : make_uint4(0u, 0u, 0u, 0u);
}

// out[m, j] = sum_k P[m,k] Q[j,k].  One CTA = 16 rows of P; its 8 warps split
// the contraction into interleaved 32-wide chunks and meet in shared memory.
// Inside a chunk, thread t (= lane & 3) owns the 8 consecutive k's 8t..8t+7;
// they fill the fragment slots {2t, 2t+1, 2t+8, 2t+9} of two m16n8k16 steps.
// The same k permutation is used for both operands, so the sum is unchanged.
// U chunks are loaded before any is used, to keep enough bytes in flight.
template <int NT, int U>  // NT = ceil(R / 8) n8 tiles
__global__ void __launch_bounds__(256) k_rowdot(const uint16_t* __restrict__ P, const uint16_t* __restrict__ Q,
                                                int M, int Kc, int R, float sa, uint16_t* __restrict__ out16a,
                                                float sb, uint16_t* __restrict__ out16b, float* __restrict__ out32) {
  __shared__ float red[8][16][NT * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int m0 = blockIdx.x * 16;
  float acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const int nchunks = (Kc + 31) / 32;
  const bool row_lo = m0 + g < M, row_hi = m0 + g + 8 < M;
  for (int c0 = warp; c0 < nchunks; c0 += 8 * U) {
    uint4 alo[U], ahi[U], b[U][NT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = (c0 + 8 * u) * 32 + 8 * t;
      const bool kin = (c0 + 8 * u < nchunks) && k < Kc;
      alo[u] = ldg_v4_or_zero(P + static_cast<int64_t>(m0 + g) * Kc + k, kin && row_lo);
      ahi[u] = ldg_v4_or_zero(P + static_cast<int64_t>(m0 + g + 8) * Kc + k, kin && row_hi);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int j = nt * 8 + g;
        b[u][nt] = ldg_v4_or_zero(Q + static_cast<int64_t>(j) * Kc + k, kin && j < R);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        mma_bf16_16816(acc[nt], alo[u].x, ahi[u].x, alo[u].y, ahi[u].y, b[u][nt].x, b[u][nt].y);
        mma_bf16_16816(acc[nt], alo[u].z, ahi[u].z, alo[u].w, ahi[u].w, b[u][nt].z, b[u][nt].w);
      }
    }
  }
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    red[warp][g][nt * 8 + 2 * t] = acc[nt][0];
    red[warp][g][nt * 8 + 2 * t + 1] = acc[nt][1];
    red[warp][g + 8][nt * 8 + 2 * t] = acc[nt][2];
    red[warp][g + 8][nt * 8 + 2 * t + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < 16 * R; idx += blockDim.x) {
    const int row = idx / R, j = idx % R;
    const int m = m0 + row;
    if (m >= M) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w][row][j];
    const __nv_bfloat16 ha = __float2bfloat16_rn(sa * v);
    out16a[static_cast<int64_t>(m) * R + j] = *reinterpret_cast<const uint16_t*>(&ha);
    if (out16b) {
      const __nv_bfloat16 hb = __float2bfloat16_rn(sb * v);
      out16b[static_cast<int64_t>(m) * R + j] = *reinterpret_cast<const uint16_t*>(&hb);
    }
    if (out32) out32[static_cast<int64_t>(m) * R + j] = sb * v;
  }
}

__device__ __forceinline__ void cp_async_16z(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// partial[split][j][c] = sum over this split's tokens m of G[m, j] P[m, c],
// on the tensor cores: D[c, j] = sum_m P^T[c, m] G[m, j] with m16n8k16 tiles.
// Both operands are row-major with the contraction (m) as the row index, so
// 32-token slabs are staged in shared memory (cp.async, double-buffered,
// rows padded by 16 B so the 8 rows of an ldmatrix phase hit distinct banks)
// and read with ldmatrix.trans.  CTA = 128 columns x all R; warp w owns
// columns 32w..32w+31.
constexpr int CD_COLS = 128, CD_SLAB = 32, CD_PPITCH = CD_COLS + 8, CD_GPITCH = 64 + 8;

template <int NT>  // NT = ceil(R / 8) rounded up to even (ldmatrix.x4 feeds two n8 tiles)
__global__ void __launch_bounds__(128) k_coldot_mma(const uint16_t* __restrict__ G, const uint16_t* __restrict__ P,
                                                    int M, int C, int R, int rows_per_split,
                                                    float* __restrict__ partial) {
  __shared__ __align__(16) uint16_t sP[2][CD_SLAB][CD_PPITCH];
  __shared__ __align__(16) uint16_t sG[2][CD_SLAB][CD_GPITCH];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int c0 = blockIdx.x * CD_COLS;
  const int split = blockIdx.y;
  const int mb0 = split * rows_per_split;
  const int mb1 = min(M, mb0 + rows_per_split);
  const int nslab = mb1 > mb0 ? (mb1 - mb0 + CD_SLAB - 1) / CD_SLAB : 0;
  const int gchunks = (R + 7) / 8;  // 16-byte chunks per G row

  auto stage = [&](int sl, int buf) {
    const int mb = mb0 + sl * CD_SLAB;
    for (int u = tid; u < CD_SLAB * (CD_COLS / 8); u += 128) {
      const int i = u / (CD_COLS / 8), cc = (u % (CD_COLS / 8)) * 8;
      const bool ok = (mb + i < mb1) && (c0 + cc < C);
      const uint16_t* src = ok ? P + static_cast<int64_t>(mb + i) * C + c0 + cc : P;
      cp_async_16z(smem_u32(&sP[buf][i][cc]), src, ok);
    }
    for (int u = tid; u < CD_SLAB * 8; u += 128) {
      const int i = u / 8, cc = (u % 8) * 8;
      const bool ok = (mb + i < mb1) && (u % 8) < gchunks;
      const uint16_t* src = ok ? G + static_cast<int64_t>(mb + i) * R + cc : G;
      cp_async_16z(smem_u32(&sG[buf][i][cc]), src, ok);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  float acc[2][NT][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[a][n][0] = acc[a][n][1] = acc[a][n][2] = acc[a][n][3] = 0.f;

  if (nslab > 0) stage(0, 0);
  for (int sl = 0; sl < nslab; ++sl) {
    const int buf = sl & 1;
    if (sl + 1 < nslab) stage(sl + 1, buf ^ 1);
    else asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncthreads();
    const int q = lane >> 3, rr = lane & 7;
#pragma unroll
    for (int ks = 0; ks < CD_SLAB / 16; ++ks) {
      uint32_t a[2][4];
#pragma unroll
      for (int ct = 0; ct < 2; ++ct) {
        // matrices: (m 0-7, c 0-7), (m 0-7, c 8-15), (m 8-15, c 0-7), (m 8-15, c 8-15)
        const int m = ks * 16 + (q >> 1) * 8 + rr;
        const int c = warp * 32 + ct * 16 + (q & 1) * 8;
        ldsm_x4_trans(smem_u32(&sP[buf][m][c]), a[ct][0], a[ct][1], a[ct][2], a[ct][3]);
      }
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        // matrices: (m 0-7, tile 2np), (m 8-15, tile 2np), (m 0-7, tile 2np+1), (m 8-15, tile 2np+1)
        const int m = ks * 16 + (q & 1) * 8 + rr;
        const int j = (2 * np + (q >> 1)) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(smem_u32(&sG[buf][m][j]), b0, b1, b2, b3);
#pragma unroll
        for (int ct = 0; ct < 2; ++ct) {
          mma_bf16_16816(acc[ct][2 * np], a[ct][0], a[ct][1], a[ct][2], a[ct][3], b0, b1);
          mma_bf16_16816(acc[ct][2 * np + 1], a[ct][0], a[ct][1], a[ct][2], a[ct][3], b2, b3);
        }
      }
    }
    __syncthreads();
  }
  float* dst = partial + static_cast<int64_t>(split) * R * C;
#pragma unroll
  for (int ct = 0; ct < 2; ++ct) {
    const int cbase = c0 + warp * 32 + ct * 16 + g;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = nt * 8 + 2 * t;
      if (cbase < C) {
        if (j < R) dst[static_cast<int64_t>(j) * C + cbase] = acc[ct][nt][0];
        if (j + 1 < R) dst[static_cast<int64_t>(j + 1) * C + cbase] = acc[ct][nt][1];
      }
      if (cbase + 8 < C) {
        if (j < R) dst[static_cast<int64_t>(j) * C + cbase + 8] = acc[ct][nt][2];
        if (j + 1 < R) dst[static_cast<int64_t>(j + 1) * C + cbase + 8] = acc[ct][nt][3];
      }
    }
  }
}

// out = bf16(scale * sum_split partial[split]), as [R, C] or transposed [C, R].
// Thread = one column c and 8 consecutive j (blockIdx.y picks the 8): every
// partial read is coalesced across the warp, and a transposed output row
// segment of 8 values is one 16-byte store.
__global__ void __launch_bounds__(64) k_coldot_reduce(const float* __restrict__ partial, int splits, int R, int C,
                                                      float scale, int transpose, uint16_t* __restrict__ out) {
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

__global__ void k_transpose_bf16(const uint16_t* __restrict__ src, int R, int C, uint16_t* __restrict__ dst) {
  __shared__ uint16_t tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int rr = r0 + i, cc = c0 + threadIdx.x;
    if (rr < R && cc < C) tile[i][threadIdx.x] = src[static_cast<int64_t>(rr) * C + cc];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int cc = c0 + i, rr = r0 + threadIdx.x;
    if (rr < R && cc < C) dst[static_cast<int64_t>(cc) * R + rr] = tile[threadIdx.x][i];
  }
}

int coldot_splits(int64_t M, int64_t C) {
  const int64_t col_tiles = (C + CD_COLS - 1) / CD_COLS;
  int64_t s = (2 * 148 + col_tiles - 1) / col_tiles;  // ~2 CTAs per SM, long token slabs
  s = std::max<int64_t>(1, std::min<int64_t>(s, (M + 255) / 256));
  return static_cast<int>(s);
}

}  // namespace

cudaError_t launch_rowdot(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((M + 15) / 16);
  const int nt = (R + 7) / 8;
#define QN_ROWDOT(NTV)                                                                            \
  case NTV:                                                                                       \
    k_rowdot<NTV, (NTV <= 2 ? 4 : 2)><<<grid, 256, 0, st>>>(P, Q, static_cast<int>(M),             \
                                                           static_cast<int>(Kc), R, sa, out16a,   \
                                                           sb, out16b, out32);                    \
    break;
  switch (nt) {
    QN_ROWDOT(1) QN_ROWDOT(2) QN_ROWDOT(3) QN_ROWDOT(4) QN_ROWDOT(5) QN_ROWDOT(6) QN_ROWDOT(7) QN_ROWDOT(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef QN_ROWDOT
  return cudaGetLastError();
}

size_t coldot_partial_floats(int64_t M, int64_t C, int R) {
  return static_cast<size_t>(coldot_splits(M, C)) * static_cast<size_t>(R) * static_cast<size_t>(C);
}

cudaError_t launch_coldot(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                          int transpose, float* partial, uint16_t* out, cudaStream_t st) {
  const int splits = coldot_splits(M, C);
  const int rows_per_split = static_cast<int>((M + splits - 1) / splits);
  const dim3 grid(static_cast<unsigned>((C + CD_COLS - 1) / CD_COLS), static_cast<unsigned>(splits));
  if (M > 0) {
    const int nt = (R + 7) / 8;
    if (nt <= 2)
      k_coldot_mma<2><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (nt <= 4)
      k_coldot_mma<4><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (nt <= 6)
      k_coldot_mma<6><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (nt <= 8)
      k_coldot_mma<8><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else
      return cudaErrorInvalidValue;
  } else {
    cudaError_t e = cudaMemsetAsync(partial, 0, sizeof(float) * R * C, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int sp = M > 0 ? splits : 1;
  const dim3 rgrid(static_cast<unsigned>((C + 63) / 64), static_cast<unsigned>(R / 8));
  k_coldot_reduce<<<rgrid, 64, 0, st>>>(partial, sp, R, int(C), scale, transpose, out);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* src, int64_t R, int64_t C, uint16_t* dst, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((R + 31) / 32));
  k_transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(src, int(R), int(C), dst);
  return cudaGetLastError();
}

}  // namespace qn
