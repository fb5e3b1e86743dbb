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
template <int NT>  // NT = ceil(R / 8) n8 tiles
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
  for (int c = warp; c < nchunks; c += 8) {
    const int k = c * 32 + 8 * t;
    const bool kin = k < Kc;
    const uint4 alo = ldg_v4_or_zero(P + static_cast<int64_t>(m0 + g) * Kc + k, kin && row_lo);
    const uint4 ahi = ldg_v4_or_zero(P + static_cast<int64_t>(m0 + g + 8) * Kc + k, kin && row_hi);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = nt * 8 + g;
      const uint4 b = ldg_v4_or_zero(Q + static_cast<int64_t>(j) * Kc + k, kin && j < R);
      mma_bf16_16816(acc[nt], alo.x, ahi.x, alo.y, ahi.y, b.x, b.y);
      mma_bf16_16816(acc[nt], alo.z, ahi.z, alo.w, ahi.w, b.z, b.w);
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

// partial[split][j][c] = sum over this split's rows m of G[m, j] P[m, c].
// Thread = 2 adjacent columns c; the split's G rows are staged in shared
// memory (fp32) 64 rows at a time and read as broadcasts.
template <int RP>  // R rounded up to 8, 16, 32 or 64
__global__ void __launch_bounds__(128) k_coldot_partial(const uint16_t* __restrict__ G,
                                                        const uint16_t* __restrict__ P, int M, int C, int R,
                                                        int rows_per_split, float* __restrict__ partial) {
  __shared__ __align__(16) float sG[64][RP];
  const int c = (blockIdx.x * 128 + threadIdx.x) * 2;
  const int split = blockIdx.y;
  const int mb0 = split * rows_per_split;
  const int mb1 = min(M, mb0 + rows_per_split);
  float acc[RP][2];
#pragma unroll
  for (int j = 0; j < RP; ++j) acc[j][0] = acc[j][1] = 0.f;
  for (int mb = mb0; mb < mb1; mb += 64) {
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * RP; idx += 128) {
      const int i = idx / RP, j = idx % RP;
      const int m = mb + i;
      float v = 0.f;
      if (m < mb1 && j < R) v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(G)[static_cast<int64_t>(m) * R + j]);
      sG[i][j] = v;
    }
    __syncthreads();
    const int iend = min(64, mb1 - mb);
    if (c < C) {
      for (int i = 0; i < iend; ++i) {
        const uint32_t pv = __ldg(reinterpret_cast<const uint32_t*>(P + static_cast<int64_t>(mb + i) * C + c));
        const float p0 = __uint_as_float(pv << 16), p1 = __uint_as_float(pv & 0xffff0000u);
#pragma unroll
        for (int j = 0; j < RP; j += 4) {
          const float4 gv = *reinterpret_cast<const float4*>(&sG[i][j]);
          acc[j][0] = fmaf(gv.x, p0, acc[j][0]);
          acc[j][1] = fmaf(gv.x, p1, acc[j][1]);
          acc[j + 1][0] = fmaf(gv.y, p0, acc[j + 1][0]);
          acc[j + 1][1] = fmaf(gv.y, p1, acc[j + 1][1]);
          acc[j + 2][0] = fmaf(gv.z, p0, acc[j + 2][0]);
          acc[j + 2][1] = fmaf(gv.z, p1, acc[j + 2][1]);
          acc[j + 3][0] = fmaf(gv.w, p0, acc[j + 3][0]);
          acc[j + 3][1] = fmaf(gv.w, p1, acc[j + 3][1]);
        }
      }
    }
  }
  if (c < C) {
    float* dst = partial + static_cast<int64_t>(split) * R * C;
#pragma unroll
    for (int j = 0; j < RP; ++j)
      if (j < R) *reinterpret_cast<float2*>(dst + static_cast<int64_t>(j) * C + c) = make_float2(acc[j][0], acc[j][1]);
  }
}

// out = bf16(scale * sum_split partial[split]), as [R, C] or transposed [C, R].
__global__ void k_coldot_reduce(const float* __restrict__ partial, int splits, int R, int C, float scale,
                                int transpose, uint16_t* __restrict__ out) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(R) * C;
  if (idx >= total) return;
  // idx enumerates the output in its own row-major order
  int j, c;
  if (transpose) {
    c = static_cast<int>(idx / R);
    j = static_cast<int>(idx % R);
  } else {
    j = static_cast<int>(idx / C);
    c = static_cast<int>(idx % C);
  }
  float v = 0.f;
  for (int s = 0; s < splits; ++s) v += partial[static_cast<int64_t>(s) * total + static_cast<int64_t>(j) * C + c];
  const __nv_bfloat16 h = __float2bfloat16_rn(scale * v);
  out[idx] = *reinterpret_cast<const uint16_t*>(&h);
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
  const int64_t col_tiles = (C + 255) / 256;
  int64_t s = (4 * 148 + col_tiles - 1) / col_tiles;  // aim for ~4 CTAs per SM
  s = std::max<int64_t>(1, std::min<int64_t>(s, (M + 63) / 64));
  return static_cast<int>(s);
}

}  // namespace

cudaError_t launch_rowdot(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((M + 15) / 16);
  const int nt = (R + 7) / 8;
#define QN_ROWDOT(NTV)                                                                                   \
  case NTV:                                                                                              \
    k_rowdot<NTV><<<grid, 256, 0, st>>>(P, Q, static_cast<int>(M), static_cast<int>(Kc), R, sa, out16a, \
                                         sb, out16b, out32);                                             \
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
  const dim3 grid(static_cast<unsigned>((C + 255) / 256), static_cast<unsigned>(splits));
  if (M > 0) {
    if (R <= 8)
      k_coldot_partial<8><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (R <= 16)
      k_coldot_partial<16><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (R <= 32)
      k_coldot_partial<32><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else if (R <= 64)
      k_coldot_partial<64><<<grid, 128, 0, st>>>(G, P, int(M), int(C), R, rows_per_split, partial);
    else
      return cudaErrorInvalidValue;
  } else {
    cudaError_t e = cudaMemsetAsync(partial, 0, sizeof(float) * R * C, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = static_cast<int64_t>(R) * C;
  k_coldot_reduce<<<static_cast<unsigned>((total + 255) / 256), 256, 0, st>>>(partial, M > 0 ? splits : 1, R,
                                                                                int(C), scale, transpose, out);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const uint16_t* src, int64_t R, int64_t C, uint16_t* dst, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((R + 31) / 32));
  k_transpose_bf16<<<grid, dim3(32, 8), 0, st>>>(src, int(R), int(C), dst);
  return cudaGetLastError();
}

}  // namespace qn
