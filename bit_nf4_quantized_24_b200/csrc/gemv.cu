// Decode-sized forward (M <= 16 tokens): Y = X deq(W)^T + Hs B^T, Hs = bf16(s X A^T).
// Bound by streaming the NF4 weight once (katajob, "NF4: 4-bit NormalFloat":
// the weight is read in 4-bit and expanded per block only inside the product).
//
// CTA = 8 warps = 2 row groups (16 weight rows each) x 4 K splits.  Per
// 256-wide K slice a lane reads one full 64-weight block (32 code bytes) of one
// row, builds that block's register lookup table and expands it straight into
// m16n8k16 B fragments -- the dequantized weight never touches memory.  Lane
// t's block supplies k-slots {2t, 2t+1, 2t+8, 2t+9} of 16 MMA steps; the
// activation fragments are read (through L1) in the same permuted k order.
// Code blocks are prefetched two slices ahead in registers; the four K splits
// of a row group are summed in shared memory at the end.
#include "internal.h"

namespace qn {

namespace {

constexpr int GV_RG = 2;   // row groups (16 rows each) per CTA
constexpr int GV_KS = 4;   // K splits per CTA
constexpr int GV_THREADS = GV_RG * GV_KS * 32;

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct Slice {  // one lane's code block for one n8 tile
  uint4 q0, q1;
  float ap;
};

__device__ __forceinline__ Slice load_slice(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                                            const float* __restrict__ dq_scale, int row, int N, int KB, int kblk) {
  Slice s;
  if (row < N && kblk < KB) {
    const uint8_t* p = codes + (static_cast<int64_t>(row) * KB + kblk) * 32;
    s.q0 = ldg_nc_v4(p);
    s.q1 = ldg_nc_v4(p + 16);
    const int64_t b = static_cast<int64_t>(row) * KB + kblk;
    s.ap = __fmul_rn(static_cast<float>(__ldg(absmax_q + b)), __ldg(dq_scale + (b >> 8)));
  } else {
    s.q0 = s.q1 = make_uint4(0u, 0u, 0u, 0u);
    s.ap = 0.0f;
  }
  return s;
}

__device__ __forceinline__ void slice_mma(float (&acc)[4], const Slice& sl, const Nf4Levels& lv, const uint4 (&alo)[8],
                                          const uint4 (&ahi)[8]) {
  const Nf4Lut lut = make_lut(lv, sl.ap);
  const uint32_t w[8] = {sl.q0.x, sl.q0.y, sl.q0.z, sl.q0.w, sl.q1.x, sl.q1.y, sl.q1.z, sl.q1.w};
#pragma unroll
  for (int ip = 0; ip < 8; ++ip) {
    uint32_t o0, o1, o2, o3;
    deq8(w[ip], lut, o0, o1, o2, o3);
    mma16816(acc, alo[ip].x, ahi[ip].x, alo[ip].y, ahi[ip].y, o0, o1);
    mma16816(acc, alo[ip].z, ahi[ip].z, alo[ip].w, ahi[ip].w, o2, o3);
  }
}

__global__ void __launch_bounds__(GV_THREADS, 2) k_gemv(const uint16_t* __restrict__ X, int M,
                                                         const uint8_t* __restrict__ codes,
                                                         const uint8_t* __restrict__ absmax_q,
                                                         const float* __restrict__ dq_scale, int N, int K,
                                                         const uint16_t* __restrict__ Hs,
                                                         const uint16_t* __restrict__ Bl, int r, Nf4Levels lv,
                                                         uint16_t* __restrict__ Y) {
  __shared__ float red[GV_RG][GV_KS][2][4][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int rg = warp % GV_RG, ks = warp / GV_RG;
  const int nrow0 = (blockIdx.x * GV_RG + rg) * 16;
  const int KB = K / 64;
  const int nsub = (K + 255) / 256;
  const bool lo_ok = g < M, hi_ok = g + 8 < M;
  const uint16_t* xlo = X + static_cast<int64_t>(g) * K + 64 * t;
  const uint16_t* xhi = X + static_cast<int64_t>(g + 8) * K + 64 * t;

  float acc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  // two slices in flight: (c0, c1) for sub, (n0, n1) for sub + GV_KS
  Slice c0 = load_slice(codes, absmax_q, dq_scale, nrow0 + g, N, KB, ks * 4 + t);
  Slice c1 = load_slice(codes, absmax_q, dq_scale, nrow0 + 8 + g, N, KB, ks * 4 + t);
  for (int sub = ks; sub < nsub; sub += GV_KS) {
    const int nxt = sub + GV_KS;
    const Slice n0 = load_slice(codes, absmax_q, dq_scale, nrow0 + g, N, KB, nxt * 4 + t);
    const Slice n1 = load_slice(codes, absmax_q, dq_scale, nrow0 + 8 + g, N, KB, nxt * 4 + t);
    uint4 alo[8], ahi[8];
    const int kb = sub * 256;
    const bool kin = kb + 64 * t < K;
#pragma unroll
    for (int ip = 0; ip < 8; ++ip) {
      alo[ip] = (lo_ok && kin) ? __ldg(reinterpret_cast<const uint4*>(xlo + kb + 8 * ip)) : make_uint4(0, 0, 0, 0);
      ahi[ip] = (hi_ok && kin) ? __ldg(reinterpret_cast<const uint4*>(xhi + kb + 8 * ip)) : make_uint4(0, 0, 0, 0);
    }
    slice_mma(acc[0], c0, lv, alo, ahi);
    slice_mma(acc[1], c1, lv, alo, ahi);
    c0 = n0;
    c1 = n1;
  }

#pragma unroll
  for (int tile = 0; tile < 2; ++tile)
#pragma unroll
    for (int i = 0; i < 4; ++i) red[rg][ks][tile][i][lane] = acc[tile][i];
  __syncthreads();
  if (ks != 0) return;
#pragma unroll
  for (int tile = 0; tile < 2; ++tile)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < GV_KS; ++q) v += red[rg][q][tile][i][lane];
      acc[tile][i] = v;
    }

  // LoRA term: + Hs[m, :] . B[n, :] in k16 steps over r (standard fragment order)
  for (int j0 = 0; j0 < r; j0 += 16) {
    auto ld2 = [&](const uint16_t* base, int row, int rows, int j) -> uint32_t {
      if (row >= rows || j >= r) return 0u;
      return __ldg(reinterpret_cast<const uint32_t*>(base + static_cast<int64_t>(row) * r + j));
    };
    const uint32_t a0 = ld2(Hs, g, M, j0 + 2 * t), a1 = ld2(Hs, g + 8, M, j0 + 2 * t);
    const uint32_t a2 = ld2(Hs, g, M, j0 + 2 * t + 8), a3 = ld2(Hs, g + 8, M, j0 + 2 * t + 8);
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
      const int n = nrow0 + 8 * tile + g;
      mma16816(acc[tile], a0, a1, a2, a3, ld2(Bl, n, N, j0 + 2 * t), ld2(Bl, n, N, j0 + 2 * t + 8));
    }
  }

#pragma unroll
  for (int tile = 0; tile < 2; ++tile) {
    const int n = nrow0 + 8 * tile + 2 * t;
    if (n >= N) continue;
    if (g < M)
      *reinterpret_cast<uint32_t*>(Y + static_cast<int64_t>(g) * N + n) = bf16x2_bits(acc[tile][0], acc[tile][1]);
    if (g + 8 < M)
      *reinterpret_cast<uint32_t*>(Y + static_cast<int64_t>(g + 8) * N + n) = bf16x2_bits(acc[tile][2], acc[tile][3]);
  }
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* X, int64_t M, const uint8_t* codes, const uint8_t* absmax_q,
                        const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B, int r,
                        uint16_t* Y, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((N + 16 * GV_RG - 1) / (16 * GV_RG));
  k_gemv<<<grid, GV_THREADS, 0, st>>>(X, int(M), codes, absmax_q, dq_scale, int(N), int(K), Hs, B, r,
                                          host_codebook().levels, Y);
  return cudaGetLastError();
}

}  // namespace qn
