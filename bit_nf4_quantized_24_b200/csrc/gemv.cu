// Decode-sized forward (M <= 16 tokens): Y = X deq(W)^T + Hs B^T, Hs = bf16(s X A^T).
// Bound by streaming the NF4 weight once (katajob, "NF4: 4-bit NormalFloat":
// the weight is read in 4-bit and expanded per block only inside the product).
//
// Expansion.  A code byte holds two weights; a 256-entry table maps it to the
// two levels as a bf16 pair.  The table lives in shared memory replicated
// once per lane (entry e of lane l at T + 256 e + 4 l), so every lookup of a
// warp is conflict-free, and T is 64 KB aligned, so one prmt assembles the
// address from the code byte and the lane's base: 1 prmt + 1 ld.shared per two
// weights, with no per-block table to build.  The per-block scale is applied
// afterwards: the four m16n8k16 steps of one 64-weight block accumulate into a
// fresh fragment, which is then added with the block's scale.  For this each
// MMA step must stay inside one block: lane t contributes k = 16t + 4s + 0..3
// at step s (its 8 code bytes 8t .. 8t+7 of the block), and the activation
// fragments are read in the same permuted order.
//
// Schedule.  One persistent CTA per SM, 8 warps.  A task is 32 weight rows:
// the 8 warps split the task's blocks along K, each warp handles the 32 rows
// as four n8 tiles with its code blocks (and scales) loaded G_DEPTH blocks
// ahead into a register ring, and the partial sums meet in shared memory
// (fixed order, so the result is deterministic).
#include <algorithm>

#include "internal.h"

namespace qn {

namespace {

constexpr int G_WARPS = 8;
constexpr int G_DEPTH = 6;                        // code blocks in flight per warp
constexpr int G_THREADS = G_WARPS * 32;
constexpr int G_ROWS = 32;                        // weight rows per task (4 n8 tiles)
constexpr int G_RED_BYTES = G_WARPS * 4 * 4 * 32 * 4;  // partial sums of one task
constexpr int G_TABLE_BYTES = 256 * 256;          // 256 entries x 256 B (128 B used)
constexpr int G_SMEM = G_TABLE_BYTES + 65536 + G_RED_BYTES;  // room to align the table to 64 KB

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// bf16x2 pair of the levels of a code byte, from the lane's table copy:
// address = [lane base byte 0, code byte, table base bytes 2-3].
template <int BYTE>
__device__ __forceinline__ uint32_t lut_pair(uint32_t word, uint32_t lane_base) {
  return lds32(prmt(word, lane_base, 0x7604u | (BYTE << 4)));
}

struct RowScale {
  float ap0, ap1;  // block scales of W rows 2t and 2t+1 of an n8 tile
};

__global__ void __launch_bounds__(G_THREADS, 1) k_gemv(const uint16_t* __restrict__ X, int M,
                                                        const uint8_t* __restrict__ codes,
                                                        const uint8_t* __restrict__ absmax_q,
                                                        const float* __restrict__ dq_scale, int N, int K,
                                                        const uint16_t* __restrict__ Hs,
                                                        const uint16_t* __restrict__ Bl, int r, Nf4Levels lv,
                                                        uint16_t* __restrict__ Y, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t table = (raw + 65535u) & ~65535u;
  if (table + G_TABLE_BYTES + G_RED_BYTES > raw + G_SMEM) {  // cannot happen with G_SMEM; never index past it
    if (threadIdx.x == 0) atomicExch(status, kDevTimeout);
    return;
  }
  float* red = reinterpret_cast<float*>(smem_raw + (table - raw) + G_TABLE_BYTES);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  // table: entry e -> {bf16(L[e & 15]), bf16(L[e >> 4])}, one copy per lane
  for (int idx = tid; idx < 256 * 32; idx += G_THREADS) {
    const int e = idx >> 5, l = idx & 31;
    const uint32_t v = bf16x2_bits(lv.v[e & 15], lv.v[e >> 4]);
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(table + e * 256 + l * 4), "r"(v) : "memory");
  }
  __syncthreads();
  const uint32_t lane_base = table + lane * 4;

  const int KB = K / 64;
  const int b_lo = (warp * KB) / G_WARPS, b_hi = ((warp + 1) * KB) / G_WARPS;  // this warp's blocks
  const bool lo_ok = g < M, hi_ok = g + 8 < M;
  const int ntasks = (N + G_ROWS - 1) / G_ROWS;

  for (int task = blockIdx.x; task < ntasks; task += gridDim.x) {
    const int n0 = task * G_ROWS;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    // per tile: this lane's code row and the two rows whose scales it applies
    const int crow[4] = {n0 + g, n0 + 8 + g, n0 + 16 + g, n0 + 24 + g};
    auto load_codes = [&](int b, uint2 (&cw)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        cw[i] = (crow[i] < N && b < b_hi)
                    ? ldg_nc_v2(codes + (static_cast<int64_t>(crow[i]) * KB + b) * 32 + 8 * t)
                    : make_uint2(0u, 0u);
    };
    auto load_scales = [&](int b, RowScale (&sc)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r0 = n0 + 8 * i + 2 * t;
        float a[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          a[h] = 0.0f;
          if (r0 + h < N && b < b_hi) {
            const int64_t blk = static_cast<int64_t>(r0 + h) * KB + b;
            a[h] = __fmul_rn(static_cast<float>(__ldg(absmax_q + blk)), __ldg(dq_scale + (blk >> 8)));
          }
        }
        sc[i].ap0 = a[0];
        sc[i].ap1 = a[1];
      }
    };

    // register ring of G_DEPTH blocks: slot j holds block b_lo + j (mod G_DEPTH)
    uint2 cw[G_DEPTH][4];
    RowScale sc[G_DEPTH][4];
#pragma unroll
    for (int j = 0; j < G_DEPTH; ++j) {
      load_codes(b_lo + j, cw[j]);
      load_scales(b_lo + j, sc[j]);
    }
    for (int b0 = b_lo; b0 < b_hi; b0 += G_DEPTH) {
#pragma unroll
      for (int j = 0; j < G_DEPTH; ++j) {
        const int b = b0 + j;
        if (b >= b_hi) break;
        // activation fragments of this block: X[row][64b + 16t .. +15]
        uint4 x0 = make_uint4(0, 0, 0, 0), x1 = x0, y0 = x0, y1 = x0;
        if (lo_ok) {
          const uint4* p = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(g) * K + 64 * b + 16 * t);
          x0 = __ldg(p);
          x1 = __ldg(p + 1);
        }
        if (hi_ok) {
          const uint4* p = reinterpret_cast<const uint4*>(X + static_cast<int64_t>(g + 8) * K + 64 * b + 16 * t);
          y0 = __ldg(p);
          y1 = __ldg(p + 1);
        }
        const uint32_t xg[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        const uint32_t xh[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint2 c = cw[j][i];
          float tmp[4] = {0.f, 0.f, 0.f, 0.f};
          mma16816(tmp, xg[0], xh[0], xg[1], xh[1], lut_pair<0>(c.x, lane_base), lut_pair<1>(c.x, lane_base));
          mma16816(tmp, xg[2], xh[2], xg[3], xh[3], lut_pair<2>(c.x, lane_base), lut_pair<3>(c.x, lane_base));
          mma16816(tmp, xg[4], xh[4], xg[5], xh[5], lut_pair<0>(c.y, lane_base), lut_pair<1>(c.y, lane_base));
          mma16816(tmp, xg[6], xh[6], xg[7], xh[7], lut_pair<2>(c.y, lane_base), lut_pair<3>(c.y, lane_base));
          acc[i][0] = fmaf(sc[j][i].ap0, tmp[0], acc[i][0]);
          acc[i][1] = fmaf(sc[j][i].ap1, tmp[1], acc[i][1]);
          acc[i][2] = fmaf(sc[j][i].ap0, tmp[2], acc[i][2]);
          acc[i][3] = fmaf(sc[j][i].ap1, tmp[3], acc[i][3]);
        }
        load_codes(b + G_DEPTH, cw[j]);  // refill the slot G_DEPTH blocks ahead
        load_scales(b + G_DEPTH, sc[j]);
      }
    }

    // K-split partial sums meet in shared memory
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) red[((warp * 4 + i) * 4 + c) * 32 + lane] = acc[i][c];
    __syncthreads();
    if (warp < 4) {  // warp i finishes tile i: sum, LoRA term, store
      const int i = warp;
      float v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float s = 0.f;
        for (int w = 0; w < G_WARPS; ++w) s += red[((w * 4 + i) * 4 + c) * 32 + lane];
        v[c] = s;
      }
      // + Hs[m, :] . B[n, :] in k16 steps over r (standard fragment order)
      for (int j0 = 0; j0 < r; j0 += 16) {
        auto ld2 = [&](const uint16_t* base_p, int row, int rows, int j) -> uint32_t {
          if (row >= rows || j >= r) return 0u;
          return __ldg(reinterpret_cast<const uint32_t*>(base_p + static_cast<int64_t>(row) * r + j));
        };
        const int n = n0 + 8 * i + g;
        mma16816(v, ld2(Hs, g, M, j0 + 2 * t), ld2(Hs, g + 8, M, j0 + 2 * t), ld2(Hs, g, M, j0 + 2 * t + 8),
                 ld2(Hs, g + 8, M, j0 + 2 * t + 8), ld2(Bl, n, N, j0 + 2 * t), ld2(Bl, n, N, j0 + 2 * t + 8));
      }
      const int n = n0 + 8 * i + 2 * t;
      if (n < N) {
        if (g < M) *reinterpret_cast<uint32_t*>(Y + static_cast<int64_t>(g) * N + n) = bf16x2_bits(v[0], v[1]);
        if (g + 8 < M)
          *reinterpret_cast<uint32_t*>(Y + static_cast<int64_t>(g + 8) * N + n) = bf16x2_bits(v[2], v[3]);
      }
    }
    __syncthreads();  // red is reused by the next task
  }
}

}  // namespace

cudaError_t launch_gemv(const uint16_t* X, int64_t M, const uint8_t* codes, const uint8_t* absmax_q,
                        const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B, int r,
                        uint16_t* Y, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(k_gemv, cudaFuncAttributeMaxDynamicSharedMemorySize, G_SMEM);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t ntasks = (N + G_ROWS - 1) / G_ROWS;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ntasks, sms));
  k_gemv<<<grid, G_THREADS, G_SMEM, st>>>(X, int(M), codes, absmax_q, dq_scale, int(N), int(K), Hs, B, r,
                                           host_codebook().levels, Y, device_status_ptr());
  return cudaGetLastError();
}

}  // namespace qn
