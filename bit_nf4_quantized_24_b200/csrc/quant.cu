// NF4 quantize (blockwise absmax + 4-bit codes + 8-bit double quantization of
// the absmax values) and dequantize kernels.  Both are HBM-bound streams.
//
// Method (katajob, "NF4: 4-bit NormalFloat" and "Double quantization"):
// each block of 64 contiguous weights is scaled by its absmax and every value
// is replaced by the index of the nearest of 16 levels; the per-block absmax
// values are themselves coded in 8 bits against one fp32 scale per group of
// 256 blocks.  Exact rules (shared with the CPU oracle by specification, not by
// code): t = fl32(w / a_b); code = number of midpoints strictly below t; an
// all-zero block encodes the zero level; s2 = fl32(max a / 255);
// q = min(255, rint(fl32(a / s2))).
#include "internal.h"

namespace qn {

namespace {

constexpr int kBlock = 64;
constexpr int kGroup = 256;  // blocks per double-quant group

// Code of t = fl32(w / a) in [-1, 1]: the number of midpoints strictly below
// t.  t is placed exactly on a grid of 129 cells of width 1/64 (cell j holds
// the t with rn(64 t) = j - 64); every cell holds at most one midpoint (their
// spacing is above 1/32) and none lies on a cell edge, so
// code = base[j] + (t > mid[j]) with base[j] = midpoints below the cell and
// mid[j] = the midpoint inside it (+inf if none).  rn(64 t) + 64 is read from
// the low mantissa bits of fl32(64 t + 1.5 * 2^23 + 64); the index is masked to
// 8 bits so a non-finite t (its block is reported) still reads inside the table.
struct Cell {
  int base;
  float mid;
};
constexpr int kCells = 256;

__device__ __forceinline__ int nf4_code(float t, const Cell* cells) {
  const float f = __fmaf_rn(t, 64.0f, 12582976.0f);
  const Cell c = cells[(__float_as_int(f) - 0x4B400000) & (kCells - 1)];
  return c.base + (t > c.mid ? 1 : 0);
}

// fl32(w / a), correctly rounded, from the block's reciprocal r = fl32(1 / a):
// Markstein's refinement (q0 = fl32(w r) is within one ulp of w / a, the
// residual w - q0 a is exact with an FMA, and q0 + residual * r rounded once is
// the correctly rounded quotient), valid while a and 1 / a are normal numbers;
// callers use it for 2^-100 <= a <= 2^100.  Where the quotient is too small for
// the refinement's assumptions it is far below the smallest midpoint magnitude
// and the code does not depend on its last bits.
__device__ __forceinline__ float div_by_absmax(float w, float a, float r) {
  const float q0 = __fmul_rn(w, r);
  const float e = __fmaf_rn(-q0, a, w);
  return __fmaf_rn(e, r, q0);
}

// One CTA per double-quant group (256 blocks = 16384 weights, 64 KB of fp32).
// A warp covers two blocks per step: 16 lanes per block, one float4 per lane.
// Four steps' loads are issued before any is used, to keep HBM busy.
__global__ void __launch_bounds__(256) k_quantize(const float* __restrict__ W, int64_t nblocks, Nf4Mids mids,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ absmax_q,
                                                  float* __restrict__ dq_scale, int* nonfinite) {
  __shared__ Cell s_cell[kCells];
  __shared__ float s_amax[kGroup];
  __shared__ float s_red[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, sl = lane & 15;
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kGroup;
  const int64_t rem = nblocks - b0;
  const int nb = rem < kGroup ? static_cast<int>(rem) : kGroup;
  {  // cell table (kCells == blockDim.x)
    const float lo = (static_cast<float>(tid) - 64.5f) * 0.015625f, hi = lo + 0.015625f;
    int base = 0;
    float mid = __int_as_float(0x7f800000);
    for (int i = 0; i < 15; ++i) {
      base += mids.v[i] < lo ? 1 : 0;
      if (mids.v[i] > lo && mids.v[i] < hi) mid = mids.v[i];
    }
    s_cell[tid] = Cell{base, mid};
  }
  __syncthreads();

  const int npairs = (nb + 1) >> 1;
  float nan_probe = 0.0f;  // becomes NaN if any weight is NaN or infinite (x * 0)
  for (int p0 = warp; p0 < npairs; p0 += 32) {
    float4 x[4];
    bool ok[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = 2 * (p0 + 8 * u) + half;
      ok[u] = (p0 + 8 * u < npairs) && (i < nb);
      x[u] = ok[u] ? __ldcs(reinterpret_cast<const float4*>(W + (b0 + i) * kBlock) + sl)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (p0 + 8 * u >= npairs) break;  // warp-uniform
      const int i = 2 * (p0 + 8 * u) + half;
      nan_probe = __fmaf_rn(x[u].x, 0.0f, __fmaf_rn(x[u].y, 0.0f, __fmaf_rn(x[u].z, 0.0f, __fmaf_rn(x[u].w, 0.0f, nan_probe))));
      float m = fmaxf(fmaxf(fabsf(x[u].x), fabsf(x[u].y)), fmaxf(fabsf(x[u].z), fabsf(x[u].w)));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (ok[u]) {
        uint32_t c;
        if (m == 0.0f) {
          c = 0x7777u;  // an all-zero block encodes the zero level
        } else if (m >= 0x1p-100f && m <= 0x1p100f) {
          const float r = __frcp_rn(m);
          c = nf4_code(div_by_absmax(x[u].x, m, r), s_cell) | (nf4_code(div_by_absmax(x[u].y, m, r), s_cell) << 4) |
              (nf4_code(div_by_absmax(x[u].z, m, r), s_cell) << 8) |
              (nf4_code(div_by_absmax(x[u].w, m, r), s_cell) << 12);
        } else {
          c = nf4_code(__fdiv_rn(x[u].x, m), s_cell) | (nf4_code(__fdiv_rn(x[u].y, m), s_cell) << 4) |
              (nf4_code(__fdiv_rn(x[u].z, m), s_cell) << 8) | (nf4_code(__fdiv_rn(x[u].w, m), s_cell) << 12);
        }
        reinterpret_cast<uint16_t*>(codes + (b0 + i) * (kBlock / 2))[sl] = static_cast<uint16_t>(c);
        if (sl == 0) s_amax[i] = m;
      }
    }
  }
  const bool bad = !(nan_probe == 0.0f);
  __syncthreads();

  // double quantization of the group's absmax values
  float m = (tid < nb) ? s_amax[tid] : 0.0f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  float c2 = s_red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) c2 = fmaxf(c2, s_red[w]);
  const float s2 = (c2 > 0.0f) ? __fdiv_rn(c2, 255.0f) : 0.0f;
  if (tid < nb) {
    uint8_t q = 0;
    if (s2 != 0.0f) q = static_cast<uint8_t>(fminf(255.0f, rintf(__fdiv_rn(s_amax[tid], s2))));
    absmax_q[b0 + tid] = q;
  }
  if (tid == 0) dq_scale[g] = s2;
  if (__syncthreads_or(bad) && tid == 0) atomicExch(nonfinite, 1);
}

// One thread expands one 64-weight block (one register table, 32 code bytes
// in, 128 bytes of bf16 out); a warp's 32 blocks pass through shared memory
// (16-byte chunks XOR-swizzled by lane) so that the global stores are 512
// contiguous bytes per instruction.
__global__ void __launch_bounds__(256) k_dequantize(const uint8_t* __restrict__ codes,
                                                    const uint8_t* __restrict__ absmax_q,
                                                    const float* __restrict__ dq_scale, int64_t nblocks,
                                                    Nf4Levels L, uint16_t* __restrict__ out) {
  __shared__ uint4 s_out[8][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wb0 = (static_cast<int64_t>(blockIdx.x) * 8 + warp) * 32;  // first block of this warp
  const int64_t b = wb0 + lane;
  if (wb0 >= nblocks) return;  // warp-uniform
  if (b < nblocks) {
    const uint4 c0 = ldg_nc_v4(codes + b * 32);
    const uint4 c1 = ldg_nc_v4(codes + b * 32 + 16);
    const float ap = __fmul_rn(static_cast<float>(absmax_q[b]), dq_scale[b / kGroup]);
    const Nf4Lut t = make_lut(L, ap);
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint4 o;
      deq8(w[i], t, o.x, o.y, o.z, o.w);
      s_out[warp][lane * 8 + (i ^ (lane & 7))] = o;
    }
  }
  __syncwarp();
  const int64_t nchunks = (nblocks - wb0 < 32 ? nblocks - wb0 : 32) * 8;
  uint4* dst = reinterpret_cast<uint4*>(out + wb0 * kBlock);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = i * 32 + lane;  // chunk q of the warp's 32 x 128 bytes
    if (q < nchunks) __stcs(dst + q, s_out[warp][(q >> 3) * 8 + ((q & 7) ^ ((q >> 3) & 7))]);
  }
}

}  // namespace

cudaError_t launch_quantize(const float* W, int64_t numel, uint8_t* codes, uint8_t* absmax_q, float* dq_scale,
                            int* nonfinite, cudaStream_t st) {
  const int64_t nblocks = numel / kBlock;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  if (ngroups == 0) return cudaSuccess;
  k_quantize<<<static_cast<unsigned>(ngroups), 256, 0, st>>>(W, nblocks, host_codebook().mids, codes, absmax_q,
                                                            dq_scale, nonfinite);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t numel,
                              uint16_t* out, cudaStream_t st) {
  const int64_t nblocks = numel / kBlock;
  if (nblocks == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((nblocks + 255) / 256);  // 8 warps x 32 blocks per CTA
  k_dequantize<<<grid, 256, 0, st>>>(codes, absmax_q, dq_scale, nblocks, host_codebook().levels, out);
  return cudaGetLastError();
}

}  // namespace qn
