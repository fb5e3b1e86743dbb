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

__device__ __forceinline__ int nf4_code(float v, float m, const float* s_mid) {
  if (m == 0.0f) return 7;
  const float t = __fdiv_rn(v, m);
  int c = 0;
  if (t > s_mid[c + 7]) c += 8;
  if (t > s_mid[c + 3]) c += 4;
  if (t > s_mid[c + 1]) c += 2;
  if (t > s_mid[c]) c += 1;
  return c;
}

// One CTA per double-quant group (256 blocks = 16384 weights, 64 KB of fp32).
// A warp covers two blocks per step: 16 lanes per block, one float4 per lane.
// Four steps' loads are issued before any is used, to keep HBM busy.
__global__ void __launch_bounds__(256) k_quantize(const float* __restrict__ W, int64_t nblocks, Nf4Mids mids,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ absmax_q,
                                                  float* __restrict__ dq_scale, int* nonfinite) {
  __shared__ float s_mid[16];
  __shared__ float s_amax[kGroup];
  __shared__ float s_red[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = lane >> 4, sl = lane & 15;
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kGroup;
  const int64_t rem = nblocks - b0;
  const int nb = rem < kGroup ? static_cast<int>(rem) : kGroup;
  if (tid < 15) s_mid[tid] = mids.v[tid];
  if (tid == 15) s_mid[15] = __int_as_float(0x7f800000);  // +inf sentinel
  __syncthreads();

  const int npairs = (nb + 1) >> 1;
  bool bad = false;
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
      bad |= !(isfinite(x[u].x) && isfinite(x[u].y) && isfinite(x[u].z) && isfinite(x[u].w));
      float m = fmaxf(fmaxf(fabsf(x[u].x), fabsf(x[u].y)), fmaxf(fabsf(x[u].z), fabsf(x[u].w)));
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (ok[u]) {
        const uint32_t c = nf4_code(x[u].x, m, s_mid) | (nf4_code(x[u].y, m, s_mid) << 4) |
                           (nf4_code(x[u].z, m, s_mid) << 8) | (nf4_code(x[u].w, m, s_mid) << 12);
        reinterpret_cast<uint16_t*>(codes + (b0 + i) * (kBlock / 2))[sl] = static_cast<uint16_t>(c);
        if (sl == 0) s_amax[i] = m;
      }
    }
  }
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

// One thread per 64-weight block: one register table, 32 code bytes in,
// 128 bytes of bf16 out.
__global__ void __launch_bounds__(256) k_dequantize(const uint8_t* __restrict__ codes,
                                                    const uint8_t* __restrict__ absmax_q,
                                                    const float* __restrict__ dq_scale, int64_t nblocks,
                                                    Nf4Levels L, uint16_t* __restrict__ out) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
  const uint4 c0 = ldg_nc_v4(codes + b * 32);
  const uint4 c1 = ldg_nc_v4(codes + b * 32 + 16);
  const float ap = __fmul_rn(static_cast<float>(absmax_q[b]), dq_scale[b / kGroup]);
  const Nf4Lut t = make_lut(L, ap);
  uint4* dst = reinterpret_cast<uint4*>(out + b * kBlock);
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint4 o;
    deq8(w[i], t, o.x, o.y, o.z, o.w);
    __stcs(dst + i, o);
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
  const unsigned grid = static_cast<unsigned>((nblocks + 255) / 256);
  k_dequantize<<<grid, 256, 0, st>>>(codes, absmax_q, dq_scale, nblocks, host_codebook().levels, out);
  return cudaGetLastError();
}

}  // namespace qn
