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
#include <atomic>
#include <mutex>

#include "internal.h"

namespace qn {

namespace {

constexpr int kGroup = 256;  // blocks per double-quant group (and per quantize CTA)

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

// The cell table is a function of the codebook alone: built once on the host
// (cell j covers [(j - 64.5) / 64, (j - 63.5) / 64), the same fp32 expressions
// the code below relies on) and copied to each device at its first use.
__device__ Cell g_cells[kCells];

void build_cells(const Nf4Mids& mids, Cell* out) {
  for (int j = 0; j < kCells; ++j) {
    const float lo = (static_cast<float>(j) - 64.5f) * 0.015625f, hi = lo + 0.015625f;
    int base = 0;
    float mid = __builtin_huge_valf();
    for (int i = 0; i < 15; ++i) {
      base += mids.v[i] < lo ? 1 : 0;
      if (mids.v[i] > lo && mids.v[i] < hi) mid = mids.v[i];
    }
    out[j] = Cell{base, mid};
  }
}

// Device address of the cell table on the current device, uploaded the first
// time it is asked for there (nullptr and the error on failure).
const Cell* device_cells(cudaError_t* err) {
  static std::atomic<uint64_t> done{0};
  static std::mutex mu;
  static Cell host[kCells];
  static std::once_flag built;
  std::call_once(built, [] { build_cells(host_codebook().mids, host); });
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_cells);
  if (*err != cudaSuccess) return nullptr;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (!bit || !(done.load(std::memory_order_acquire) & bit)) {
    std::lock_guard<std::mutex> lock(mu);
    if (!bit || !(done.load(std::memory_order_acquire) & bit)) {
      *err = cudaMemcpy(p, host, sizeof(host), cudaMemcpyHostToDevice);
      if (*err != cudaSuccess) return nullptr;
      if (bit) done.fetch_or(bit, std::memory_order_release);
    }
  }
  return static_cast<const Cell*>(p);
}

// The index of t's cell is the low 8 bits of fl32(64 t + 1.5 * 2^23 + 64)
// (the bias has zeros there), masked so that any t reads inside the table.
__device__ __forceinline__ int nf4_code(float t, const Cell* cells) {
  const float f = __fmaf_rn(t, 64.0f, 12582976.0f);
  const Cell c = cells[__float_as_int(f) & (kCells - 1)];
  return c.base + (t > c.mid ? 1 : 0);
}

// max with NaN propagation (IEEE maximum): a NaN operand gives NaN, so the
// block maximum of |w| is NaN or infinite exactly when the block holds a
// non-finite weight.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
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

// Source of the values to quantize: an fp32 weight, or (merge) the NF4 weight
// the layer uses plus the folded adapter ("QLoRA and Quantized Fine-Tuning",
// "The two mechanisms combined": the merged model computes with W' + BA):
//   merged[n, k] = fl32(w'[n, k] + fl32(s * sum_j B[n, j] A[j, k])),
// w' = bf16(L[code] * a') as dequantized for the layer, the sum in fp32 in the
// order j = 0 .. r-1 (every product of two bf16 values is exact in fp32, so
// each FMA adds one exact product).
struct MergeSrc {
  const uint8_t* codes;
  const uint8_t* absmax_q;
  const float* dq_scale;
  int lg;  // log2 of the input block size
  int dq;  // input has double quantization
  const uint16_t* A;  // bf16 [r, K]
  const uint16_t* B;  // bf16 [N, r]
  int r;
  float s;
  int64_t K;
};

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// Merged values of the F groups of 4 elements e0 + f * STRIDE + 0..3
// (f < F; all in one row, one output block; each group inside one input
// block); lv: the 16 levels in shared memory.  B[n, j] is loaded once per j
// for all F groups; A[j, k..k+3] with one 8-byte load per group and j.
template <int F, int STRIDE>
__device__ __forceinline__ void mergedF(const MergeSrc& m, const float* lv, int64_t e0, float4 (&x)[F]) {
  const int64_t n = e0 / m.K, k0 = e0 - n * m.K;
  float acc[F][4];
#pragma unroll
  for (int f = 0; f < F; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.f;
  const uint16_t* arow = m.A + k0;
  const uint16_t* brow = m.B + n * m.r;
  for (int j = 0; j < m.r; ++j) {
    const float bj = bf16_bits_to_f32(__ldg(brow + j));
    const uint16_t* aj = arow + static_cast<int64_t>(j) * m.K;
#pragma unroll
    for (int f = 0; f < F; ++f) {
      const uint2 a4 = __ldg(reinterpret_cast<const uint2*>(aj + f * STRIDE));
      acc[f][0] = __fmaf_rn(bj, __uint_as_float(a4.x << 16), acc[f][0]);
      acc[f][1] = __fmaf_rn(bj, __uint_as_float(a4.x & 0xffff0000u), acc[f][1]);
      acc[f][2] = __fmaf_rn(bj, __uint_as_float(a4.y << 16), acc[f][2]);
      acc[f][3] = __fmaf_rn(bj, __uint_as_float(a4.y & 0xffff0000u), acc[f][3]);
    }
  }
#pragma unroll
  for (int f = 0; f < F; ++f) {
    const int64_t e = e0 + f * STRIDE;
    const int64_t b = e >> m.lg;  // the input block of this group
    const float a = m.dq ? __fmul_rn(static_cast<float>(m.absmax_q[b]), m.dq_scale[b >> 8]) : m.dq_scale[b];
    const uint32_t c = *reinterpret_cast<const uint16_t*>(m.codes + e / 2);
    float w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(lv[(c >> (4 * i)) & 15u], a)));
    x[f] = make_float4(__fadd_rn(w[0], __fmul_rn(m.s, acc[f][0])), __fadd_rn(w[1], __fmul_rn(m.s, acc[f][1])),
                       __fadd_rn(w[2], __fmul_rn(m.s, acc[f][2])), __fadd_rn(w[3], __fmul_rn(m.s, acc[f][3])));
  }
}

// One CTA per group of 256 blocks (the double-quant group).  A block of B
// weights is spread over LP = B / 16 lanes with F = 4 float4s (16 weights) per
// lane, so the block maximum needs log2(LP) shuffles and one reciprocal per 16
// weights; a warp step covers 32 / LP blocks and each warp issues the loads of
// U steps before it uses any, to keep HBM busy.  A block whose maximum is not
// finite (NaN or infinity inside) is reported and not coded.  DQ: double
// quantization of the group's absmax values (else each block's fp32 absmax is
// stored as is).
// Bulk copy of `bytes` (a multiple of 16) from global to this CTA's shared
// memory, completing on the mbarrier at `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <int B, bool DQ, bool MERGE>
__global__ void __launch_bounds__(256, 3) k_quantize(const float* __restrict__ W, MergeSrc msrc, Nf4Levels levels,
                                                  int64_t nblocks, const Cell* __restrict__ cells,
                                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ absmax_q,
                                                  float* __restrict__ dq_scale, int* nonfinite) {
  constexpr int F = 4;
  constexpr int LP = B / (4 * F);  // 2, 4, 8, 16
  constexpr int BPW = 32 / LP;     // blocks per warp step
  constexpr int U = MERGE ? 1 : 2; // warp steps whose loads are in flight together
  __shared__ Cell s_cell[kCells];
  __shared__ float s_amax[kGroup];
  __shared__ float s_red[8];
  __shared__ float s_lv[16];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / LP, sl = lane % LP;
  if (MERGE && tid < 16) s_lv[tid] = levels.v[tid];
  s_cell[tid] = cells[tid];  // kCells == blockDim.x
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * kGroup;
  const int64_t rem = nblocks - b0;
  const int nb = rem < kGroup ? static_cast<int>(rem) : kGroup;
  __syncthreads();

  const int nsteps = (nb + BPW - 1) / BPW;
  bool bad = false;
  for (int p0 = warp; p0 < nsteps; p0 += 8 * U) {  // steps p0, p0 + 8, ..., p0 + 8 (U - 1)
    float4 x[U][F];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = BPW * (p0 + 8 * u) + sub;
      ok[u] = (p0 + 8 * u < nsteps) && (i < nb);
      if (MERGE) {
        if (ok[u]) {
          mergedF<F, 4 * LP>(msrc, s_lv, (b0 + i) * B + sl * 4, x[u]);
        } else {
#pragma unroll
          for (int f = 0; f < F; ++f) x[u][f] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      } else {
#pragma unroll
        for (int f = 0; f < F; ++f)
          x[u][f] = ok[u] ? __ldcs(reinterpret_cast<const float4*>(W + (b0 + i) * B) + f * LP + sl)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (p0 + 8 * u >= nsteps) break;  // warp-uniform
      const int i = BPW * (p0 + 8 * u) + sub;
      float m = 0.0f;
#pragma unroll
      for (int f = 0; f < F; ++f) {
        const float4 v = x[u][f];
        m = fmax_nan(m, fmax_nan(fmax_nan(fabsf(v.x), fabsf(v.y)), fmax_nan(fabsf(v.z), fabsf(v.w))));
      }
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (ok[u]) {
        const bool finite = m <= 3.402823466e38f;  // false for NaN and infinity
        bad |= !finite;
        const bool fast = m >= 0x1p-100f && m <= 0x1p100f;
        const float r = fast ? __frcp_rn(m) : 0.0f;
        uint16_t* dst = reinterpret_cast<uint16_t*>(codes + (b0 + i) * (B / 2)) + sl;
#pragma unroll
        for (int f = 0; f < F; ++f) {
          const float4 v = x[u][f];
          uint32_t c;
          if (m == 0.0f || !finite) {
            c = 0x7777u;  // an all-zero block encodes the zero level (a non-finite one is reported)
          } else if (fast) {
            c = nf4_code(div_by_absmax(v.x, m, r), s_cell) | (nf4_code(div_by_absmax(v.y, m, r), s_cell) << 4) |
                (nf4_code(div_by_absmax(v.z, m, r), s_cell) << 8) |
                (nf4_code(div_by_absmax(v.w, m, r), s_cell) << 12);
          } else {
            c = nf4_code(__fdiv_rn(v.x, m), s_cell) | (nf4_code(__fdiv_rn(v.y, m), s_cell) << 4) |
                (nf4_code(__fdiv_rn(v.z, m), s_cell) << 8) | (nf4_code(__fdiv_rn(v.w, m), s_cell) << 12);
          }
          dst[f * LP] = static_cast<uint16_t>(c);
        }
        if (sl == 0) {
          if (DQ)
            s_amax[i] = m;
          else
            dq_scale[b0 + i] = m;
        }
      }
    }
  }
  if (!DQ) {
    if (__syncthreads_or(bad) && tid == 0) atomicExch(nonfinite, 1);
    return;
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

// The same quantization for fp32 input in blocks of at most 64 weights, with
// the weights staged in shared memory: a persistent CTA takes groups
// blockIdx.x, + gridDim.x, ... and streams each as two halves of 128 blocks
// (32 KB for 64-weight blocks) by bulk copies into two buffers, so the copy of
// the next half is in flight while a half is coded.  Lanes read their float4s
// with 16-byte shared loads in an order rotated by block (f ^ (block & ROT))
// so that the eight lanes of a quarter-warp fall on distinct banks.  Every wait
// is bounded; on expiry the CTA lets its copies land and leaves.
template <int B, bool DQ>
__global__ void __launch_bounds__(256, 3) k_quantize_staged(const float* __restrict__ W, int64_t nblocks,
                                                         const Cell* __restrict__ cells, uint8_t* __restrict__ codes,
                                                         uint8_t* __restrict__ absmax_q, float* __restrict__ dq_scale,
                                                         int* nonfinite, int* status) {
  constexpr int F = 4;
  constexpr int LP = B / (4 * F);  // 2 or 4 lanes per block
  constexpr int BPW = 32 / LP;     // blocks per warp step
  constexpr int ROT = 8 / LP - 1;  // blocks of a quarter-warp: 8 / LP
  constexpr int HB = kGroup / 2;   // blocks per half-group (one buffer)
  constexpr int HV = HB * B / 4;   // float4s per buffer
  extern __shared__ __align__(128) float4 s_w[];  // two buffers of HV float4s
  __shared__ Cell s_cell[kCells];
  __shared__ float s_amax[kGroup];
  __shared__ float s_red[8];
  __shared__ __align__(8) uint64_t s_full[2];
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane / LP, sl = lane % LP;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  const int64_t nh = 2 * ((ngroups - blockIdx.x + gridDim.x - 1) / gridDim.x);  // this CTA's halves
  const uint32_t full0 = smem_u32(&s_full[0]), w0 = smem_u32(s_w);
  // first block and block count of the CTA's half h
  auto half = [&](int64_t h, int64_t& bstart) {
    bstart = (blockIdx.x + (h >> 1) * static_cast<int64_t>(gridDim.x)) * kGroup + (h & 1) * HB;
    const int64_t n = nblocks - bstart;
    return static_cast<int>(n < 0 ? 0 : n < HB ? n : HB);
  };
  auto issue = [&](int64_t h) {  // one thread
    int64_t bs;
    const uint32_t bytes = static_cast<uint32_t>(half(h, bs)) * B * 4, bar = full0 + 8u * (h & 1);
    mbar_arrive_expect_tx(bar, bytes);
    for (uint32_t off = 0; off < bytes; off += 16384u)
      bulk_g2s(w0 + (h & 1) * HV * 16 + off, reinterpret_cast<const uint8_t*>(W + bs * B) + off,
               min(16384u, bytes - off), bar);
  };
  if (tid == 0) {
    s_abort = 0;
    mbar_init(full0, 1);
    mbar_init(full0 + 8u, 1);
    fence_mbar_init();
    if (nh > 0) issue(0);
    if (nh > 1) issue(1);
  }
  s_cell[tid] = cells[tid];  // kCells == blockDim.x
  __syncthreads();
  bool bad = false;
  for (int64_t h = 0; h < nh; ++h) {
    const uint32_t bar = full0 + 8u * (h & 1), par = static_cast<uint32_t>(h >> 1) & 1u;
    if (!wait_bounded(bar, par, &s_abort, status)) {
      wait_drain(bar, par);  // let the copies in flight land before the CTA leaves
      if (h + 1 < nh) wait_drain(full0 + 8u * ((h + 1) & 1), static_cast<uint32_t>((h + 1) >> 1) & 1u);
      return;
    }
    int64_t bs;
    const int n = half(h, bs);
    const float4* buf = s_w + (h & 1) * HV;
    for (int p = warp; p * BPW < n; p += 8) {
      const int i = p * BPW + sub;
      const bool ok = i < n;
      float4 x[F];
#pragma unroll
      for (int f = 0; f < F; ++f)
        x[f] = ok ? buf[i * (B / 4) + (f ^ (sub & ROT)) * LP + sl] : make_float4(0.f, 0.f, 0.f, 0.f);
      float m = 0.0f;
#pragma unroll
      for (int f = 0; f < F; ++f)
        m = fmax_nan(m, fmax_nan(fmax_nan(fabsf(x[f].x), fabsf(x[f].y)), fmax_nan(fabsf(x[f].z), fabsf(x[f].w))));
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) m = fmax_nan(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (ok) {
        const bool finite = m <= 3.402823466e38f;  // false for NaN and infinity
        bad |= !finite;
        const bool fast = m >= 0x1p-100f && m <= 0x1p100f;
        const float r = fast ? __frcp_rn(m) : 0.0f;
        uint16_t* dst = reinterpret_cast<uint16_t*>(codes + (bs + i) * (B / 2)) + sl;
#pragma unroll
        for (int f = 0; f < F; ++f) {
          const float4 v = x[f];
          uint32_t c;
          if (m == 0.0f || !finite) {
            c = 0x7777u;  // an all-zero block encodes the zero level (a non-finite one is reported)
          } else if (fast) {
            c = nf4_code(div_by_absmax(v.x, m, r), s_cell) | (nf4_code(div_by_absmax(v.y, m, r), s_cell) << 4) |
                (nf4_code(div_by_absmax(v.z, m, r), s_cell) << 8) |
                (nf4_code(div_by_absmax(v.w, m, r), s_cell) << 12);
          } else {
            c = nf4_code(__fdiv_rn(v.x, m), s_cell) | (nf4_code(__fdiv_rn(v.y, m), s_cell) << 4) |
                (nf4_code(__fdiv_rn(v.z, m), s_cell) << 8) | (nf4_code(__fdiv_rn(v.w, m), s_cell) << 12);
          }
          dst[(f ^ (sub & ROT)) * LP] = static_cast<uint16_t>(c);
        }
        if (sl == 0) {
          if (DQ)
            s_amax[(h & 1) * HB + i] = m;
          else
            dq_scale[bs + i] = m;
        }
      }
    }
    __syncthreads();  // the buffer is read (and this half's maxima are in s_amax)
    if (tid == 0 && h + 2 < nh) issue(h + 2);
    if (DQ && (h & 1)) {  // the group is complete: double quantization of its absmax values
      const int64_t g = blockIdx.x + (h >> 1) * static_cast<int64_t>(gridDim.x);
      const int64_t gr = nblocks - g * kGroup;
      const int nbg = static_cast<int>(gr < kGroup ? gr : kGroup);
      float mg = (tid < nbg) ? s_amax[tid] : 0.0f;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mg = fmaxf(mg, __shfl_xor_sync(0xffffffffu, mg, off));
      if (lane == 0) s_red[warp] = mg;
      __syncthreads();
      float c2 = s_red[0];
#pragma unroll
      for (int w = 1; w < 8; ++w) c2 = fmaxf(c2, s_red[w]);
      const float s2 = (c2 > 0.0f) ? __fdiv_rn(c2, 255.0f) : 0.0f;
      if (tid < nbg) {
        uint8_t q = 0;
        if (s2 != 0.0f) q = static_cast<uint8_t>(fminf(255.0f, rintf(__fdiv_rn(s_amax[tid], s2))));
        absmax_q[g * kGroup + tid] = q;
      }
      if (tid == 0) dq_scale[g] = s2;
      __syncthreads();  // s_amax and s_red are free for the next group
    }
  }
  if (__syncthreads_or(bad) && tid == 0) atomicExch(nonfinite, 1);
}

// Merge into the default output format (blocks of 64 weights, double
// quantization over groups of 256 blocks) when K % 1024 == 0: a CTA owns
// MG_ROWS = 16 rows, which hold whole double-quantization groups (16 K / 64 is a
// multiple of 256), and walks them in chunks of MG_COLS = 256 columns.  Per
// chunk the adapter's A[:, chunk] is converted to fp32 in shared memory once
// and serves all 16 rows; B of the 16 rows sits there too, transposed, each
// value twice.  Two phases per chunk:
//  * a thread forms 4 rows x 4 columns of sum_j B[n, j] A[j, k] (j in order,
//    one FMA per exact product, as the general path; a warp covers 16 rows x
//    32 columns) and the merged values
//    fl32(w' + fl32(s * sum)), which go to shared memory (a byte of input codes
//    reads the two levels it selects with one 8-byte shared load);
//  * the 64 blocks of the chunk are coded with 4 threads per block and 16
//    weights per thread (k_quantize's layout: two shuffles and one reciprocal
//    per 16 weights).  Blocks sit 80 words apart in shared memory, so the
//    16-byte accesses of each quarter-warp fall on distinct banks in both
//    phases.
// The arithmetic runs on pairs where it can (the f32x2 FMA, multiply and add
// of sm_100 round each lane as the scalar instruction does).  The loads of the
// next chunk are in flight while a chunk is computed: its A slice by cp.async
// into a second bf16 staging buffer, its input codes and scales in registers.
// The exact block maxima wait in shared memory until the row range is done,
// then each group of 256 blocks is double-quantized as k_quantize does.  Same
// results, bit for bit, as the general path (the merge source of k_quantize).
constexpr int MG_ROWS = 16, MG_COLS = 256;

constexpr int MG_XP = 80;  // words from one block of merged values to the next

__host__ __device__ constexpr int merge64_smem_bytes(int r, int K) {
  return r * MG_COLS * 4 + 2 * r * MG_COLS * 2 + r * MG_ROWS * 8 + MG_ROWS * (MG_COLS / 64) * MG_XP * 4 +
         MG_ROWS * (K / 64) * 4;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Pairs of fp32 values in one 64-bit register (low half = first value).
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Both values rounded to bf16 and back to fp32.
__device__ __forceinline__ uint64_t bf16_round2(uint64_t v) {
  uint32_t h;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hi2(v)), "f"(lo2(v)));
  return pk2(__uint_as_float(h << 16), __uint_as_float(h & 0xffff0000u));
}

// Input codes (4 per row) and the input block scale of this thread's 4 rows
// in one chunk.  Offsets are relative to the CTA's first row (32-bit: a CTA
// covers 16 K <= 2^20 weights).
struct MergeIn {
  uint32_t c[4];
  float a[4];
};

struct MergeBase {
  const uint8_t* codes;     // input codes of the CTA's first row
  const uint8_t* absmax_q;  // input block scales (codes when dq) of that row
  const float* dq_scale;    // fp32 scales: per block, or per group of 256 blocks when dq
  int lg, dq;
  uint32_t bphase;          // dq: index of the first row's first block inside its group
};

__device__ __forceinline__ void merge_in_load(const MergeBase& mb, uint32_t e0, uint32_t K, int nrows, int rg,
                                              MergeIn& in) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    in.c[i] = 0;
    in.a[i] = 0.f;
    if (4 * rg + i < nrows) {
      const uint32_t e = e0 + static_cast<uint32_t>(4 * rg + i) * K;
      in.c[i] = __ldg(reinterpret_cast<const uint16_t*>(mb.codes + (e >> 1)));
      const uint32_t b = e >> mb.lg;
      in.a[i] = mb.dq ? __fmul_rn(static_cast<float>(__ldg(mb.absmax_q + b)), __ldg(mb.dq_scale + ((mb.bphase + b) >> 8)))
                      : __ldg(mb.dq_scale + b);
    }
  }
}

__global__ void __launch_bounds__(256, 4) k_merge64(MergeSrc m, Nf4Levels levels, int64_t N,
                                                    const Cell* __restrict__ cells, uint8_t* __restrict__ codes,
                                                    uint8_t* __restrict__ absmax_q, float* __restrict__ dq_scale,
                                                    int* nonfinite) {
  extern __shared__ __align__(16) float msm[];
  __shared__ Cell s_cell[kCells];
  __shared__ uint64_t s_lv2[256];  // byte of two codes -> {L[low nibble], L[high nibble]}
  __shared__ float s_red[8];
  const int K = static_cast<int>(m.K), KB = K / 64, r = m.r, nch = K / MG_COLS;
  float* As = msm;                                                      // [r][MG_COLS] fp32
  uint16_t* St = reinterpret_cast<uint16_t*>(As + r * MG_COLS);         // 2 x [r][MG_COLS] bf16 staging
  float* Bs = reinterpret_cast<float*>(St + 2 * r * MG_COLS);           // [r][MG_ROWS][2]
  float* Xs = Bs + r * MG_ROWS * 2;                                     // [MG_ROWS * 4 blocks][MG_XP] merged
  float* ab = Xs + MG_ROWS * (MG_COLS / 64) * MG_XP;                    // [MG_ROWS][KB] exact block maxima
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // columns 4 cg .. 4 cg + 3 of a chunk, rows 4 rg .. 4 rg + 3 (a warp covers 16 rows x 32 columns)
  const int cg = warp * 8 + (lane & 7), rg = lane >> 3;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * MG_ROWS;
  const int nrows = static_cast<int>(N - n0 < MG_ROWS ? N - n0 : MG_ROWS);
  const int a16 = r * MG_COLS / 8;  // 16-byte pieces of one chunk of A

  auto stage = [&](int c) {  // A[:, chunk c] -> staging buffer c & 1
    uint16_t* dst = St + (c & 1) * r * MG_COLS;
    for (int i = tid; i < a16; i += 256) {
      const int j = i / (MG_COLS / 8), k8 = i - j * (MG_COLS / 8);
      cp_async16(dst + j * MG_COLS + k8 * 8, m.A + static_cast<int64_t>(j) * K + c * MG_COLS + k8 * 8);
    }
    cp_async_commit();
  };
  stage(0);
  s_cell[tid] = cells[tid];  // kCells == blockDim.x
  s_lv2[tid] = pk2(levels.v[tid & 15], levels.v[tid >> 4]);
  for (int i = tid; i < r * MG_ROWS; i += 256) {
    const int j = i / MG_ROWS, row = i - j * MG_ROWS;
    const float b = row < nrows ? bf16_bits_to_f32(m.B[(n0 + row) * r + j]) : 0.f;
    Bs[2 * i] = b;
    Bs[2 * i + 1] = b;
  }
  const uint64_t s_2 = pk2(m.s, m.s);
  const uint64_t k64 = pk2(64.0f, 64.0f), kbias = pk2(12582976.0f, 12582976.0f);
  const int64_t e_cta = n0 * K;  // first weight of the CTA (a multiple of 16384)
  const int64_t b_cta = e_cta >> m.lg;  // its input block
  const MergeBase mb{m.codes + e_cta / 2, m.dq ? m.absmax_q + b_cta : nullptr,
                     m.dq_scale + (m.dq ? b_cta >> 8 : b_cta), m.lg, m.dq, static_cast<uint32_t>(b_cta & 255)};
  uint8_t* const codes_cta = codes + e_cta / 2;
  MergeIn cur, nxt;
  merge_in_load(mb, 4 * cg, K, nrows, rg, cur);
  bool bad = false;
  for (int c = 0; c < nch; ++c) {
    cp_async_wait_all();
    __syncthreads();  // chunk c staged by all threads; everyone is done with As of chunk c - 1
    {
      const uint16_t* src = St + (c & 1) * r * MG_COLS;
      for (int i = tid; i < a16; i += 256) {
        const uint4 a = *reinterpret_cast<const uint4*>(src + i * 8);
        float4* dst = reinterpret_cast<float4*>(As + i * 8);
        dst[0] = make_float4(__uint_as_float(a.x << 16), __uint_as_float(a.x & 0xffff0000u),
                             __uint_as_float(a.y << 16), __uint_as_float(a.y & 0xffff0000u));
        dst[1] = make_float4(__uint_as_float(a.z << 16), __uint_as_float(a.z & 0xffff0000u),
                             __uint_as_float(a.w << 16), __uint_as_float(a.w & 0xffff0000u));
      }
    }
    if (c + 1 < nch) {
      stage(c + 1);  // buffer (c + 1) & 1 was last read before the barrier above
      merge_in_load(mb, (c + 1) * MG_COLS + 4 * cg, K, nrows, rg, nxt);
    }
    __syncthreads();  // As holds chunk c
    uint64_t acc[4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0;
#pragma unroll 4
    for (int j = 0; j < r; ++j) {
      const ulonglong2 a4 = *reinterpret_cast<const ulonglong2*>(As + j * MG_COLS + 4 * cg);
      const ulonglong2 b01 = *reinterpret_cast<const ulonglong2*>(Bs + (j * MG_ROWS + 4 * rg) * 2);
      const ulonglong2 b23 = *reinterpret_cast<const ulonglong2*>(Bs + (j * MG_ROWS + 4 * rg) * 2 + 4);
      acc[0][0] = fma2(b01.x, a4.x, acc[0][0]);
      acc[0][1] = fma2(b01.x, a4.y, acc[0][1]);
      acc[1][0] = fma2(b01.y, a4.x, acc[1][0]);
      acc[1][1] = fma2(b01.y, a4.y, acc[1][1]);
      acc[2][0] = fma2(b23.x, a4.x, acc[2][0]);
      acc[2][1] = fma2(b23.x, a4.y, acc[2][1]);
      acc[3][0] = fma2(b23.y, a4.x, acc[3][0]);
      acc[3][1] = fma2(b23.y, a4.y, acc[3][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {  // merged values of row 4 rg + i -> Xs
      const uint64_t a2 = pk2(cur.a[i], cur.a[i]);
      const uint64_t w01 = bf16_round2(mul2(s_lv2[cur.c[i] & 255u], a2));
      const uint64_t w23 = bf16_round2(mul2(s_lv2[cur.c[i] >> 8], a2));
      ulonglong2 x;
      x.x = add2(w01, mul2(s_2, acc[i][0]));
      x.y = add2(w23, mul2(s_2, acc[i][1]));
      *reinterpret_cast<ulonglong2*>(Xs + ((4 * rg + i) * 4 + (cg >> 4)) * MG_XP + (cg & 15) * 4) = x;
    }
    __syncthreads();  // Xs holds the chunk's merged values
    {
      const int bid = tid >> 2, sl = tid & 3;  // block bid of the chunk: row bid / 4, column block bid % 4
      const int row = bid >> 2;
      const float* xb = Xs + bid * MG_XP;
      ulonglong2 v[4];
#pragma unroll
      for (int f = 0; f < 4; ++f) v[f] = *reinterpret_cast<const ulonglong2*>(xb + (f * 4 + sl) * 4);
      float mx = 0.0f;
#pragma unroll
      for (int f = 0; f < 4; ++f)
        mx = fmax_nan(mx, fmax_nan(fmax_nan(fabsf(lo2(v[f].x)), fabsf(hi2(v[f].x))),
                                   fmax_nan(fabsf(lo2(v[f].y)), fabsf(hi2(v[f].y)))));
      mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmax_nan(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (row < nrows) {
        uint16_t* dst = reinterpret_cast<uint16_t*>(codes_cta + ((static_cast<uint32_t>(row) * K + c * MG_COLS) >> 1) +
                                                    (bid & 3) * 32) + sl;
        if (__builtin_expect(mx >= 0x1p-100f && mx <= 0x1p100f, 1)) {
          // div_by_absmax on pairs: q0 = x r, e = fma(q0, -a, x) (= fma(-q0, a, x)), t = fma(e, r, q0)
          const float rr = __frcp_rn(mx);
          const uint64_t r2 = pk2(rr, rr), na2 = pk2(-mx, -mx);
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const uint64_t q01 = mul2(v[f].x, r2), q23 = mul2(v[f].y, r2);
            const uint64_t t01 = fma2(fma2(q01, na2, v[f].x), r2, q01);
            const uint64_t t23 = fma2(fma2(q23, na2, v[f].y), r2, q23);
            const uint64_t f01 = fma2(t01, k64, kbias), f23 = fma2(t23, k64, kbias);
            const float t[4] = {lo2(t01), hi2(t01), lo2(t23), hi2(t23)};
            const float g[4] = {lo2(f01), hi2(f01), lo2(f23), hi2(f23)};
            uint32_t code = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const Cell cl = s_cell[__float_as_uint(g[q]) & (kCells - 1)];
              code |= static_cast<uint32_t>(cl.base + (t[q] > cl.mid ? 1 : 0)) << (4 * q);
            }
            dst[f * 4] = static_cast<uint16_t>(code);
          }
        } else {
          const bool finite = mx <= 3.402823466e38f;  // false for NaN and infinity
          bad |= !finite;
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const float x[4] = {lo2(v[f].x), hi2(v[f].x), lo2(v[f].y), hi2(v[f].y)};
            uint32_t code = 0x7777u;
            if (mx != 0.0f && finite)
              code = nf4_code(__fdiv_rn(x[0], mx), s_cell) | (nf4_code(__fdiv_rn(x[1], mx), s_cell) << 4) |
                     (nf4_code(__fdiv_rn(x[2], mx), s_cell) << 8) | (nf4_code(__fdiv_rn(x[3], mx), s_cell) << 12);
            dst[f * 4] = static_cast<uint16_t>(code);
          }
        }
        if (sl == 0) ab[row * KB + c * (MG_COLS / 64) + (bid & 3)] = mx;
      }
    }
    cur = nxt;
  }
  __syncthreads();
  // double quantization of the row range's groups (256 consecutive blocks each)
  const int nb = nrows * KB;
  for (int g0 = 0; g0 < nb; g0 += kGroup) {
    const int i = g0 + tid;
    const float v = i < nb ? ab[i] : 0.0f;
    float mv = v;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mv = fmaxf(mv, __shfl_xor_sync(0xffffffffu, mv, off));
    if (lane == 0) s_red[warp] = mv;
    __syncthreads();
    float c2 = s_red[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) c2 = fmaxf(c2, s_red[w]);
    const float s2 = (c2 > 0.0f) ? __fdiv_rn(c2, 255.0f) : 0.0f;
    if (i < nb) {
      uint8_t q = 0;
      if (s2 != 0.0f) q = static_cast<uint8_t>(fminf(255.0f, rintf(__fdiv_rn(v, s2))));
      absmax_q[n0 * KB + i] = q;
    }
    if (tid == 0) dq_scale[(n0 * KB + g0) / kGroup] = s2;
    __syncthreads();  // s_red is reused by the next group
  }
  if (__syncthreads_or(bad) && tid == 0) atomicExch(nonfinite, 1);
}

// One thread expands 64 consecutive weights (one register table per block
// of B weights it touches: two for B = 32, one otherwise; 32 code bytes in,
// 128 bytes of bf16 out); a warp's 32 x 64 weights pass through shared memory
// (16-byte chunks XOR-swizzled by lane) so that the global stores are 512
// contiguous bytes per instruction.  DQ: block scale = absmax_q * dq_scale of
// its group; else the stored fp32 absmax.
template <int B, bool DQ>
__global__ void __launch_bounds__(256) k_dequantize(const uint8_t* __restrict__ codes,
                                                    const uint8_t* __restrict__ absmax_q,
                                                    const float* __restrict__ dq_scale, int64_t nchunks64,
                                                    Nf4Levels L, uint16_t* __restrict__ out) {
  __shared__ uint4 s_out[8][32 * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t wc0 = (static_cast<int64_t>(blockIdx.x) * 8 + warp) * 32;  // first 64-weight chunk of this warp
  const int64_t c = wc0 + lane;
  if (wc0 >= nchunks64) return;  // warp-uniform
  auto scale = [&](int64_t b) -> float {
    return DQ ? __fmul_rn(static_cast<float>(absmax_q[b]), dq_scale[b / kGroup]) : dq_scale[b];
  };
  if (c < nchunks64) {
    const uint4 c0 = ldg_nc_v4(codes + c * 32);
    const uint4 c1 = ldg_nc_v4(codes + c * 32 + 16);
    const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    if (B == 32) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const Nf4Lut t = make_lut(L, scale(2 * c + h));
#pragma unroll
        for (int i = 4 * h; i < 4 * h + 4; ++i) {
          uint4 o;
          deq8(w[i], t, o.x, o.y, o.z, o.w);
          s_out[warp][lane * 8 + (i ^ (lane & 7))] = o;
        }
      }
    } else {
      const Nf4Lut t = make_lut(L, scale(c * 64 / B));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint4 o;
        deq8(w[i], t, o.x, o.y, o.z, o.w);
        s_out[warp][lane * 8 + (i ^ (lane & 7))] = o;
      }
    }
  }
  __syncwarp();
  const int64_t nout = (nchunks64 - wc0 < 32 ? nchunks64 - wc0 : 32) * 8;
  uint4* dst = reinterpret_cast<uint4*>(out + wc0 * 64);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = i * 32 + lane;  // 16-byte chunk q of the warp's 32 x 128 bytes
    if (q < nout) __stcs(dst + q, s_out[warp][(q >> 3) * 8 + ((q & 7) ^ ((q >> 3) & 7))]);
  }
}

template <int B, bool DQ>
cudaError_t quantize_launch(const float* W, const MergeSrc* merge, int64_t numel, uint8_t* codes,
                            uint8_t* absmax_q, float* dq_scale, int* nonfinite, cudaStream_t st) {
  const int64_t nblocks = numel / B;
  const int64_t ngroups = (nblocks + kGroup - 1) / kGroup;
  if (ngroups == 0) return cudaSuccess;
  const HostCodebook& cb = host_codebook();
  cudaError_t e;
  const Cell* cells = device_cells(&e);
  if (!cells) return e;
  if (merge) {
    k_quantize<B, DQ, true><<<static_cast<unsigned>(ngroups), 256, 0, st>>>(
        nullptr, *merge, cb.levels, nblocks, cells, codes, absmax_q, dq_scale, nonfinite);
  } else if (B <= 64) {  // staged: two 128-block buffers, three CTAs per SM, each looping over groups
    constexpr int smem = kGroup * (B <= 64 ? B : 64) * 4;
    e = smem_limit_once<k_quantize_staged<B <= 64 ? B : 64, DQ>>(smem);
    if (e != cudaSuccess) return e;
    const int64_t grid = std::min<int64_t>(ngroups, 3 * static_cast<int64_t>(device_sm_count()));
    k_quantize_staged<B <= 64 ? B : 64, DQ><<<static_cast<unsigned>(grid), 256, smem, st>>>(
        W, nblocks, cells, codes, absmax_q, dq_scale, nonfinite, device_status_ptr());
  } else {
    k_quantize<B, DQ, false><<<static_cast<unsigned>(ngroups), 256, 0, st>>>(
        W, MergeSrc{}, cb.levels, nblocks, cells, codes, absmax_q, dq_scale, nonfinite);
  }
  return cudaGetLastError();
}

template <int B, bool DQ>
cudaError_t dequantize_launch(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t numel,
                              uint16_t* out, cudaStream_t st) {
  const int64_t nchunks = numel / 64;
  if (nchunks == 0) return cudaSuccess;
  const unsigned grid = static_cast<unsigned>((nchunks + 255) / 256);  // 8 warps x 32 chunks per CTA
  k_dequantize<B, DQ><<<grid, 256, 0, st>>>(codes, absmax_q, dq_scale, nchunks, host_codebook().levels, out);
  return cudaGetLastError();
}

}  // namespace

// Formats: block in {32, 64, 128, 256}; dq_block 256 (double quantization) or
// 0 (none).  The caller has validated them.
#define QN_CODEC_DISPATCH(FN, ...)                                                  \
  switch (block * 2 + (dq_block ? 1 : 0)) {                                        \
    case 64 * 2 + 1: return FN<64, true>(__VA_ARGS__);                              \
    case 64 * 2: return FN<64, false>(__VA_ARGS__);                                 \
    case 32 * 2 + 1: return FN<32, true>(__VA_ARGS__);                              \
    case 32 * 2: return FN<32, false>(__VA_ARGS__);                                 \
    case 128 * 2 + 1: return FN<128, true>(__VA_ARGS__);                            \
    case 128 * 2: return FN<128, false>(__VA_ARGS__);                               \
    case 256 * 2 + 1: return FN<256, true>(__VA_ARGS__);                            \
    case 256 * 2: return FN<256, false>(__VA_ARGS__);                               \
    default: return cudaErrorInvalidValue;                                         \
  }

cudaError_t launch_quantize(const float* W, int64_t numel, int block, int dq_block, uint8_t* codes,
                            uint8_t* absmax_q, float* dq_scale, int* nonfinite, cudaStream_t st) {
  QN_CODEC_DISPATCH(quantize_launch, W, nullptr, numel, codes, absmax_q, dq_scale, nonfinite, st)
}

cudaError_t launch_merge_quantize(const uint8_t* codes_in, const uint8_t* absmax_in, const float* dq_in, int block_in,
                                  int dq_block_in, int64_t N, int64_t K, const uint16_t* A, const uint16_t* Bl, int r,
                                  float scale, int block, int dq_block, uint8_t* codes, uint8_t* absmax_q,
                                  float* dq_scale, int* nonfinite, cudaStream_t st) {
  int lg = 0;
  while ((1 << lg) < block_in) ++lg;
  const MergeSrc m{codes_in, absmax_in, dq_in, lg, dq_block_in ? 1 : 0, A, Bl, r, scale, K};
  if (block == 64 && dq_block == 256 && K % 1024 == 0 && K <= 65536) {  // the tiled path (default output format)
    cudaError_t e;
    const Cell* cells = device_cells(&e);
    if (!cells) return e;
    const int smem = merge64_smem_bytes(r, static_cast<int>(K));
    e = cudaFuncSetAttribute(k_merge64, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>((N + MG_ROWS - 1) / MG_ROWS);
    k_merge64<<<grid, 256, smem, st>>>(m, host_codebook().levels, N, cells, codes, absmax_q, dq_scale, nonfinite);
    return cudaGetLastError();
  }
  const MergeSrc* mp = &m;
  const int64_t numel = N * K;
  const float* W = nullptr;
  QN_CODEC_DISPATCH(quantize_launch, W, mp, numel, codes, absmax_q, dq_scale, nonfinite, st)
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t numel,
                              int block, int dq_block, uint16_t* out, cudaStream_t st) {
  QN_CODEC_DISPATCH(dequantize_launch, codes, absmax_q, dq_scale, numel, out, st)
}

#undef QN_CODEC_DISPATCH

}  // namespace qn
