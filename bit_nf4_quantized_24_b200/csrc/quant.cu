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
  if (merge)
    k_quantize<B, DQ, true><<<static_cast<unsigned>(ngroups), 256, 0, st>>>(
        nullptr, *merge, cb.levels, nblocks, cells, codes, absmax_q, dq_scale, nonfinite);
  else
    k_quantize<B, DQ, false><<<static_cast<unsigned>(ngroups), 256, 0, st>>>(
        W, MergeSrc{}, cb.levels, nblocks, cells, codes, absmax_q, dq_scale, nonfinite);
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
