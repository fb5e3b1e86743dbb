// Launchers shared between the translation units of libqlora_nf4.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "common.cuh"

namespace qn {

// 2D row-major TMA tensor map: `inner` elements per row, `outer` rows, row
// pitch `pitch_bytes`, box {box_inner, box_outer}; out-of-range elements read
// as zero.  Returns false if the driver rejects the description.
bool make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
              uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz);

// Host-side NF4 table (computed once by codebook.cu).
struct HostCodebook {
  Nf4Levels levels;
  Nf4Mids mids;
};
const HostCodebook& host_codebook();

// Status of a CUDA runtime result for the C ABI: QLORA_OK, or QLORA_ERR_CUDA
// after recording the error for qlora_last_cuda_error() on this host thread.
int cuda_status(cudaError_t e);
// Shape rules of the layer entry points (M, N, K, r; QLORA_OK or the status
// to return) and the NF4 formats the layer reads (block in {32, 64, 128, 256},
// dq_block 256 or 0, K % block == 0).
int check_layer_shapes(int64_t M, int64_t N, int64_t K, int r);
int check_format(int64_t K, int block, int dq_block);

// Per-device status word (timeouts of bounded waits) and the non-finite
// flag of nf4_quantize; both live in file-scope device memory.
int* device_status_ptr();      // device address of the status word
int* device_nonfinite_ptr();   // device address of the non-finite flag

// ----- quantize / dequantize (HBM-bound)
// block in {32, 64, 128, 256}; dq_block 256 or 0 (no double quantization:
// dq_scale then holds each block's fp32 absmax and absmax_q is unused).
cudaError_t launch_quantize(const float* W, int64_t numel, int block, int dq_block, uint8_t* codes,
                            uint8_t* absmax_q, float* dq_scale, int* nonfinite, cudaStream_t st);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                              int64_t numel, int block, int dq_block, uint16_t* out, cudaStream_t st);
// Quantize (into block / dq_block) the merge of an NF4 weight (block_in /
// dq_block_in) with the adapter: fl32(w' + fl32(scale * sum_j B[n,j] A[j,k])).
cudaError_t launch_merge_quantize(const uint8_t* codes_in, const uint8_t* absmax_in, const float* dq_in, int block_in,
                                  int dq_block_in, int64_t N, int64_t K, const uint16_t* A, const uint16_t* Bl, int r,
                                  float scale, int block, int dq_block, uint8_t* codes, uint8_t* absmax_q,
                                  float* dq_scale, int* nonfinite, cudaStream_t st);

// ----- fused dequant-GEMM on tcgen05 (tensor cores)
// mode 0 (forward):  Y[M,N]  = X[M,K]  deq(W)^T + Ht[M,r] Bt^T, Bt = lora_B [N,r]
// mode 1 (dX):       dX[M,K] = dY[M,N] deq(W)   + Ht[M,r] A,   A  = lora_A [r,K]
// Ht is the bf16 tail operand (s*H for the forward, dH for dX).
struct GemmArgs {
  int mode;
  const uint16_t* act;     // X or dY, bf16 [M, Kc]
  const uint16_t* tail_a;  // bf16 [M, r]
  const uint16_t* tail_b;  // lora_B [N, r] (mode 0) or lora_A [r, K] (mode 1)
  const uint8_t* codes;
  const uint8_t* absmax_q;
  const float* dq_scale;
  int64_t M, N, K;
  int r;
  uint16_t* out;  // Y [M, N] or dX [M, K]
  bool pdl;       // launched right after another kernel of the layer (programmatic dependent launch)
  int block = 64;       // NF4 format: weights per block (32, 64, 128, 256)
  int dq_block = 256;   // 256: double quantization; 0: fp32 absmax per block in dq_scale
  float* part = nullptr;  // room for the split tiles' fp32 partial sums (nullable: no split)
  size_t part_bytes = 0;
};
cudaError_t launch_nf4_gemm(const GemmArgs& a, cudaStream_t st);
// How a launch of the fused GEMM divides its tiles on the current device: the
// tiles that would form a partial last wave on the resident CTA pairs are
// split along K into nsplit pieces each (fp32 partial sums, part_bytes of
// them, summed in piece order by a second kernel).  nsplit = 1: no split.
struct SplitPlan {
  int64_t npairs = 0, nout_tiles = 0, nwhole = 0, ntail = 0;
  int nsplit = 1;
  size_t part_bytes = 0;
};
SplitPlan gemm_split_plan(int mode, int64_t M, int64_t N, int64_t K);
// CTA pairs of the fused GEMM that fit on the current device at once
// (negative: the occupancy query failed).
int nf4_gemm_max_active_pairs(int mode);

// ----- adapter kernels
// out[m, j] = sum_k P[m,k] Q[j,k]  (P bf16 [M, Kc], Q bf16 [R, Kc]); writes
// out16a = bf16(sa * acc) [M,R], out16b = bf16(sb * acc) (nullable),
// out32 = sb * acc fp32 (nullable).  M <= 16 runs a split-contraction kernel
// that allows the next kernel of the stream an early (programmatic) launch.
cudaError_t launch_rowdot(const uint16_t* P, const uint16_t* Q, int64_t M, int64_t Kc, int R, float sa,
                          uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st,
                          bool pdl = false);
// out[j, c] = sum_m G[m, j] P[m, c] over all m (G bf16 [M, R], P bf16 [M, C]),
// written as bf16(scale * out) either [R, C] (transpose = 0) or [C, R]
// (transpose = 1).  One kernel; the token splits meet in a thread-block
// cluster, so no scratch is needed.
cudaError_t launch_coldot(const uint16_t* G, const uint16_t* P, int64_t M, int64_t C, int R, float scale,
                          int transpose, uint16_t* out, cudaStream_t st, bool pdl = false);
// The same with Q given transposed, Qt bf16 [Kc, R] (lora_B read in place).
cudaError_t launch_rowdot_qt(const uint16_t* P, const uint16_t* Qt, int64_t M, int64_t Kc, int R, float sa,
                             uint16_t* out16a, float sb, uint16_t* out16b, float* out32, cudaStream_t st,
                             bool pdl = false);

// ----- decode GEMV (M <= 16): Y = X deq(W)^T + Hs B^T, Hs = bf16(s X A^T)
// withhold_one_stage: the testing aid of qlora_test_decode_timeout (a 1 ms
// wait limit and one code stage never copied, so a bounded wait runs out).
// block in {64, 128, 256} (a 64-weight block lies in one scale block), dq_block
// 256 or 0 (the fp32 absmax of each block in dq_scale).
cudaError_t launch_gemv(const uint16_t* X, int64_t M, const uint8_t* codes, const uint8_t* absmax_q,
                        const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B, int r,
                        uint16_t* Y, cudaStream_t st, const int32_t* aidx = nullptr, int na = 0,
                        bool withhold_one_stage = false, int block = 64, int dq_block = 256);
// Decode tiles (see gemv.cu): bytes of the tiled copy of an N x K weight's
// codes, the repacking kernel (K % 1024 == 0), and the decode forward that
// reads them (M <= 16, default format).
int64_t decode_tiles_bytes(int64_t N, int64_t K);
cudaError_t launch_pack_tiles(const uint8_t* codes, int64_t N, int64_t K, uint8_t* tiles, cudaStream_t st);
cudaError_t launch_gemv_tiles(const uint16_t* X, int64_t M, const uint8_t* tiles, const uint8_t* absmax_q,
                              const float* dq_scale, int64_t N, int64_t K, const uint16_t* Hs, const uint16_t* B,
                              int r, uint16_t* Y, cudaStream_t st, const int32_t* aidx = nullptr, int na = 0,
                              int block = 64, int dq_block = 256);
// LoRA dropout: Xd = mask ? bf16(fl32(X * keep)) : 0 over n elements (n % 8 == 0,
// 16-byte aligned); dX += mask * keep * (dH A) (see adapter.cu).
// The adapter products on Xd = mask ? bf16(fl32(X keep)) : 0 without Xd in
// memory: the kernels apply the mask to their X tiles in shared memory.
// launch_rowdot_masked: out = sa/sb * Xd Q^T (Q [R, Kc]), M > 16 only.
// launch_coldot_masked: out[j, c] = bf16(scale * sum_m G[m, j] Xd[m, c]).
cudaError_t launch_rowdot_masked(const uint16_t* X, const uint8_t* mask, float keep, const uint16_t* Q, int64_t M,
                                 int64_t Kc, int R, float sa, uint16_t* out16a, float sb, uint16_t* out16b,
                                 cudaStream_t st, bool pdl);
cudaError_t launch_coldot_masked(const uint16_t* G, const uint16_t* X, const uint8_t* mask, float keep, int64_t M,
                                 int64_t C, int R, float scale, uint16_t* out, cudaStream_t st, bool pdl);
cudaError_t launch_dropout_input(const uint16_t* X, const uint8_t* mask, float keep, int64_t n, uint16_t* Xd,
                                 cudaStream_t st, bool pdl);
cudaError_t launch_dx_add_masked(uint16_t* dX, const uint16_t* dH, const uint16_t* A, const uint8_t* mask, float keep,
                                 int64_t M, int64_t K, int r, cudaStream_t st, bool pdl);
// Multi-adapter Hs for the decode kernel: Hs[m, j] = bf16(scales[a] *
// sum_k X[m, k] A_all[a, j, k]) with a = aidx[m] (0 when a is outside [0, na)).
cudaError_t launch_rows_multi(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A_all, int na, int r,
                              const float* scales, const int32_t* aidx, uint16_t* Hs, cudaStream_t st);

// ----- per-device launch setup, done once per device and kernel

// Raises the dynamic shared-memory limit of kernel KERN to `bytes` on the
// current device the first time it is asked for that device.
template <auto KERN>
cudaError_t smem_limit_once(int bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(KERN, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_release);
  return e;
}
// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();

// Launches `kern` on `st`; with pdl the launch may begin while the previous
// kernel of the stream is still running (the kernel synchronises with
// pdl_wait, see common.cuh).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ----- tracing of the fused GEMM launches
void trace_before(cudaStream_t st);
void trace_after(cudaStream_t st);

}  // namespace qn
