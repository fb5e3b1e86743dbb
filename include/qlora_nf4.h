/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA frozen-NF4 linear layer.
 *
 * The operations follow the QLoRA pages (cited by title and section):
 *  - "What does QLoRA change compared with plain LoRA when fine-tuning Llama?"
 *    (katajob): "NF4: 4-bit NormalFloat" (16-level type for normally
 *    distributed weights; per-block scaling over small groups of contiguous
 *    weights, 64 being the usual size; expanded block by block to bf16 for
 *    the matmul only), "Double quantization" (the per-block scales are
 *    themselves quantized to 8 bits with a second-level scale over groups),
 *    "What stays in full precision" (A, B are bf16; gradients reach them
 *    through the dequantized base; the base gets no update).
 *  - "QLoRA: fine-tuning a large model on one GPU" (pranaymahendrakar),
 *    "LoRA, stated once": h = W0 x + (alpha/r) B A x with B in R^{d x r},
 *    A in R^{r x k}.
 *  - "QLoRA and Quantized Fine-Tuning" (quantmemo), "The two mechanisms
 *    combined": W' = W_4bit + BA, only B and A are trained.
 *
 * Conventions shared by every entry point
 *  - Types: bf16 tensors are passed as raw bit patterns (qlora_bf16_t =
 *    uint16_t); fp32 as float; NF4 codes, absmax codes as uint8_t.
 *  - Layout: every matrix is row-major and contiguous.  Weights are [N, K]
 *    (out_features x in_features, the nn.Linear layout); X is [M, K];
 *    Y and dY are [M, N]; LoRA A is [r, K] and B is [N, r].
 *  - NF4 format (produced by nf4_quantize, consumed by everything else):
 *      codes     uint8 [N*K/2]   element 2j in the low nibble of byte j,
 *                                element 2j+1 in the high nibble; the code is
 *                                the index (0..15) of the ascending level.
 *      absmax_q  uint8 [N*K/block]      8-bit code of each block's absmax.
 *      dq_scale  fp32  [ceil(N*K/block/dq_block)]  second-level scale of each
 *                                group of dq_block consecutive blocks.
 *    Blocks are `block` consecutive elements of the flattened weight (they
 *    never straddle a row: K % block == 0).  The codec entry points
 *    (nf4_quantized_sizes, nf4_quantize, nf4_dequantize) accept block in
 *    {32, 64, 128, 256} and dq_block 256 or 0.  dq_block == 0 turns double
 *    quantization off: absmax_q is then empty (NULL allowed) and dq_scale holds
 *    the exact fp32 absmax of every block ([N*K/block]).  The layer entry
 *    points (qlora_linear_*) read the default format, block 64 with
 *    dq_block 256.  Other values: QLORA_ERR_UNSUPPORTED.
 *  - Pointers: every tensor pointer is a DEVICE pointer of the current CUDA
 *    device unless stated otherwise; the caller owns all memory.  The library
 *    never frees or retains caller memory.
 *  - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *    device work is enqueued asynchronously on it; argument errors are
 *    returned synchronously before anything is enqueued.
 *  - Status: every function returns QLORA_OK (0) or a negative QLORA_ERR_*.
 *    A launch failure returns QLORA_ERR_CUDA (the CUDA error is readable via
 *    qlora_last_cuda_error()).
 *  - Device-side waits inside the tensor-core kernels are bounded; a wait
 *    that runs out records QLORA_ERR_TIMEOUT in a device status word that
 *    qlora_device_status() reads (it synchronizes the device).
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t qlora_bf16_t;

#define QLORA_OK 0
#define QLORA_ERR_ARG (-1)         /* null pointer, negative size, bad r or scale */
#define QLORA_ERR_SHAPE (-2)       /* K % block != 0, misaligned sizes */
#define QLORA_ERR_NONFINITE (-3)   /* the weight holds a NaN or an infinity */
#define QLORA_ERR_WORKSPACE (-4)   /* workspace null or smaller than required */
#define QLORA_ERR_CUDA (-5)        /* a CUDA runtime call or launch failed */
#define QLORA_ERR_TIMEOUT (-6)     /* a bounded device-side wait ran out */
#define QLORA_ERR_UNSUPPORTED (-7) /* block/dq_block/r outside this build's set */

/* Human-readable name of a status code (static string, never NULL). */
const char* qlora_status_string(int status);

/* Last CUDA error code seen by the library on this host thread (0 if none). */
int qlora_last_cuda_error(void);

/* ABI version: (major << 16) | minor. */
int qlora_version(void);

/* Byte sizes of the three NF4 buffers of an [N, K] weight.
 * Errors: QLORA_ERR_ARG (negative sizes, null outputs),
 * QLORA_ERR_SHAPE (K % block != 0), QLORA_ERR_UNSUPPORTED. */
int nf4_quantized_sizes(int64_t N, int64_t K, int block, int dq_block,
                        size_t* codes_bytes, size_t* absmax_bytes, size_t* dq_scale_bytes);

/* The 16 NF4 levels (fp32, ascending, HOST memory) this library encodes with.
 * They are equal-probability quantiles of the standard normal on each side of
 * an exact zero (8 positive, 7 negative), scaled to [-1, 1] (katajob,
 * "NF4: 4-bit NormalFloat": levels optimal for a zero-centred normal).
 * levels_out: host pointer to 16 floats.  Errors: QLORA_ERR_ARG. */
int nf4_codebook(float* levels_out);

/* Quantize an fp32 weight [N, K] to NF4 with double quantization (katajob,
 * "NF4: 4-bit NormalFloat" and "Double quantization").  Per block b:
 * a_b = max |w|; code = index of the nearest level to fl32(w / a_b) (ties at
 * a midpoint take the lower code; an all-zero block encodes the zero level).
 * Per group g of dq_block blocks: s2_g = fl32(max_b a_b / 255);
 * absmax_q[b] = min(255, round_half_even(fl32(a_b / s2_g))) (0 if s2_g == 0);
 * with dq_block == 0, dq_scale[b] = a_b instead.
 * W: device fp32 [N, K]; codes, absmax_q, dq_scale: device outputs sized by
 * nf4_quantized_sizes.  Synchronizes `stream` to report non-finite input:
 * returns QLORA_ERR_NONFINITE if W holds a NaN or an infinity (the outputs are
 * then unspecified).  Calls on different streams or host threads run
 * independently (each takes its own non-finite flag from a per-device pool of
 * 64; a 65th concurrent call waits for a flag to come free).
 * Other errors: ARG, SHAPE, UNSUPPORTED, CUDA. */
int nf4_quantize(const float* W, int64_t N, int64_t K, int block, int dq_block,
                 uint8_t* codes, uint8_t* absmax_q, float* dq_scale, void* stream);

/* Dequantize NF4 to bf16 (katajob, "NF4: 4-bit NormalFloat": the block is
 * expanded to the compute dtype).  w' = bf16_rne(fl32(level[code] * a')) with
 * a' = fl32(absmax_q[b] * dq_scale[g]) (or a' = dq_scale[b] when dq_block is
 * 0).  W_out: device bf16 [N, K].
 * Errors: ARG, SHAPE, UNSUPPORTED, CUDA. */
int nf4_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                   int64_t N, int64_t K, int block, int dq_block,
                   qlora_bf16_t* W_out, void* stream);

/* Merge the trained adapter into the frozen weight and store the sum as NF4
 * again ("QLoRA and Quantized Fine-Tuning", "The two mechanisms combined": the
 * merged model computes with W' + BA):
 *     merged[n, k] = fl32(w'[n, k] + fl32(scale * sum_j B[n, j] A[j, k]))
 * where w' is the bf16 weight the layer dequantizes (format block / dq_block)
 * and the sum runs in fp32 in the order j = 0 .. r-1 (each product of two
 * bf16 values is exact in fp32); merged is then quantized exactly as
 * nf4_quantize does, into the format out_block / out_dq_block.
 * codes, absmax_q, dq_scale: the input weight (device); A: bf16 [r, K];
 * B: bf16 [N, r]; 1 <= r <= 64; out_*: device outputs sized by
 * nf4_quantized_sizes(N, K, out_block, out_dq_block).  The input is only read,
 * so the outputs must not alias it.  Synchronizes `stream` like nf4_quantize
 * and returns QLORA_ERR_NONFINITE if a merged value is not finite.
 * Errors: ARG, SHAPE, UNSUPPORTED, NONFINITE, CUDA. */
int nf4_merge_lora(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                   int block, int dq_block, int64_t N, int64_t K,
                   const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                   int out_block, int out_dq_block, uint8_t* out_codes,
                   uint8_t* out_absmax_q, float* out_dq_scale, void* stream);

/* Workspace bytes needed by qlora_linear_fwd / qlora_linear_bwd for these
 * shapes (the caller allocates it, 256-byte aligned, device memory). */
int qlora_linear_fwd_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes);
int qlora_linear_bwd_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes);

/* Forward of the QLoRA linear ("QLoRA: fine-tuning a large model on one GPU",
 * "LoRA, stated once"):
 *     Y = X deq(W)^T + scale * (X A^T) B^T
 * with deq(W) expanded to bf16 on the fly inside the tensor-core GEMM and
 * never written to memory.  Accumulation is fp32; Y is rounded to bf16.
 * X: bf16 [M, K]; A: bf16 [r, K]; B: bf16 [N, r]; Y: bf16 [M, N] output.
 * H_save (nullable): bf16 [M, r] output receiving H = X A^T for the backward.
 * scale = alpha / r.  1 <= r <= 64, r % 8 == 0; K % 64 == 0; N % 8 == 0.
 * M <= 16 runs the bandwidth-bound decode kernel; larger M the tensor-core
 * GEMM (one selection by shape, both exact to the same tolerance).
 * workspace: device scratch of qlora_linear_fwd_workspace bytes.
 * Errors: ARG, SHAPE, UNSUPPORTED, WORKSPACE, CUDA. */
int qlora_linear_fwd(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                     int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                     const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                     qlora_bf16_t* Y, qlora_bf16_t* H_save,
                     void* workspace, size_t workspace_bytes, void* stream);

/* qlora_linear_fwd for an NF4 weight in any format the codec writes: block
 * in {32, 64, 128, 256}, dq_block 256 or 0 (absmax_q may then be NULL; see
 * the NF4 format above; K % block == 0).  qlora_linear_fwd is this call with
 * block 64, dq_block 256.  For M <= 16 the bandwidth-bound decode kernel reads
 * blocks of 64, 128 and 256 with double quantization on or off (each
 * 64-weight group of a row then has one scale); block 32 runs the tensor-core
 * GEMM for every M. */
int qlora_linear_fwd_fmt(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                         int block, int dq_block, int64_t N, int64_t K,
                         const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A,
                         const qlora_bf16_t* B, int r, float scale, qlora_bf16_t* Y,
                         qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Multi-adapter decode (one frozen NF4 base serving many adapters;
 * "QLoRA and Quantized Fine-Tuning", "The two mechanisms combined"): token m
 * uses adapter a = adapter_idx[m] of a stack,
 *     Y[m] = X[m] deq(W)^T + scales[a] * (X[m] A_a^T) B_a^T.
 * A_all: bf16 [n_adapters, r, K]; B_all: bf16 [n_adapters, N, r];
 * scales: device fp32 [n_adapters]; adapter_idx: device int32 [M].  A token
 * whose index is outside [0, n_adapters) gets no LoRA term.  M <= 16 (the
 * decode kernel; larger M: QLORA_ERR_UNSUPPORTED); the default NF4 format.
 * workspace: qlora_linear_fwd_workspace(M, N, K, r) bytes.  Same shape rules
 * and errors as qlora_linear_fwd. */
int qlora_linear_fwd_multi(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                           int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                           const qlora_bf16_t* A_all, const qlora_bf16_t* B_all, int n_adapters,
                           int r, const float* scales, const int32_t* adapter_idx, qlora_bf16_t* Y,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Decode tiles: a serving layout of an NF4 weight's codes for the decode
 * calls below (M <= 16), made once when the weight is loaded.  It holds the
 * same code bytes as the row-major codes (the NF4 format above, "NF4: 4-bit
 * NormalFloat": two 4-bit codes per byte, first element in the low nibble),
 * rearranged so that every 16-row x 64-column unit is 512 contiguous bytes:
 * for tile tau (rows 16 tau .. 16 tau + 15), block kb and i = 4g + t
 * (g < 8, t < 4), bytes [16 i, 16 i + 16) of unit (tau, kb) at offset
 * (tau * K/64 + kb) * 512 are codes[16 tau + g][32 kb + 8t .. + 7] followed by
 * codes[16 tau + g + 8][32 kb + 8t .. + 7]; rows past N hold zeros.  absmax_q
 * and dq_scale keep their layout.  K % 1024 == 0 (QLORA_ERR_SHAPE otherwise).
 * nf4_decode_tiles_bytes: size of the tiles, ceil(N / 16) * K / 64 * 512.
 * nf4_decode_tiles: codes (device, row-major [N, K/2], 16-byte aligned) ->
 * tiles (device, caller-owned, 16-byte aligned), asynchronous on `stream`.
 * Errors: ARG, SHAPE, CUDA. */
int nf4_decode_tiles_bytes(int64_t N, int64_t K, size_t* bytes);
int nf4_decode_tiles(const uint8_t* codes, int64_t N, int64_t K, uint8_t* tiles, void* stream);

/* qlora_linear_fwd and qlora_linear_fwd_multi for M <= 16 tokens with the
 * codes given as decode tiles (default NF4 format: block 64, double
 * quantization over 256 blocks).  The result is the same sum in the same fp32
 * order per 16-block item, so it equals the row-major decode call to within
 * rounding of the per-item partial sums.  M > 16: QLORA_ERR_UNSUPPORTED.
 * Same shape rules, workspace and errors as the row-major calls, plus
 * K % 1024 == 0. */
int qlora_linear_fwd_tiles(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale,
                           int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                           const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                           qlora_bf16_t* Y, qlora_bf16_t* H_save,
                           void* workspace, size_t workspace_bytes, void* stream);
/* qlora_linear_fwd_tiles for an NF4 weight in block 64, 128 or 256 with
 * double quantization on (dq_block 256) or off (dq_block 0; absmax_q may then
 * be NULL); the decode tiles do not depend on the format.  block 32:
 * QLORA_ERR_UNSUPPORTED.  qlora_linear_fwd_tiles is this call with block 64,
 * dq_block 256. */
int qlora_linear_fwd_tiles_fmt(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale,
                               int block, int dq_block, int64_t N, int64_t K, const qlora_bf16_t* X,
                               int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B, int r,
                               float scale, qlora_bf16_t* Y, qlora_bf16_t* H_save, void* workspace,
                               size_t workspace_bytes, void* stream);
int qlora_linear_fwd_multi_tiles(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale,
                                 int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                                 const qlora_bf16_t* A_all, const qlora_bf16_t* B_all, int n_adapters,
                                 int r, const float* scales, const int32_t* adapter_idx, qlora_bf16_t* Y,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the QLoRA linear: gradients flow through deq(W) to the
 * adapters and to the input; the frozen base gets none (katajob, "What stays
 * in full precision"):
 *     dH = scale * dY B                 [M, r]
 *     dX = dY deq(W) + dH A             [M, K]
 *     dA = dH^T X                       [r, K]
 *     dB = scale * dY^T H,  H = X A^T   [N, r]
 * dY: bf16 [M, N].  H: bf16 [M, r] from qlora_linear_fwd's H_save, or NULL to
 * recompute it.  dX, dA, dB: bf16 outputs (dX may be NULL to skip it).
 * With dX, dA and dB are computed on an internal side stream that forks from
 * `stream` after dH and joins it before the call returns (two events), so they
 * overlap the dX GEMM; every output is ready when the work enqueued on
 * `stream` is, also inside a CUDA graph captured from `stream`.  Each caller
 * stream gets its own side stream and events (up to 64 caller streams per
 * device; further ones run all kernels on `stream`), so backward calls on
 * independent streams do not wait for each other.  A side stream is created
 * outside any capture: a first call on a stream made during a capture runs all
 * kernels on `stream`.
 * Same shape rules and errors as qlora_linear_fwd. */
int qlora_linear_bwd(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                     int64_t N, int64_t K, const qlora_bf16_t* X, const qlora_bf16_t* dY,
                     int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B, int r,
                     float scale, const qlora_bf16_t* H,
                     qlora_bf16_t* dX, qlora_bf16_t* dA, qlora_bf16_t* dB,
                     void* workspace, size_t workspace_bytes, void* stream);

/* qlora_linear_bwd for an NF4 weight in any codec format (as
 * qlora_linear_fwd_fmt); qlora_linear_bwd is this call with block 64,
 * dq_block 256. */
int qlora_linear_bwd_fmt(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                         int block, int dq_block, int64_t N, int64_t K,
                         const qlora_bf16_t* X, const qlora_bf16_t* dY, int64_t M,
                         const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                         const qlora_bf16_t* H, qlora_bf16_t* dX, qlora_bf16_t* dA,
                         qlora_bf16_t* dB, void* workspace, size_t workspace_bytes, void* stream);

/* LoRA dropout on the adapter input ("QLoRA: fine-tuning a large model on one
 * GPU": lora_dropout in the LoraConfig).  The adapter branch reads
 *     Xd = keep_mask ? bf16(fl32(X * keep_scale)) : 0
 * (keep_mask: device uint8 [M, K], 1 = keep, the caller's random draw;
 * keep_scale = 1 / (1 - p)); the base product reads X itself:
 *     Y  = X deq(W)^T + scale * (Xd A^T) B^T
 *     dX = dY deq(W) + keep_mask * keep_scale * (dH A),  dH = scale * dY B
 *     dA = dH^T Xd,  dB = scale * dY^T H,  H = Xd A^T  (H_save / H hold it).
 * Xd is not stored for M > 16: the H and dA kernels apply the mask to the X
 * tiles they load (for M <= 16 a small Xd sits in the workspace).
 * workspace: qlora_linear_dropout_workspace bytes (shared by both calls).
 * Shapes, format and errors as qlora_linear_fwd / qlora_linear_bwd; keep_mask
 * 16-byte aligned; a nonzero byte keeps. */
int qlora_linear_dropout_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes);
int qlora_linear_fwd_dropout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                             int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                             const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                             const uint8_t* keep_mask, float keep_scale, qlora_bf16_t* Y,
                             qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes,
                             void* stream);
int qlora_linear_bwd_dropout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                             int64_t N, int64_t K, const qlora_bf16_t* X, const qlora_bf16_t* dY,
                             int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B, int r,
                             float scale, const uint8_t* keep_mask, float keep_scale,
                             const qlora_bf16_t* H, qlora_bf16_t* dX, qlora_bf16_t* dA,
                             qlora_bf16_t* dB, void* workspace, size_t workspace_bytes, void* stream);

/* Largest M * r that qlora_linear_fwd_noalloc accepts: its fixed device
 * scratch holds this many bf16 values (2 MiB on every device that loads the
 * library, held until the process exits). */
#define QLORA_NOALLOC_MAX_TOKENS_X_RANK (1 << 20)

/* qlora_linear_fwd for callers that cannot allocate device memory -- for
 * example a plugin inside a framework that owns all device memory and gives
 * the plugin no allocator, a service that reserves its memory up front and
 * forbids later allocations, or a latency-critical thread that cannot take
 * cudaMalloc's implicit device synchronization.  The QLoRA pages have no
 * counterpart to this entry point; it exists only for such callers.
 * Same arguments, result and errors as qlora_linear_fwd, minus the workspace:
 * the scratch lives in a fixed array in device memory inside the library, and
 * no cudaMalloc, cudaFree or other allocating routine is called.
 * Limits: M * r <= QLORA_NOALLOC_MAX_TOKENS_X_RANK, else QLORA_ERR_WORKSPACE
 * (returned before anything is enqueued).
 * Sharing: all calls on a device share the one scratch array, which keeps the
 * last call's contents; calls that overlap on the GPU (streams without
 * ordering between them) race on it.
 * Set-up: the first call on each device looks up the array's device address
 * with that device current; make that first call before any stream capture. */
int qlora_linear_fwd_noalloc(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                             int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                             const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                             qlora_bf16_t* Y, qlora_bf16_t* H_save, void* stream);

/* Reads and clears the device status word of the current device (a
 * QLORA_ERR_TIMEOUT left by a bounded wait, else QLORA_OK).  Synchronizes the
 * device. */
int qlora_device_status(void);

/* Testing aid for the bounded device waits (the QLoRA pages have no
 * counterpart; it exists so that the failure path can be exercised without a
 * fault).  Runs the row-major decode forward of qlora_linear_fwd (1 <= M <= 16,
 * the default NF4 format, the same arguments minus H_save) with every wait of
 * the decode kernel limited to 1 ms and its copy producer told to skip the
 * copy of its second code stage in every CTA.  The consumers' wait for that
 * stage runs out; the kernel then lets the copies it did issue land and
 * returns, leaving Y unspecified and QLORA_ERR_TIMEOUT in the device status
 * word (qlora_device_status).  No memory outside Y and the workspace is
 * written, and later calls run normally.
 * Errors: as qlora_linear_fwd; M > 16: UNSUPPORTED. */
int qlora_test_decode_timeout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                              int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                              const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                              qlora_bf16_t* Y, void* workspace, size_t workspace_bytes, void* stream);

/* Kernel-level tracing for profiling.  While enabled, each launch of the
 * fused dequant-GEMM kernel (forward or dX) records events[2i] before and
 * events[2i+1] after it on the launching stream, for i = 0, 1, ... up to
 * n_pairs - 1 (later launches are not recorded).  `events` is a host array of
 * cudaEvent_t owned by the caller; n_pairs = 0 disables tracing.  Tracing is
 * per host thread: it records the launches made by the thread that set it.
 * Errors: ARG. */
int qlora_trace_gemm_events(void** events, int n_pairs);

/* Number of event pairs recorded on this host thread since its last
 * qlora_trace_gemm_events. */
int qlora_trace_gemm_count(void);

/* How many CTA pairs (2-SM clusters) of the fused dequant-GEMM kernel can be
 * resident at once on the current device; mode 0 = forward, 1 = dX.  A value
 * of 0 means the kernel cannot launch on this device.  Errors: ARG, CUDA. */
int qlora_gemm_resident_pairs(int mode);

/* How the fused GEMM divides an M x N x K layer's tiles on the current device
 * (mode 0 = forward: N outputs, contraction K; 1 = dX: K outputs, contraction
 * N).  Tiles are 512 tokens x 256 outputs, one per CTA pair; when the tiles
 * leave a partial last wave on the resident pairs, each of those *ntail_tiles
 * tiles is split along the contraction into *nsplit pieces of at least 16
 * 64-wide stages, whose fp32 partial sums (*partial_bytes in all) a second
 * kernel adds in piece order before the one bf16 rounding.  The layer entry
 * points split only when the caller's workspace holds the partial sums too
 * (the workspace functions above include them); with a smaller workspace
 * they run every tile whole.  *nsplit = 1: no split.  Without a device (or
 * for M <= 16, which runs the decode kernel) the plan is no split.  Any
 * output pointer may be NULL.  Errors: ARG (mode, negative sizes). */
int qlora_gemm_split_plan(int mode, int64_t M, int64_t N, int64_t K, int* nsplit, int64_t* ntail_tiles,
                          size_t* partial_bytes);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
