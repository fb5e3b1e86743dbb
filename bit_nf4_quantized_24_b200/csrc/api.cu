// The C ABI (include/qlora_nf4.h): argument checks, workspace layout, the
// sequence of kernel launches for each call, device status and tracing.
#include <climits>
#include <cstring>
#include <mutex>
#include <thread>
#include <unordered_map>

#include "internal.h"
#include "qlora_nf4.h"

namespace qn {

// File-scope device words: the status of bounded waits, and a pool of
// non-finite flags for nf4_quantize / nf4_merge_lora (one per call in flight;
// a call takes a free slot, clears it, lets the kernel set it and reads it back
// before it returns).  Every device that loads the library holds its own copy.
constexpr int kFlagSlots = 64;
__device__ int g_device_status;
__device__ int g_nonfinite[kFlagSlots];

namespace {

thread_local int t_last_cuda_error = 0;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
int* g_nonfinite_ptr[kMaxDevices];
std::mutex g_symbol_mutex;
std::atomic<uint64_t> g_flag_busy[kMaxDevices];

// Tracing of the fused-GEMM launches, per host thread (each thread records
// the launches it makes).
thread_local void** t_trace_events = nullptr;
thread_local int t_trace_pairs = 0;
thread_local int t_trace_count = 0;

// Side streams of the backward: dA and dB run on a side stream while the dX
// GEMM runs on the caller's stream (fork and join through two events).  Each
// caller stream of a device gets its own side stream and events, so the
// backward calls of independent streams never wait for one another; the
// mutex guards only the lookup and creation.
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
constexpr size_t kMaxSideStreams = 64;  // per device; further caller streams run the backward on one stream
std::unordered_map<cudaStream_t, SideStream> g_side[kMaxDevices];
std::mutex g_side_mutex;

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

}  // namespace

int device_sm_count() {
  static std::atomic<int> cache[kMaxDevices] = {};
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  int v = cache[d].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) return 148;
  cache[d].store(v, std::memory_order_relaxed);
  return v;
}

namespace {


template <typename T>
T* symbol_ptr(T** cache, const void* symbol) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_symbol_mutex);
  if (!cache[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    cache[d] = static_cast<T*>(p);
  }
  return cache[d];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Scratch of the dropout variants: Xd [M, K] bf16 and a zero [M, r] bf16
// tail (the dX GEMM then adds no adapter term; k_dx_add_masked does, masked).
struct DropWorkspace {
  uint16_t* Xd;
  uint16_t* zero_tail;
  size_t bytes;
};
DropWorkspace drop_layout(void* ws, size_t off0, int64_t M, int64_t K, int r) {
  DropWorkspace w{};
  size_t off = (off0 + 255) & ~size_t(255);
  uint8_t* p = static_cast<uint8_t*>(ws);
  w.Xd = p ? reinterpret_cast<uint16_t*>(p + off) : nullptr;
  // Xd [M, K] only for M <= 16 (larger M applies the mask inside the adapter kernels)
  off += M <= 16 ? (static_cast<size_t>(M) * K * 2 + 255) & ~size_t(255) : 0;
  w.zero_tail = p ? reinterpret_cast<uint16_t*>(p + off) : nullptr;
  off += (static_cast<size_t>(M) * r * 2 + 255) & ~size_t(255);
  w.bytes = off;
  return w;
}


struct FwdWorkspace {
  uint16_t* Hs;  // bf16(scale * X A^T) [M, r]
  size_t bytes;
};
FwdWorkspace fwd_layout(void* ws, int64_t M, int r) {
  FwdWorkspace w{};
  uint8_t* p = static_cast<uint8_t*>(ws);
  w.Hs = reinterpret_cast<uint16_t*>(p);
  w.bytes = align256(static_cast<size_t>(M) * r * 2);
  if (w.bytes == 0) w.bytes = 256;
  return w;
}

struct BwdWorkspace {
  uint16_t* dH16;   // bf16(scale * dY B) [M, r]
  uint16_t* H16;    // bf16(X A^T) [M, r] when recomputed
  size_t bytes;
};
BwdWorkspace bwd_layout(void* ws, int64_t M, int64_t N, int64_t K, int r) {
  BwdWorkspace w{};
  size_t off = 0;
  uint8_t* p = static_cast<uint8_t*>(ws);
  auto take = [&](size_t n) {
    uint8_t* q = p ? p + off : nullptr;
    off += align256(n);
    return q;
  };
  w.dH16 = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(M) * r * 2));
  w.H16 = reinterpret_cast<uint16_t*>(take(static_cast<size_t>(M) * r * 2));
  w.bytes = off;
  return w;
}

// The fused GEMM's room for the fp32 partial sums of split tiles: whatever
// the workspace holds past its first `used` bytes (the launch splits only if
// that is at least the plan's part_bytes).
void gemm_part(GemmArgs& a, void* ws, size_t used, size_t ws_bytes) {
  const size_t off = align256(used);
  if (ws && ws_bytes > off) {
    a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + off);
    a.part_bytes = ws_bytes - off;
  }
}
size_t gemm_part_bytes(int mode, int64_t M, int64_t N, int64_t K) {
  return M > 16 ? align256(gemm_split_plan(mode, M, N, K).part_bytes) : 0;
}

// The side stream of caller stream `s` on the current device, created on
// first use.  Returns false (the backward then runs on `s` alone) if creation
// fails, if the device already has kMaxSideStreams of them, or if `s` is being
// captured into a CUDA graph before its side stream exists (creating a stream
// inside a capture is not allowed everywhere).  The entry, once made, is never
// changed or removed, so the copy returned stays valid.
bool side_stream(cudaStream_t s, SideStream* out) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(g_side_mutex);
  auto& map = g_side[d];
  auto it = map.find(s);
  if (it != map.end()) {
    *out = it->second;
    return true;
  }
  if (map.size() >= kMaxSideStreams) return false;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) return false;
  SideStream ss;
  if (cudaStreamCreateWithFlags(&ss.st, cudaStreamNonBlocking) != cudaSuccess) return false;
  if (cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
    if (ss.fork) cudaEventDestroy(ss.fork);
    cudaStreamDestroy(ss.st);
    return false;
  }
  map.emplace(s, ss);
  *out = ss;
  return true;
}

// A free non-finite flag slot of the current device (its index), held until
// release_flag.  More than kFlagSlots calls in flight at once on one device
// wait here for a slot to come free.
int acquire_flag(int dev) {
  std::atomic<uint64_t>& busy = g_flag_busy[dev];
  for (;;) {
    uint64_t cur = busy.load(std::memory_order_relaxed);
    while (~cur) {
      const int slot = __builtin_ctzll(~cur);
      if (busy.compare_exchange_weak(cur, cur | (uint64_t(1) << slot), std::memory_order_acquire))
        return slot;
    }
    std::this_thread::yield();
  }
}
void release_flag(int dev, int slot) {
  g_flag_busy[dev].fetch_and(~(uint64_t(1) << slot), std::memory_order_release);
}

// Runs `launch(flag)` on `s` with a cleared per-call non-finite flag and
// reports it (synchronizes `s`).
template <typename F>
int run_with_nonfinite_flag(cudaStream_t s, F&& launch) {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return cuda_status(cudaErrorInvalidDevice);
  int* flags = device_nonfinite_ptr();
  if (!flags) return cuda_status(cudaErrorInvalidSymbol);
  const int slot = acquire_flag(dev);
  int* flag = flags + slot;
  cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int), s);
  if (e == cudaSuccess) e = launch(flag);
  int host_flag = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host_flag, flag, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaStreamSynchronize(s);  // nothing of this call may still touch the slot once it is released
    release_flag(dev, slot);
    return cuda_status(e);
  }
  release_flag(dev, slot);
  return host_flag ? QLORA_ERR_NONFINITE : QLORA_OK;
}

}  // namespace

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QLORA_OK;
  t_last_cuda_error = static_cast<int>(e);
  return QLORA_ERR_CUDA;
}

int check_layer_shapes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 0 || N <= 0 || K <= 0) return QLORA_ERR_ARG;
  if (r < 8 || r > 64 || r % 8) return r <= 0 ? QLORA_ERR_ARG : QLORA_ERR_UNSUPPORTED;
  if (K % 64 || N % 8) return QLORA_ERR_SHAPE;
  if (M > (1 << 24) || N > (1 << 24) || K > (1 << 24) || N * K / 2 > (int64_t(1) << 40)) return QLORA_ERR_SHAPE;
  return QLORA_OK;
}

int check_format(int64_t K, int block, int dq_block) {
  if ((block != 32 && block != 64 && block != 128 && block != 256) || (dq_block != 256 && dq_block != 0))
    return QLORA_ERR_UNSUPPORTED;
  return K % block ? QLORA_ERR_SHAPE : QLORA_OK;
}

int* device_status_ptr() { return symbol_ptr(g_status_ptr, &g_device_status); }
int* device_nonfinite_ptr() { return symbol_ptr(g_nonfinite_ptr, &g_nonfinite); }

void trace_before(cudaStream_t st) {
  if (t_trace_events && t_trace_count < t_trace_pairs)
    cudaEventRecord(static_cast<cudaEvent_t>(t_trace_events[2 * t_trace_count]), st);
}
void trace_after(cudaStream_t st) {
  if (t_trace_events && t_trace_count < t_trace_pairs) {
    cudaEventRecord(static_cast<cudaEvent_t>(t_trace_events[2 * t_trace_count + 1]), st);
    ++t_trace_count;
  }
}

}  // namespace qn

using namespace qn;

extern "C" {

const char* qlora_status_string(int status) {
  switch (status) {
    case QLORA_OK: return "QLORA_OK";
    case QLORA_ERR_ARG: return "QLORA_ERR_ARG: null pointer or invalid argument";
    case QLORA_ERR_SHAPE: return "QLORA_ERR_SHAPE: unsupported or misaligned shape";
    case QLORA_ERR_NONFINITE: return "QLORA_ERR_NONFINITE: the weight holds NaN or infinity";
    case QLORA_ERR_WORKSPACE: return "QLORA_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case QLORA_ERR_CUDA: return "QLORA_ERR_CUDA: a CUDA call failed";
    case QLORA_ERR_TIMEOUT: return "QLORA_ERR_TIMEOUT: a bounded device wait ran out";
    case QLORA_ERR_UNSUPPORTED: return "QLORA_ERR_UNSUPPORTED: parameter outside this build's set";
    default: return "QLORA_ERR_UNKNOWN";
  }
}

int qlora_last_cuda_error(void) { return t_last_cuda_error; }

int qlora_version(void) { return (1 << 16) | 0; }

int nf4_quantized_sizes(int64_t N, int64_t K, int block, int dq_block, size_t* codes_bytes, size_t* absmax_bytes,
                        size_t* dq_scale_bytes) {
  if (N < 0 || K < 0 || !codes_bytes || !absmax_bytes || !dq_scale_bytes) return QLORA_ERR_ARG;
  if ((block != 32 && block != 64 && block != 128 && block != 256) || (dq_block != 256 && dq_block != 0))
    return QLORA_ERR_UNSUPPORTED;
  if (K % block) return QLORA_ERR_SHAPE;
  const int64_t numel = N * K, nblocks = numel / block;
  *codes_bytes = static_cast<size_t>(numel / 2);
  *absmax_bytes = dq_block ? static_cast<size_t>(nblocks) : 0;
  *dq_scale_bytes = static_cast<size_t>(dq_block ? (nblocks + dq_block - 1) / dq_block : nblocks) * 4;
  return QLORA_OK;
}

int nf4_codebook(float* levels_out) {
  if (!levels_out) return QLORA_ERR_ARG;
  std::memcpy(levels_out, host_codebook().levels.v, sizeof(float) * 16);
  return QLORA_OK;
}

int nf4_quantize(const float* W, int64_t N, int64_t K, int block, int dq_block, uint8_t* codes,
                 uint8_t* absmax_q, float* dq_scale, void* stream) {
  size_t cb, ab, db;
  int st = nf4_quantized_sizes(N, K, block, dq_block, &cb, &ab, &db);
  if (st) return st;
  if (N * K == 0) return QLORA_OK;
  if (!W || !codes || (dq_block && !absmax_q) || !dq_scale) return QLORA_ERR_ARG;
  if (!aligned(W, 16) || !aligned(codes, 4)) return QLORA_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return run_with_nonfinite_flag(s, [&](int* flag) {
    return launch_quantize(W, N * K, block, dq_block, codes, absmax_q, dq_scale, flag, s);
  });
}

int nf4_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N, int64_t K,
                   int block, int dq_block, qlora_bf16_t* W_out, void* stream) {
  size_t cb, ab, db;
  int st = nf4_quantized_sizes(N, K, block, dq_block, &cb, &ab, &db);
  if (st) return st;
  if (N * K == 0) return QLORA_OK;
  if (!codes || (dq_block && !absmax_q) || !dq_scale || !W_out) return QLORA_ERR_ARG;
  if (!aligned(codes, 16) || !aligned(W_out, 16)) return QLORA_ERR_SHAPE;
  return cuda_status(
      launch_dequantize(codes, absmax_q, dq_scale, N * K, block, dq_block, W_out, static_cast<cudaStream_t>(stream)));
}

int nf4_merge_lora(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int block, int dq_block,
                   int64_t N, int64_t K, const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                   int out_block, int out_dq_block, uint8_t* out_codes, uint8_t* out_absmax_q, float* out_dq_scale,
                   void* stream) {
  size_t cb, ab, db;
  int st = nf4_quantized_sizes(N, K, block, dq_block, &cb, &ab, &db);
  if (st) return st;
  st = nf4_quantized_sizes(N, K, out_block, out_dq_block, &cb, &ab, &db);
  if (st) return st;
  if (r < 1 || r > 64 || !std::isfinite(scale)) return r < 1 ? QLORA_ERR_ARG : QLORA_ERR_UNSUPPORTED;
  if (N * K == 0) return QLORA_OK;
  if (!codes || (dq_block && !absmax_q) || !dq_scale || !A || !B || !out_codes || (out_dq_block && !out_absmax_q) ||
      !out_dq_scale)
    return QLORA_ERR_ARG;
  if (!aligned(codes, 4) || !aligned(A, 16) || !aligned(out_codes, 4)) return QLORA_ERR_SHAPE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return run_with_nonfinite_flag(s, [&](int* flag) {
    return launch_merge_quantize(codes, absmax_q, dq_scale, block, dq_block, N, K, A, B, r, scale, out_block,
                                 out_dq_block, out_codes, out_absmax_q, out_dq_scale, flag, s);
  });
}

int qlora_linear_fwd_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes) {
  if (!bytes) return QLORA_ERR_ARG;
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  *bytes = fwd_layout(nullptr, M, r).bytes + gemm_part_bytes(0, M, N, K);
  return QLORA_OK;
}

int qlora_linear_bwd_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes) {
  if (!bytes) return QLORA_ERR_ARG;
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  *bytes = bwd_layout(nullptr, M, N, K, r).bytes + gemm_part_bytes(1, M, N, K);
  return QLORA_OK;
}

int qlora_linear_fwd_fmt(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int block,
                         int dq_block, int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A,
                         const qlora_bf16_t* B, int r, float scale, qlora_bf16_t* Y, qlora_bf16_t* H_save,
                         void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  st = check_format(K, block, dq_block);
  if (st) return st;
  if (!codes || (dq_block && !absmax_q) || !dq_scale || !A || !B || (M > 0 && (!X || !Y))) return QLORA_ERR_ARG;
  if (!std::isfinite(scale)) return QLORA_ERR_ARG;
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {codes, X, A, B, Y};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  if (H_save && !aligned(H_save, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e = launch_rowdot(X, A, M, K, r, scale, w.Hs, 1.0f, H_save, nullptr, s, true);
  if (e != cudaSuccess) return cuda_status(e);
  if (M <= 16 && block >= 64) {  // the decode kernel (one scale per 64-weight block: not for block 32)
    e = launch_gemv(X, M, codes, absmax_q, dq_scale, N, K, w.Hs, B, r, Y, s, nullptr, 0, false, block, dq_block);
  } else {
    GemmArgs a{};
    a.mode = 0;
    a.act = X;
    a.tail_a = w.Hs;
    a.tail_b = B;
    a.codes = codes;
    a.absmax_q = absmax_q;
    a.dq_scale = dq_scale;
    a.M = M;
    a.N = N;
    a.K = K;
    a.r = r;
    a.out = Y;
    a.pdl = true;  // its main loop runs while the H kernel finishes; the LoRA tail waits
    a.block = block;
    a.dq_block = dq_block;
    gemm_part(a, workspace, w.bytes, workspace_bytes);
    e = launch_nf4_gemm(a, s);
  }
  return cuda_status(e);
}

int qlora_linear_fwd_multi(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N, int64_t K,
                           const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A_all, const qlora_bf16_t* B_all,
                           int n_adapters, int r, const float* scales, const int32_t* adapter_idx, qlora_bf16_t* Y,
                           void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (M > 16 || n_adapters < 1) return n_adapters < 1 ? QLORA_ERR_ARG : QLORA_ERR_UNSUPPORTED;
  if (!codes || !absmax_q || !dq_scale || !A_all || !B_all || !scales || (M > 0 && (!X || !Y || !adapter_idx)))
    return QLORA_ERR_ARG;
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {codes, X, A_all, B_all, Y};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rows_multi(X, M, K, A_all, n_adapters, r, scales, adapter_idx, w.Hs, s);
  if (e == cudaSuccess)
    e = launch_gemv(X, M, codes, absmax_q, dq_scale, N, K, w.Hs, B_all, r, Y, s, adapter_idx, n_adapters);
  return cuda_status(e);
}

int nf4_decode_tiles_bytes(int64_t N, int64_t K, size_t* bytes) {
  if (!bytes || N <= 0 || K <= 0) return QLORA_ERR_ARG;
  if (K % 1024 || N > (1 << 24) || K > (1 << 24)) return QLORA_ERR_SHAPE;
  *bytes = static_cast<size_t>(decode_tiles_bytes(N, K));
  return QLORA_OK;
}

int nf4_decode_tiles(const uint8_t* codes, int64_t N, int64_t K, uint8_t* tiles, void* stream) {
  size_t bytes = 0;
  int st = nf4_decode_tiles_bytes(N, K, &bytes);
  if (st) return st;
  if (!codes || !tiles) return QLORA_ERR_ARG;
  if (!aligned(codes, 16) || !aligned(tiles, 16)) return QLORA_ERR_SHAPE;
  return cuda_status(launch_pack_tiles(codes, N, K, tiles, static_cast<cudaStream_t>(stream)));
}

int qlora_linear_fwd_tiles_fmt(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale, int block,
                               int dq_block, int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                               const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale, qlora_bf16_t* Y,
                               qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  st = check_format(K, block, dq_block);
  if (st) return st;
  if (K % 1024) return QLORA_ERR_SHAPE;
  if (M > 16 || block == 32) return QLORA_ERR_UNSUPPORTED;
  if (!tiles || (dq_block && !absmax_q) || !dq_scale || !A || !B || (M > 0 && (!X || !Y))) return QLORA_ERR_ARG;
  if (!std::isfinite(scale)) return QLORA_ERR_ARG;
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {tiles, X, A, B, Y};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  if (H_save && !aligned(H_save, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rowdot(X, A, M, K, r, scale, w.Hs, 1.0f, H_save, nullptr, s, true);
  if (e == cudaSuccess)
    e = launch_gemv_tiles(X, M, tiles, absmax_q, dq_scale, N, K, w.Hs, B, r, Y, s, nullptr, 0, block, dq_block);
  return cuda_status(e);
}

int qlora_linear_fwd_tiles(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale, int64_t N, int64_t K,
                           const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B, int r,
                           float scale, qlora_bf16_t* Y, qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes,
                           void* stream) {
  return qlora_linear_fwd_tiles_fmt(tiles, absmax_q, dq_scale, 64, 256, N, K, X, M, A, B, r, scale, Y, H_save,
                                    workspace, workspace_bytes, stream);
}

int qlora_linear_fwd_multi_tiles(const uint8_t* tiles, const uint8_t* absmax_q, const float* dq_scale, int64_t N,
                                 int64_t K, const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A_all,
                                 const qlora_bf16_t* B_all, int n_adapters, int r, const float* scales,
                                 const int32_t* adapter_idx, qlora_bf16_t* Y, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (K % 1024) return QLORA_ERR_SHAPE;
  if (M > 16 || n_adapters < 1) return n_adapters < 1 ? QLORA_ERR_ARG : QLORA_ERR_UNSUPPORTED;
  if (!tiles || !absmax_q || !dq_scale || !A_all || !B_all || !scales || (M > 0 && (!X || !Y || !adapter_idx)))
    return QLORA_ERR_ARG;
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {tiles, absmax_q, X, A_all, B_all, Y};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rows_multi(X, M, K, A_all, n_adapters, r, scales, adapter_idx, w.Hs, s);
  if (e == cudaSuccess)
    e = launch_gemv_tiles(X, M, tiles, absmax_q, dq_scale, N, K, w.Hs, B_all, r, Y, s, adapter_idx, n_adapters);
  return cuda_status(e);
}

int qlora_linear_dropout_workspace(int64_t M, int64_t N, int64_t K, int r, size_t* bytes) {
  if (!bytes) return QLORA_ERR_ARG;
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  const size_t base = std::max(fwd_layout(nullptr, M, r).bytes, bwd_layout(nullptr, M, N, K, r).bytes);
  *bytes = drop_layout(nullptr, base, M, K, r).bytes +
           std::max(gemm_part_bytes(0, M, N, K), gemm_part_bytes(1, M, N, K));
  return QLORA_OK;
}

int qlora_linear_fwd_dropout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N,
                             int64_t K, const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B,
                             int r, float scale, const uint8_t* keep_mask, float keep_scale, qlora_bf16_t* Y,
                             qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (!codes || !absmax_q || !dq_scale || !A || !B || (M > 0 && (!X || !Y || !keep_mask))) return QLORA_ERR_ARG;
  if (!std::isfinite(scale) || !std::isfinite(keep_scale)) return QLORA_ERR_ARG;
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {codes, X, A, B, Y, keep_mask};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  if (H_save && !aligned(H_save, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  const size_t base = std::max(w.bytes, bwd_layout(nullptr, M, N, K, r).bytes);
  DropWorkspace d = drop_layout(workspace, base, M, K, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < d.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // H from the dropped-out input (masked inside the H kernel; small M from a
  // materialised Xd); the base product from X itself
  cudaError_t e;
  if (M > 16) {
    e = launch_rowdot_masked(X, keep_mask, keep_scale, A, M, K, r, scale, w.Hs, 1.0f, H_save, s, true);
  } else {
    e = launch_dropout_input(X, keep_mask, keep_scale, M * K, d.Xd, s, true);
    if (e == cudaSuccess) e = launch_rowdot(d.Xd, A, M, K, r, scale, w.Hs, 1.0f, H_save, nullptr, s, true);
  }
  if (e != cudaSuccess) return cuda_status(e);
  if (M <= 16) {
    e = launch_gemv(X, M, codes, absmax_q, dq_scale, N, K, w.Hs, B, r, Y, s);
  } else {
    GemmArgs a{};
    a.mode = 0;
    a.act = X;
    a.tail_a = w.Hs;
    a.tail_b = B;
    a.codes = codes;
    a.absmax_q = absmax_q;
    a.dq_scale = dq_scale;
    a.M = M;
    a.N = N;
    a.K = K;
    a.r = r;
    a.out = Y;
    a.pdl = true;
    gemm_part(a, workspace, d.bytes, workspace_bytes);
    e = launch_nf4_gemm(a, s);
  }
  return cuda_status(e);
}

int qlora_linear_bwd_dropout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N,
                             int64_t K, const qlora_bf16_t* X, const qlora_bf16_t* dY, int64_t M, const qlora_bf16_t* A,
                             const qlora_bf16_t* B, int r, float scale, const uint8_t* keep_mask, float keep_scale,
                             const qlora_bf16_t* H, qlora_bf16_t* dX, qlora_bf16_t* dA, qlora_bf16_t* dB,
                             void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (!codes || !absmax_q || !dq_scale || !A || !B || !dA || !dB || (M > 0 && (!X || !dY || !keep_mask)))
    return QLORA_ERR_ARG;
  if (!std::isfinite(scale) || !std::isfinite(keep_scale)) return QLORA_ERR_ARG;
  const void* ptrs[] = {codes, A, B, dA, dB};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  if ((X && !aligned(X, 16)) || (dY && !aligned(dY, 16)) || (dX && !aligned(dX, 16)) || (H && !aligned(H, 16)) ||
      (keep_mask && !aligned(keep_mask, 16)))
    return QLORA_ERR_SHAPE;
  BwdWorkspace w = bwd_layout(workspace, M, N, K, r);
  const size_t base = std::max(fwd_layout(nullptr, M, r).bytes, w.bytes);
  DropWorkspace d = drop_layout(workspace, base, M, K, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < d.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (M == 0) {
    e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 2, s);
    return cuda_status(e);
  }
  const bool masked = M > 16;  // the adapter kernels apply the mask; else Xd is materialised
  if (dX) e = cudaMemsetAsync(d.zero_tail, 0, static_cast<size_t>(M) * r * 2, s);
  if (e == cudaSuccess && !masked) e = launch_dropout_input(X, keep_mask, keep_scale, M * K, d.Xd, s, true);
  if (e == cudaSuccess) e = launch_rowdot_qt(dY, B, M, N, r, scale, w.dH16, scale, nullptr, nullptr, s, true);
  const uint16_t* Huse = H;
  if (e == cudaSuccess && !H) {
    e = masked ? launch_rowdot_masked(X, keep_mask, keep_scale, A, M, K, r, 1.0f, w.H16, 1.0f, nullptr, s, true)
               : launch_rowdot(d.Xd, A, M, K, r, 1.0f, w.H16, 1.0f, nullptr, nullptr, s, true);
    Huse = w.H16;
  }
  // dA = dH^T Xd
  auto run_da = [&](cudaStream_t st, bool pdl) {
    return masked ? launch_coldot_masked(w.dH16, X, keep_mask, keep_scale, M, K, r, 1.0f, dA, st, pdl)
                  : launch_coldot(w.dH16, d.Xd, M, K, r, 1.0f, 0, dA, st, pdl);
  };
  if (e != cudaSuccess) return cuda_status(e);
  // dY deq(W) with a zero adapter tail, then the masked adapter term
  auto run_dx = [&]() {
    GemmArgs a{};
    a.mode = 1;
    a.act = dY;
    a.tail_a = d.zero_tail;
    a.tail_b = A;
    a.codes = codes;
    a.absmax_q = absmax_q;
    a.dq_scale = dq_scale;
    a.M = M;
    a.N = N;
    a.K = K;
    a.r = r;
    a.out = dX;
    a.pdl = true;
    gemm_part(a, workspace, d.bytes, workspace_bytes);
    cudaError_t x = launch_nf4_gemm(a, s);
    if (x == cudaSuccess) x = launch_dx_add_masked(dX, w.dH16, A, keep_mask, keep_scale, M, K, r, s, true);
    return x;
  };
  // dA, dB beside the dX GEMM on the caller stream's side stream, as in the
  // plain backward (joined before the call returns)
  SideStream ss;
  if (dX && side_stream(s, &ss)) {
    e = cudaEventRecord(ss.fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.st, ss.fork, 0);
    if (e != cudaSuccess) return cuda_status(e);
    e = run_da(ss.st, false);
    if (e == cudaSuccess) e = launch_coldot(Huse, dY, M, N, r, scale, 1, dB, ss.st, true);
    if (e == cudaSuccess) e = run_dx();
    // join on every path, so that nothing of this call stays unordered with `s`
    cudaError_t j = cudaEventRecord(ss.join, ss.st);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(s, ss.join, 0);
    return cuda_status(e != cudaSuccess ? e : j);
  }
  e = run_da(s, true);
  if (e == cudaSuccess) e = launch_coldot(Huse, dY, M, N, r, scale, 1, dB, s, true);
  if (e == cudaSuccess && dX) e = run_dx();
  return cuda_status(e);
}

int qlora_linear_fwd(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N, int64_t K,
                     const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A, const qlora_bf16_t* B, int r,
                     float scale, qlora_bf16_t* Y, qlora_bf16_t* H_save, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return qlora_linear_fwd_fmt(codes, absmax_q, dq_scale, 64, 256, N, K, X, M, A, B, r, scale, Y, H_save, workspace,
                              workspace_bytes, stream);
}

namespace qn {
namespace {
// dX = dY deq(W) + dH A: the fused GEMM in its MN-major mode with the LoRA
// tail (dH, A); a programmatic dependent launch (it waits before the tail).
cudaError_t launch_dx_gemm(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int block,
                           int dq_block, int64_t N, int64_t K, const uint16_t* dY, int64_t M, const uint16_t* A, int r,
                           const uint16_t* dH, uint16_t* dX, void* ws, size_t used, size_t ws_bytes, cudaStream_t s) {
  GemmArgs a{};
  a.mode = 1;
  a.act = dY;
  a.tail_a = dH;
  a.tail_b = A;
  a.codes = codes;
  a.absmax_q = absmax_q;
  a.dq_scale = dq_scale;
  a.M = M;
  a.N = N;
  a.K = K;
  a.r = r;
  a.out = dX;
  a.pdl = true;
  a.block = block;
  a.dq_block = dq_block;
  gemm_part(a, ws, used, ws_bytes);
  return launch_nf4_gemm(a, s);
}
}  // namespace
}  // namespace qn

int qlora_linear_bwd_fmt(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int block,
                         int dq_block, int64_t N, int64_t K, const qlora_bf16_t* X, const qlora_bf16_t* dY, int64_t M,
                         const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale, const qlora_bf16_t* H,
                         qlora_bf16_t* dX, qlora_bf16_t* dA, qlora_bf16_t* dB, void* workspace, size_t workspace_bytes,
                         void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  st = check_format(K, block, dq_block);
  if (st) return st;
  if (!codes || (dq_block && !absmax_q) || !dq_scale || !A || !B || !dA || !dB || (M > 0 && (!X || !dY)))
    return QLORA_ERR_ARG;
  if (!std::isfinite(scale)) return QLORA_ERR_ARG;
  const void* ptrs[] = {codes, A, B, dA, dB};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  if ((X && !aligned(X, 16)) || (dY && !aligned(dY, 16)) || (dX && !aligned(dX, 16)) || (H && !aligned(H, 16)))
    return QLORA_ERR_SHAPE;
  BwdWorkspace w = bwd_layout(workspace, M, N, K, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e = cudaSuccess;
  if (M == 0) {  // no tokens: zero adapter gradients
    e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, static_cast<size_t>(N) * r * 2, s);
    return cuda_status(e);
  }
  // dH = scale * dY B  (B [N, r] read in place: its rows are the contraction),
  // then H if the caller did not keep it.  The second is a programmatic
  // dependent launch that waits for the first before touching shared data.
  e = launch_rowdot_qt(dY, B, M, N, r, scale, w.dH16, scale, nullptr, nullptr, s, true);
  const uint16_t* Huse = H;
  if (e == cudaSuccess && !H) {
    e = launch_rowdot(X, A, M, K, r, 1.0f, w.H16, 1.0f, nullptr, nullptr, s, true);
    Huse = w.H16;
  }
  if (e != cudaSuccess) return cuda_status(e);
  // dA = dH^T X and dB = scale * dY^T H do not feed the dX GEMM: they run on
  // the side stream while the GEMM runs on s, taking the SMs its last,
  // partial wave leaves idle; the call joins them before it returns.
  SideStream ss;
  if (dX && side_stream(s, &ss)) {
    e = cudaEventRecord(ss.fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ss.st, ss.fork, 0);
    if (e != cudaSuccess) return cuda_status(e);
    e = launch_dx_gemm(codes, absmax_q, dq_scale, block, dq_block, N, K, dY, M, A, r, w.dH16, dX, workspace, w.bytes,
                       workspace_bytes, s);
    if (e == cudaSuccess) e = launch_coldot(w.dH16, X, M, K, r, 1.0f, 0, dA, ss.st, false);
    if (e == cudaSuccess) e = launch_coldot(Huse, dY, M, N, r, scale, 1, dB, ss.st, true);
    // join on every path, so that nothing of this call stays unordered with `s`
    cudaError_t j = cudaEventRecord(ss.join, ss.st);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(s, ss.join, 0);
    return cuda_status(e != cudaSuccess ? e : j);
  }
  // one stream: dA, dB, then the dX GEMM (programmatic dependent launches:
  // the GEMM's main loop starts while the adapter kernels finish; only its
  // LoRA tail reads dH)
  e = launch_coldot(w.dH16, X, M, K, r, 1.0f, 0, dA, s, true);
  if (e == cudaSuccess) e = launch_coldot(Huse, dY, M, N, r, scale, 1, dB, s, true);
  if (e == cudaSuccess && dX)
    e = launch_dx_gemm(codes, absmax_q, dq_scale, block, dq_block, N, K, dY, M, A, r, w.dH16, dX, workspace, w.bytes,
                       workspace_bytes, s);
  return cuda_status(e);
}

int qlora_linear_bwd(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N, int64_t K,
                     const qlora_bf16_t* X, const qlora_bf16_t* dY, int64_t M, const qlora_bf16_t* A,
                     const qlora_bf16_t* B, int r, float scale, const qlora_bf16_t* H, qlora_bf16_t* dX,
                     qlora_bf16_t* dA, qlora_bf16_t* dB, void* workspace, size_t workspace_bytes, void* stream) {
  return qlora_linear_bwd_fmt(codes, absmax_q, dq_scale, 64, 256, N, K, X, dY, M, A, B, r, scale, H, dX, dA, dB,
                              workspace, workspace_bytes, stream);
}

int qlora_test_decode_timeout(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale, int64_t N,
                              int64_t K, const qlora_bf16_t* X, int64_t M, const qlora_bf16_t* A,
                              const qlora_bf16_t* B, int r, float scale, qlora_bf16_t* Y, void* workspace,
                              size_t workspace_bytes, void* stream) {
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (M < 1 || M > 16) return M < 1 ? QLORA_ERR_ARG : QLORA_ERR_UNSUPPORTED;
  if (!codes || !absmax_q || !dq_scale || !X || !A || !B || !Y || !std::isfinite(scale)) return QLORA_ERR_ARG;
  const void* ptrs[] = {codes, X, A, B, Y};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return QLORA_ERR_SHAPE;
  FwdWorkspace w = fwd_layout(workspace, M, r);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.bytes) return QLORA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_rowdot(X, A, M, K, r, scale, w.Hs, 1.0f, nullptr, nullptr, s);
  if (e == cudaSuccess) e = launch_gemv(X, M, codes, absmax_q, dq_scale, N, K, w.Hs, B, r, Y, s, nullptr, 0, true);
  return cuda_status(e);
}

int qlora_device_status(void) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e);
  int* p = device_status_ptr();
  if (!p) return cuda_status(cudaErrorInvalidSymbol);
  int v = 0;
  e = cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_status(e);
  return v == kDevTimeout ? QLORA_ERR_TIMEOUT : QLORA_OK;
}

int qlora_trace_gemm_events(void** events, int n_pairs) {
  if (n_pairs < 0 || (n_pairs > 0 && !events)) return QLORA_ERR_ARG;
  t_trace_events = n_pairs > 0 ? events : nullptr;
  t_trace_pairs = n_pairs;
  t_trace_count = 0;
  return QLORA_OK;
}

int qlora_trace_gemm_count(void) { return t_trace_count; }

int qlora_gemm_split_plan(int mode, int64_t M, int64_t N, int64_t K, int* nsplit, int64_t* ntail_tiles,
                          size_t* partial_bytes) {
  if ((mode != 0 && mode != 1) || M < 0 || N <= 0 || K <= 0) return QLORA_ERR_ARG;
  SplitPlan p{};
  if (M > 16) p = gemm_split_plan(mode, M, N, K);
  if (nsplit) *nsplit = p.nsplit;
  if (ntail_tiles) *ntail_tiles = p.nsplit > 1 ? p.ntail : 0;
  if (partial_bytes) *partial_bytes = p.part_bytes;
  return QLORA_OK;
}

int qlora_gemm_resident_pairs(int mode) {
  if (mode != 0 && mode != 1) return QLORA_ERR_ARG;
  const int n = nf4_gemm_max_active_pairs(mode);
  return n < 0 ? QLORA_ERR_CUDA : n;
}

}  // extern "C"
