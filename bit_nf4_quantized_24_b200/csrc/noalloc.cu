// qlora_linear_fwd_noalloc: the forward of the QLoRA linear for callers that
// cannot allocate device memory.
//
// qlora_linear_fwd needs a little scratch (the bf16 tensor scale * X A^T that
// feeds the GEMM's LoRA stage), which its caller passes in as `workspace`.
// Some callers have no way to provide it: a plugin hosted by a framework that
// owns the whole device memory and exposes no allocator to it, a service that
// reserves all memory up front and forbids allocations afterwards, or a
// latency-critical thread that cannot afford cudaMalloc's implicit device
// synchronization.  This entry point takes the same inputs and outputs but
// keeps its scratch in a fixed array in device memory that is part of the
// library image: it calls no cudaMalloc, cudaFree or allocating library
// routine.
//
// Limits and sharing:
//  - The array holds kScratchElems bf16 values, so M * r must not exceed it
//    (QLORA_NOALLOC_MAX_TOKENS_X_RANK); larger calls are rejected with
//    QLORA_ERR_WORKSPACE before anything is enqueued.
//  - Every device that loads the library holds its own copy for the life of
//    the process.
//  - All calls on a device share the one array and it keeps whatever the last
//    call wrote.  Each call writes the whole region it reads before reading it,
//    so nothing needs clearing, but two calls that overlap on the GPU (on
//    different streams without ordering between them) race on it.
//  - The first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before any stream capture begins.
#include <cmath>
#include <mutex>

#include "internal.h"
#include "qlora_nf4.h"

namespace qn {

namespace {

constexpr int64_t kScratchElems = QLORA_NOALLOC_MAX_TOKENS_X_RANK;
static_assert(kScratchElems * 2 % 256 == 0, "scratch size");

// Host code must not use this name as a pointer: on the host it is only a
// stand-in for the symbol.  Its device address comes from cudaGetSymbolAddress.
__device__ __align__(256) uint16_t g_fwd_scratch[kScratchElems];

constexpr int kMaxDev = 64;
uint16_t* g_scratch_addr[kMaxDev];
std::mutex g_scratch_mutex;

// Device address of g_fwd_scratch on the current device (looked up once per
// device, with that device current); nullptr on failure.
uint16_t* scratch_on_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDev) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_fwd_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = static_cast<uint16_t*>(p);
  }
  *err = cudaSuccess;
  return g_scratch_addr[dev];
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

}  // namespace qn

using namespace qn;

extern "C" int qlora_linear_fwd_noalloc(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                                        int64_t N, int64_t K, const qlora_bf16_t* X, int64_t M,
                                        const qlora_bf16_t* A, const qlora_bf16_t* B, int r, float scale,
                                        qlora_bf16_t* Y, qlora_bf16_t* H_save, void* stream) {
  // the same shape and pointer rules as qlora_linear_fwd (shared checks)
  int st = check_layer_shapes(M, N, K, r);
  if (st) return st;
  if (!codes || !absmax_q || !dq_scale || !A || !B || (M > 0 && (!X || !Y))) return QLORA_ERR_ARG;
  if (!std::isfinite(scale)) return QLORA_ERR_ARG;
  if (M * r > kScratchElems) return QLORA_ERR_WORKSPACE;  // beyond the fixed scratch
  if (M == 0) return QLORA_OK;
  const void* ptrs[] = {codes, X, A, B, Y};
  for (const void* p : ptrs)
    if (!is_aligned16(p)) return QLORA_ERR_SHAPE;
  if (H_save && !is_aligned16(H_save)) return QLORA_ERR_SHAPE;

  cudaError_t e;
  uint16_t* Hs = scratch_on_current_device(&e);
  if (!Hs) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = launch_rowdot(X, A, M, K, r, scale, Hs, 1.0f, H_save, nullptr, s, true);
  if (e == cudaSuccess) {
    if (M <= 16) {
      e = launch_gemv(X, M, codes, absmax_q, dq_scale, N, K, Hs, B, r, Y, s);
    } else {
      GemmArgs a{};
      a.mode = 0;
      a.act = X;
      a.tail_a = Hs;
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
      e = launch_nf4_gemm(a, s);
    }
  }
  return cuda_status(e);
}
