// Decode-sized forward (M <= 16 tokens): Y = X deq(W)^T + Hs B^T, Hs = bf16(s X A^T).
// Bound by streaming the NF4 weight once (katajob, "NF4: 4-bit NormalFloat":
// the weight is read in 4-bit and expanded per block only inside the product).
//
// CTA = 4 warps x 16 weight rows; every warp walks the whole K.  Per 256-wide
// K slice a lane reads one full 64-weight block (32 code bytes) of one row,
// builds that block's register lookup table and expands it straight into
// m16n8k16 B fragments -- the dequantized weight never touches memory.
// Lane t's block supplies k-slots {2t, 2t+1, 2t+8, 2t+9} of 16 MMA steps;
// the activations are staged in shared memory in the same permuted order so
// that each A fragment is one conflict-free 16-byte load.
#include "internal.h"

namespace qn {

namespace {

constexpr int GV_WARPS = 4;
constexpr int GV_CHUNK = 512;  // K elements staged per buffer
constexpr int GV_UNITS = 16 * GV_CHUNK / 8;  // 16-byte units per buffer

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // 0 source bytes -> 16 zero bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// smem 16-byte unit holding X[row][k .. k+7] (k = chunk-local, multiple of 8)
__device__ __forceinline__ int unit_of(int row, int k) {
  const int sc = k >> 8, t = (k >> 6) & 3, ip = (k >> 3) & 7;
  return ((sc * 8 + ip) * 16 + row) * 4 + t;
}

struct Slice {  // one lane's code block for one n8 tile
  uint4 q0, q1;
  float ap;
};

__device__ __forceinline__ Slice load_slice(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ absmax_q,
                                            const float* __restrict__ dq_scale, int row, int N, int K, int kblk) {
  Slice s;
  const bool ok = row < N && kblk * 64 < K;
  if (ok) {
    const uint8_t* p = codes + (static_cast<int64_t>(row) * K + kblk * 64) / 2;
    s.q0 = ldg_nc_v4(p);
    s.q1 = ldg_nc_v4(p + 16);
    const int64_t b = static_cast<int64_t>(row) * (K / 64) + kblk;
    s.ap = __fmul_rn(static_cast<float>(__ldg(absmax_q + b)), __ldg(dq_scale + (b >> 8)));
  } else {
    s.q0 = s.q1 = make_uint4(0u, 0u, 0u, 0u);
    s.ap = 0.0f;
  }
  return s;
}

__global__ void __launch_bounds__(GV_WARPS * 32) k_gemv(const uint16_t* __restrict__ X, int M,
                                                        const uint8_t* __restrict__ codes,
                                                        const uint8_t* __restrict__ absmax_q,
                                                        const float* __restrict__ dq_scale, int N, int K,
                                                        const uint16_t* __restrict__ Hs,
                                                        const uint16_t* __restrict__ Bl, int r, Nf4Levels lv,
                                                        uint16_t* __restrict__ Y) {
  __shared__ __align__(16) uint16_t sx[2][GV_UNITS * 8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int nrow0 = (blockIdx.x * GV_WARPS + warp) * 16;  // this warp's 16 weight rows
  const int nchunks = (K + GV_CHUNK - 1) / GV_CHUNK;
  const uint32_t sx_base = smem_u32(&sx[0][0]);

  auto stage = [&](int c, int buf) {
    const int k0 = c * GV_CHUNK;
    for (int u = tid; u < GV_UNITS; u += GV_WARPS * 32) {
      const int row = u / (GV_CHUNK / 8), kl = (u % (GV_CHUNK / 8)) * 8;
      const bool ok = row < M && k0 + kl < K;
      const uint16_t* src = ok ? X + static_cast<int64_t>(row) * K + k0 + kl : X;
      cp_async_16(sx_base + buf * (GV_UNITS * 16) + unit_of(row, kl) * 16, src, ok);
    }
    cp_async_commit();
  };

  float acc[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

  stage(0, 0);
  const int nsub = nchunks * 2;
  Slice cur0 = load_slice(codes, absmax_q, dq_scale, nrow0 + g, N, K, t);
  Slice cur1 = load_slice(codes, absmax_q, dq_scale, nrow0 + 8 + g, N, K, t);
  for (int sub = 0; sub < nsub; ++sub) {
    const int c = sub >> 1, sc = sub & 1;
    if (sc == 0) {
      if (c + 1 < nchunks) stage(c + 1, (c + 1) & 1);
      else cp_async_commit();
      cp_async_wait_1();
      __syncthreads();
    }
    Slice nxt0, nxt1;
    if (sub + 1 < nsub) {
      nxt0 = load_slice(codes, absmax_q, dq_scale, nrow0 + g, N, K, (sub + 1) * 4 + t);
      nxt1 = load_slice(codes, absmax_q, dq_scale, nrow0 + 8 + g, N, K, (sub + 1) * 4 + t);
    }
    const uint32_t xb = sx_base + (c & 1) * (GV_UNITS * 16);
    const Nf4Lut lut0 = make_lut(lv, cur0.ap), lut1 = make_lut(lv, cur1.ap);
    const uint32_t w0[8] = {cur0.q0.x, cur0.q0.y, cur0.q0.z, cur0.q0.w, cur0.q1.x, cur0.q1.y, cur0.q1.z, cur0.q1.w};
    const uint32_t w1[8] = {cur1.q0.x, cur1.q0.y, cur1.q0.z, cur1.q0.w, cur1.q1.x, cur1.q1.y, cur1.q1.z, cur1.q1.w};
#pragma unroll
    for (int ip = 0; ip < 8; ++ip) {
      const int u = ((sc * 8 + ip) * 16 + g) * 4 + t;
      const uint4 alo = ld_shared_v4(xb + u * 16);
      const uint4 ahi = ld_shared_v4(xb + (u + 32) * 16);
      uint32_t o0, o1, o2, o3;
      deq8(w0[ip], lut0, o0, o1, o2, o3);
      mma16816(acc[0], alo.x, ahi.x, alo.y, ahi.y, o0, o1);
      mma16816(acc[0], alo.z, ahi.z, alo.w, ahi.w, o2, o3);
      deq8(w1[ip], lut1, o0, o1, o2, o3);
      mma16816(acc[1], alo.x, ahi.x, alo.y, ahi.y, o0, o1);
      mma16816(acc[1], alo.z, ahi.z, alo.w, ahi.w, o2, o3);
    }
    if (sc == 1) __syncthreads();  // the buffer is restaged two sub-slices later
    if (sub + 1 < nsub) {
      cur0 = nxt0;
      cur1 = nxt1;
    }
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
  const unsigned grid = static_cast<unsigned>((N + 16 * GV_WARPS - 1) / (16 * GV_WARPS));
  k_gemv<<<grid, GV_WARPS * 32, 0, st>>>(X, int(M), codes, absmax_q, dq_scale, int(N), int(K), Hs, B, r,
                                          host_codebook().levels, Y);
  return cudaGetLastError();
}

}  // namespace qn
