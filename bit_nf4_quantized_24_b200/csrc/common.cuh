// Device helpers for the sm_100a kernels: mbarrier, TMA, tcgen05 (TMEM + UMMA),
// bounded waits, and the NF4 register-table dequantization.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qn {

// The 16 NF4 levels, passed to kernels by value (they land in the constant
// bank and are read with compile-time indices only).
struct Nf4Levels {
  float v[16];
};
struct Nf4Mids {
  float v[15];
};

// Device status codes written to the per-device status word.
enum : int { kDevOk = 0, kDevTimeout = 1, kDevNonfinite = 2 };

// A bounded wait gives up after this long and records kDevTimeout.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ prmt

// prmt.b32 in its default mode: selector nibble bits [2:0] pick one of the 8
// source bytes (a = bytes 0..3, b = bytes 4..7); bit 3 set replicates that
// byte's sign bit over the whole output byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t lop_select(uint32_t a, uint32_t b, uint32_t m) {
  return (a & ~m) | (b & m);  // one lop3: bytes of b where m is set, else a
}

// ------------------------------------------------- NF4 register lookup table
//
// For one 64-element block with scale a', the 16 possible bf16 outputs
// T[c] = bf16_rn(fl32(L[c] * a')) are held as byte tables in 8 registers:
// lo[0..3] = low bytes of T[0..15] (4 per register), hi[0..3] = high bytes.
// A 4-bit code then costs a fraction of a prmt: the low 3 bits select a byte
// within a half table, bit 3 selects the half.  The result equals the
// arithmetic definition bit for bit.
struct Nf4Lut {
  uint32_t lo0, lo1, lo2, lo3, hi0, hi1, hi2, hi3;
};

__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ Nf4Lut make_lut(const Nf4Levels& L, float ap) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) p[i] = bf16x2_bits(__fmul_rn(L.v[2 * i], ap), __fmul_rn(L.v[2 * i + 1], ap));
  Nf4Lut t;
  t.lo0 = prmt(p[0], p[1], 0x6420);
  t.hi0 = prmt(p[0], p[1], 0x7531);
  t.lo1 = prmt(p[2], p[3], 0x6420);
  t.hi1 = prmt(p[2], p[3], 0x7531);
  t.lo2 = prmt(p[4], p[5], 0x6420);
  t.hi2 = prmt(p[4], p[5], 0x7531);
  t.lo3 = prmt(p[6], p[7], 0x6420);
  t.hi3 = prmt(p[6], p[7], 0x7531);
  return t;
}

// Dequantize 8 codes (one 32-bit word: code i in nibble i, i.e. element 2j in
// the low nibble of byte j) into 8 bf16 values packed as 4 words, element
// order preserved: o0 = {e0, e1}, o1 = {e2, e3}, o2 = {e4, e5}, o3 = {e6, e7}.
__device__ __forceinline__ void deq8(uint32_t w, const Nf4Lut& t, uint32_t& o0, uint32_t& o1,
                                     uint32_t& o2, uint32_t& o3) {
  const uint32_t w4 = w << 4;
  // byte i = 0xff when code i (0..3) / code 4+i has bit 3 set (sign-replicate
  // mode: code 2i's bit 3 sits in the top bit of byte i of w << 4, code 2i+1's
  // in the top bit of byte i of w).
  const uint32_t m_lo = prmt(w4, w, 0xD9C8);
  const uint32_t m_hi = prmt(w4, w, 0xFBEA);
  const uint32_t s = w & 0x77777777u;
  const uint32_t s_hi = s >> 16;
  {
    const uint32_t la = prmt(t.lo0, t.lo1, s), lb = prmt(t.lo2, t.lo3, s);
    const uint32_t ha = prmt(t.hi0, t.hi1, s), hb = prmt(t.hi2, t.hi3, s);
    const uint32_t lo = lop_select(la, lb, m_lo), hi = lop_select(ha, hb, m_lo);
    o0 = prmt(lo, hi, 0x5140);
    o1 = prmt(lo, hi, 0x7362);
  }
  {
    const uint32_t la = prmt(t.lo0, t.lo1, s_hi), lb = prmt(t.lo2, t.lo3, s_hi);
    const uint32_t ha = prmt(t.hi0, t.hi1, s_hi), hb = prmt(t.hi2, t.hi3, s_hi);
    const uint32_t lo = lop_select(la, lb, m_hi), hi = lop_select(ha, hb, m_hi);
    o2 = prmt(lo, hi, 0x5140);
    o3 = prmt(lo, hi, 0x7362);
  }
}

// ------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `bar` with the given parity to complete.  Gives up
// when another thread of the CTA has already given up (*abort != 0) or after
// limit_ns (default kWaitLimitNs), in which case it sets *abort and the device
// status word.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                             int* status, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort = 1;
        atomicExch(status, kDevTimeout);
        return false;
      }
    }
  }
}

// Waits until the shared-memory counter at `addr` (a count that only grows,
// e.g. the number of times a buffer was released) reaches `target`, with the
// bounds of wait_bounded.  Unlike an mbarrier phase parity, a count cannot be
// mistaken for one two uses older, so a waiter may run any number of uses
// ahead.  Orders the caller's later memory accesses after the observation.
__device__ __forceinline__ int ld_volatile_shared(uint32_t addr) {
  int v;
  asm volatile("ld.volatile.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ bool wait_count_bounded(uint32_t addr, int target, volatile int* abort, int* status,
                                                   uint64_t limit_ns = kWaitLimitNs) {
  if (ld_volatile_shared(addr) < target) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
      if (ld_volatile_shared(addr) >= target) break;
      if ((n & 63u) == 0) {
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
          *abort = 1;
          atomicExch(status, kDevTimeout);
          return false;
        }
      }
    }
  }
  __threadfence_block();
  return true;
}
// Publishes a new count (after the caller's earlier memory accesses).
__device__ __forceinline__ void set_count(uint32_t addr, int value) {
  __threadfence_block();
  asm volatile("st.volatile.shared.s32 [%0], %1;" ::"r"(addr), "r"(value) : "memory");
}

// The same wait with cluster-scope acquire, for barriers that also receive
// arrivals from the peer CTA of a pair.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool wait_bounded_cluster(uint32_t bar, uint32_t parity, volatile int* abort,
                                                     int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((n & 63u) == 0) {
      if (*abort) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicExch(status, kDevTimeout);
        return false;
      }
    }
  }
}

// ------------------------------------------------------------- clusters

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Arrive (release, cluster scope) on an mbarrier given by a shared::cluster address.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A short bounded wait used while cleaning up after an abort.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > 200000000ull) return;
  }
}

// ------------------------------------------------ programmatic dependent launch
//
// pdl_trigger lets the next kernel of the stream begin launching once every
// CTA of this grid has called it (or exited).  pdl_wait blocks the calling
// thread until the previous kernel of the stream has completed and its writes
// are visible; it returns at once when this kernel was launched without the
// programmatic-serialization attribute.  Every kernel that is launched with the
// attribute calls pdl_wait (at least in one thread of each CTA) before it
// reads or overwrites anything an earlier kernel of the layer touches, and
// before it exits, so that its completion implies that of all earlier kernels.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// -------------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled load global -> shared, completion signalled on `bar` (tx bytes).
// x is the innermost coordinate in elements; x * elem_size must be a
// multiple of 16 bytes (every caller passes multiples of 32 bytes).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------- tcgen05 / TMEM

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Pair (cta_group::2) forms: TMEM is allocated in both CTAs of the pair, the
// leader issues MMAs that read both CTAs' shared memory and write both CTAs'
// TMEM, and completion is signalled to the same barrier offset in both CTAs.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(
          bar)
      : "memory");
}
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile
// (start address, leading/stride byte offsets, version 1, SWIZZLE_128B).
//  K-major:  rows of 128 B (64 bf16 along K), 8-row atoms of 1024 B;
//            SBO = 1024 (atom stride along M/N), LBO unused (16).
//  MN-major: rows of 128 B (64 bf16 along M/N) indexed by K, 8-row atoms;
//            LBO = stride between 64-element M/N atoms, SBO = 1024 (8 K rows).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// 32 lanes x 32 columns of 32-bit TMEM data into 32 registers per thread
// (thread i of the warp gets lane base+i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------ misc memory

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace qn
