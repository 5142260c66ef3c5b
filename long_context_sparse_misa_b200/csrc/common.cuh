// Device helpers shared by the MISA kernels: status word, bounded mbarrier
// waits, TMA bulk-tensor loads and the tcgen05 (5th-generation tensor core)
// primitives, all as inline PTX for sm_100a.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/misa.h"

namespace misa {

// ~1 s at 2 GHz.  Every spin-wait in these kernels gives up after this many
// SM cycles, sets MISA_STATUS_TIMEOUT and unwinds instead of hanging.
constexpr long long kWaitCycles = 1ll << 31;
constexpr long long kDrainCycles = 1ll << 29;  // ~0.25 s

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  atomicOr(status, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity.  Gives up when the wait
// exceeds `limit` cycles or, unless `drain` is set, when another role of the
// CTA has already given up (*abort != 0); on giving up it raises *abort and
// the status bit and returns false.  Drains (waiting for this CTA's own
// copies or MMAs to land before it exits) ignore *abort but keep the limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint32_t* status, long long limit = kWaitCycles,
                                          bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (!drain && *abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      set_status(status, MISA_STATUS_TIMEOUT);
      return false;
    }
  }
}

// All 32 lanes wait together; the outcome is warp-uniform (so .sync.aligned
// tcgen05 instructions that follow are executed by the whole warp or by none).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int* abort,
                                          uint32_t* status, long long limit = kWaitCycles) {
  const int lane = threadIdx.x & 31;
  long long t0 = 0;
  if (lane == 0) t0 = clock64();
  while (true) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    int give_up = 0;
    if (lane == 0) {
      if (*reinterpret_cast<volatile int*>(abort)) {
        give_up = 1;
      } else if (clock64() - t0 > limit) {
        *reinterpret_cast<volatile int*>(abort) = 1;
        set_status(status, MISA_STATUS_TIMEOUT);
        give_up = 1;
      }
    }
    if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
  }
}

// ---------------------------------------------------------------- dependent launch
// First statement of a kernel that may be launched with programmatic
// dependent launch: wait until the previous kernel on the stream has
// completed and its writes are visible (returns at once when launched
// normally), then let the next kernel's CTAs be scheduled.  The next kernel
// waits in turn, so no kernel runs ahead of one that it may depend on.
__device__ __forceinline__ void pdl_wait_then_release() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk-tensor load into this CTA's shared memory, completion
// counted in bytes on `bar`.  x is the innermost (element) coordinate.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// ---------------------------------------------------------------- cp.async (gathers)
__device__ __forceinline__ void cp_async_16(void* dst_smem, const void* src, bool valid) {
  const uint32_t bytes = valid ? 16u : 0u;  // zero-fill when invalid
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst_smem)),
               "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                              // D format: F32
         | (1u << 7)                            // A format: BF16
         | (1u << 10)                           // B format: BF16
         | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte-swizzle canonical layout: rows of 128 B (64 bf16 along K), groups
// of 8 rows 1024 B apart, 1024-byte-aligned atoms.  Moving along K inside the
// 128-byte row is done by adding the byte offset to the start address.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);  // start address
  d |= static_cast<uint64_t>(1u) << 16;                      // leading byte offset (unused)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;              // stride byte offset: 8 rows
  d |= static_cast<uint64_t>(1u) << 46;                      // descriptor version (sm_100)
  d |= static_cast<uint64_t>(2u) << 61;                      // SWIZZLE_128B
  return d;
}

// 32 lanes x 32 consecutive fp32 columns of TMEM -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
// 16 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Ties 32 registers filled by tcgen05.ld to a point after tcgen05.wait::ld:
// the empty volatile asm is ordered after the wait, and every later use reads
// its outputs, so the compiler cannot hoist a use above the wait.
__device__ __forceinline__ void reg_fence32(float (&v)[32]) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31]));
}

__device__ __forceinline__ void reg_fence16(float (&v)[16]) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}

// Shared-memory reduction (no return value, shared-window address).
__device__ __forceinline__ void red_add_shared(uint32_t* p, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// Predicated memory operations: the access happens only where `pred` holds,
// without a branch (no divergence, no reconvergence barrier).  The address
// must be computable on every lane but is only dereferenced under `pred`.
__device__ __forceinline__ void red_add_shared_if(uint32_t* p, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t@q red.shared.add.u32 [%0], 1;\n\t}\n" ::"r"(
          smem_u32(p)),
      "r"((int)pred)
      : "memory");
}
__device__ __forceinline__ void red_add_shared_val_if(uint32_t* p, uint32_t v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q red.shared.add.u32 [%0], %1;\n\t}\n" ::"r"(
          smem_u32(p)),
      "r"(v), "r"((int)pred)
      : "memory");
}
__device__ __forceinline__ void st_global_u2_if(void* p, uint32_t x, uint32_t y, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %3, 0;\n\t@q st.global.v2.u32 [%0], {%1, %2};\n\t}\n" ::"l"(
          p),
      "r"(x), "r"(y), "r"((int)pred)
      : "memory");
}
__device__ __forceinline__ void st_global_u32_if(void* p, uint32_t x, bool pred) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %2, 0;\n\t@q st.global.u32 [%0], %1;\n\t}\n" ::"l"(p),
      "r"(x), "r"((int)pred)
      : "memory");
}

// a0 += w0 * r0 and a1 += w1 * r1 as one packed fp32 FMA (sm_100 f32x2).
__device__ __forceinline__ void ffma2(float& a0, float& a1, float w0, float w1, float r0,
                                      float r1) {
  uint64_t a, w, r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(w) : "f"(w0), "f"(w1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(r0), "f"(r1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(w), "l"(r));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(a));
}

// acc = {a0, a1} += {w0, w1} * {r0, r1} (one packed fp32 FMA; the weights
// come as a 64-bit pair and the accumulators stay packed between calls).
__device__ __forceinline__ void ffma2_acc(uint64_t& acc, uint64_t w, float r0, float r1) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(r0), "f"(r1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(w), "l"(r));
}

// a0 + a1 of a packed pair.
__device__ __forceinline__ float sum_pair(uint64_t acc) {
  float a0, a1;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
  return a0 + a1;
}

// ReLU that keeps a NaN (max.NaN): as in the oracle's arithmetic, a NaN in
// q, w or a key reaches the score it feeds (fmaxf would drop it for 0), so a
// NaN router score can be flagged and ranked last.
__device__ __forceinline__ float relu_nan(float x) {
  float r;
  asm("max.NaN.f32 %0, %1, 0f00000000;" : "=f"(r) : "f"(x));
  return r;
}

// Head-weighted ReLU sum of one query's MH accumulator columns, the one
// summation order every scoring kernel uses (so all paths agree bit for bit):
// even heads into a0, odd heads into a1 (one packed FMA per pair), then
// a0 + a1.  `col(j)` gives the accumulator value of head j, `wq` the head
// weights as stored by relu_weight (halved).  ReLU is formed as
// a + |a| = 2 max(a, 0), exactly, on the FMA pipe (the |a| is an operand
// modifier) rather than as max(a, 0) on the integer/logic pipe; with the
// halved weight each product (w/2)(2 max(a, 0)) equals w max(a, 0) exactly,
// so the sum is the same as with the plain form.
__device__ __forceinline__ float relu_weight(float w) { return 0.5f * w; }

template <int MH, typename ColFn>
__device__ __forceinline__ float relu_wsum(ColFn col, const float* wq) {
  float a0 = 0.f, a1 = 0.f;
  if constexpr (MH == 1) {
    const float c0 = col(0);
    a0 = fmaf(wq[0], c0 + fabsf(c0), a0);
  } else {
#pragma unroll
    for (int j = 0; j < MH; j += 2) {
      const float2 wj = *reinterpret_cast<const float2*>(wq + j);
      const float c0 = col(j), c1 = col(j + 1);
      ffma2(a0, a1, wj.x, wj.y, c0 + fabsf(c0), c1 + fabsf(c1));
    }
  }
  return a0 + a1;
}

// Inverse of order_key (for bin edges).
__device__ __forceinline__ float key_to_float(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// ---------------------------------------------------------------- ordering keys
// fp32 -> uint32 whose unsigned order is the numeric order; -0 maps like +0,
// NaN maps to 0 (below every number).
__device__ __forceinline__ uint32_t order_key(float x) {
  if (x != x) return 0u;
  uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Binary search: index s with off[s] <= x < off[s+1] (off non-decreasing, n+1 entries).
template <typename T>
__device__ __forceinline__ int upper_segment(const T* off, int n, T x) {
  int lo = 0, hi = n;  // invariant: off[lo] <= x, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

}  // namespace misa
