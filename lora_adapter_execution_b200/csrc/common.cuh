// Device helpers for sm_100a: bounded mbarrier waits, TMA, tcgen05 (UMMA + TMEM),
// shared-memory matrix descriptors, the SplitMix64 mask hash and the status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lora.h"

namespace lora {

// Per-device status word: kernels OR LORA_DEV_* bits into it instead of trapping.
__device__ uint32_t g_status;

// A wait that sees no progress for this long gives up, flags LORA_DEV_TIMEOUT and
// lets its kernel wind down. Legitimate waits inside one launch are microseconds.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ void flag_status(uint32_t bits) { atomicOr(&g_status, bits); }

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}


// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
// End an mbarrier object's life: no thread may wait on or arrive at it any more.
// The location may then hold a new barrier (mbarrier.init) or other data; a
// second init of a barrier that is still valid does not reset its phase.
__device__ __forceinline__ void mbar_inval(uint32_t bar) {
  asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase of `parity` to complete. Returns false (after flagging
// LORA_DEV_TIMEOUT) if it has not completed within `limit_ns`.
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) {
      flag_status(LORA_DEV_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  return mbar_wait_for(bar, parity, kWaitLimitNs);
}

// Wait until the global counter *cnt reaches `need` (an acquire load, so what the
// counting threads wrote before their release is visible). Returns false (after
// flagging LORA_DEV_TIMEOUT) if it has not within kWaitLimitNs.
__device__ __forceinline__ bool wait_counter(const int *cnt, int need) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
  if (v >= need) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    __nanosleep(64);
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    if (v >= need) return true;
    if (globaltimer() - t0 > kWaitLimitNs) {
      flag_status(LORA_DEV_TIMEOUT);
      return false;
    }
  }
}
// Add one to a global counter after every write this thread made, or saw
// through a barrier, before it (release at GPU scope).
__device__ __forceinline__ void signal_counter(int *cnt) {
  __threadfence();
  asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(cnt) : "memory");
}

// ------------------------------------------------------------------ programmatic dependent launch
// Let the next kernel on the stream (launched with programmatic serialization)
// start its prologue while this grid still runs.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the grids this one depends on have completed and their memory is
// visible (returns at once when the kernel was launched without the attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ TMA / bulk copies
// Bring a kernel-parameter tensor map into the TMA unit's descriptor cache
// before its first copy.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
// 3-D tile: coordinates innermost first (c0 is the 16-byte-aligned column inside a
// 64-column block, c1 the row, c2 the column block).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Contiguous copy from this CTA's shared memory into another CTA of the cluster
// (dst and bar are cluster addresses from mapa), completing on that CTA's
// mbarrier. 16-byte aligned addresses, size a multiple of 16.
__device__ __forceinline__ void bulk_s2s_cluster(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_cluster),
      "r"(src), "r"(bytes), "r"(bar_cluster)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk copy of this thread has finished reading its source.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Contiguous shared -> global copy (16-byte aligned addresses, size a multiple of
// 16), in this thread's current bulk group.
__device__ __forceinline__ void bulk_s2g(void *dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
// Wait until every committed bulk copy of this thread is complete (its writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Order global-memory accesses of the generic proxy against the async proxy.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Contiguous global -> shared copy (16-byte aligned addresses, size multiple of 16).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
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
// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate. Issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
// Same with accumulate = 1 (no predicate to compute).
__device__ __forceinline__ void umma_bf16_acc(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.eq.u32 p, 1, 1;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle.
//  K-major operand: rows of 128 B (64 bf16 of K), 8-row atoms `sbo` bytes apart;
//                   `lbo` unused (16). A K=16 step advances the start by 32 B.
//  MN-major operand: rows of 128 B (64 bf16 of M or N) per K index, 8-K-row atoms
//                   `sbo` bytes apart along K, 64-wide M/N blocks `lbo` bytes apart.
// Atoms must start on 1024-byte boundaries (base offset field 0).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D = f32
         | (1u << 7)                                 // A = bf16
         | (1u << 10)                                // B = bf16
         | ((a_mn_major ? 1u : 0u) << 15)            // A major
         | ((b_mn_major ? 1u : 0u) << 16)            // B major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Byte offset of element (row, col) inside a [rows x 64] bf16 tile stored with the
// 128-byte swizzle (row r at r*128; 16-byte chunk j of the row at chunk j ^ (r & 7)).
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col) {
  return row * 128u + ((((col >> 3) ^ (row & 7u)) & 7u) << 4) + ((col & 7u) << 1);
}

// ------------------------------------------------------------------ dropout mask hash
// SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) seeded with `seed`: output n
// (0-based) mixes the state z = seed + (n + 1) * 0x9E3779B97F4A7C15 (the state
// after n + 1 golden-ratio increments) with x ^= x >> 30, x *= 0xBF58476D1CE4E5B9,
// x ^= x >> 27, x *= 0x94D049BB133111EB, x ^= x >> 31. Element (t, col) of the
// LoRA-branch input is dropped when output t * d_in + col is below thr = p * 2^64.
//
// keep_state: whether the output of state z (the state after its increment) is
// >= thr, i.e. the element is kept. The comparison needs only the high word of the output unless
// it ties with the high word of thr (a 2^-32 event): the last product's low word
// and the last shift's low half are formed only then.
__device__ __forceinline__ bool keep_state(uint64_t z, uint64_t thr) {
  const uint64_t x = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  const uint64_t u = x ^ (x >> 27);
  constexpr uint64_t kM2 = 0x94D049BB133111EBull;
  const uint32_t ul = static_cast<uint32_t>(u), uh = static_cast<uint32_t>(u >> 32);
  const uint32_t ph = __umulhi(ul, static_cast<uint32_t>(kM2)) + ul * static_cast<uint32_t>(kM2 >> 32) +
                      uh * static_cast<uint32_t>(kM2);  // high word of u * kM2
  const uint32_t oh = ph ^ (ph >> 31);                   // high word of the output
  const uint32_t th = static_cast<uint32_t>(thr >> 32);
  if (oh != th) return oh > th;
  const uint64_t p = u * kM2;
  return (p ^ (p >> 31)) >= thr;
}
// true if element (t, col) of the LoRA-branch input is kept.
__device__ __forceinline__ bool keep_elem(uint64_t seed, uint64_t thr, int64_t t, int64_t col,
                                          int64_t d_in) {
  return thr == 0 || keep_state(seed + (static_cast<uint64_t>(t * d_in + col) + 1ull) * 0x9E3779B97F4A7C15ull, thr);
}

// Keep bits of 32 consecutive mask positions idx0 .. idx0+31 (bit i set if kept):
// the same SplitMix64 outputs as keep_elem, with the state advanced by one
// increment per position instead of recomputed.
__device__ __forceinline__ uint32_t keep_mask32(uint64_t seed, uint64_t thr, uint64_t idx0) {
  if (thr == 0) return 0xFFFFFFFFu;
  uint64_t z = seed + (idx0 + 1ull) * 0x9E3779B97F4A7C15ull;
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    m |= (keep_state(z, thr) ? 1u : 0u) << i;
    z += 0x9E3779B97F4A7C15ull;
  }
  return m;
}

// ------------------------------------------------------------------ bf16 packing
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

}  // namespace lora
