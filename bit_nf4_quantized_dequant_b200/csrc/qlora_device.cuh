// Device-side building blocks for sm_100a: mbarriers with bounded waits, TMA
// tile loads, tcgen05 (UMMA + TMEM) wrappers, UMMA descriptors, and the NF4
// block-table expansion used by every kernel that dequantises.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "qlora_internal.h"

namespace qlora {

// ---------------------------------------------------------------------------
// NF4 levels (float32, ascending). Normal quantiles: 8 positive at
// probabilities 1/2 + (o - 1/2) j / 8 (j = 1..8), 7 negative at
// 1/2 + (o - 1/2) j / 7 (j = 1..7), an exact zero, all divided by Phi^{-1}(o),
// with o = 1 - (1/32 + 1/30) / 2 ("QLoRA and Fine-Tuning on One Consumer GPU",
// "NF4 and double quantisation": sixteen levels at normal quantiles).
// ---------------------------------------------------------------------------
#define QLORA_NF4_LEVELS                                                     \
  {-0x1.000000p+0f, -0x1.647362p-1f, -0x1.0cd65cp-1f, -0x1.94653cp-2f,       \
   -0x1.234496p-2f, -0x1.7a6a7ap-3f, -0x1.74f0d2p-4f, 0x0.0p+0f,             \
   0x1.45f602p-4f,  0x1.4995bep-3f,  0x1.f809b4p-3f,  0x1.5a066cp-2f,        \
   0x1.c3496ap-2f,  0x1.200f52p-1f,  0x1.722760p-1f,  0x1.000000p+0f}

// Comparison codebook: evenly spaced int4 levels (k - 8) / 7, k = 0..15, as
// float32 ("What is QLoRA ...", "Follow-up questions to expect": plain int4
// spaces its levels evenly and wastes them on rare large values). The same
// block constants and 8-bit double quantisation apply; code 8 is zero and
// level 0 (-8/7) is never chosen, since |w / c1| <= 1.
#define QLORA_INT4_LEVELS                                                    \
  {-0x1.24924ap+0f, -0x1.000000p+0f, -0x1.b6db6ep-1f, -0x1.6db6dcp-1f,       \
   -0x1.24924ap-1f, -0x1.b6db6ep-2f, -0x1.24924ap-2f, -0x1.24924ap-3f,       \
   0x0.0p+0f,       0x1.24924ap-3f,  0x1.24924ap-2f,  0x1.b6db6ep-2f,        \
   0x1.24924ap-1f,  0x1.6db6dcp-1f,  0x1.b6db6ep-1f,  0x1.000000p+0f}

// Codebook identifiers (the values of qlora_codebook_t).
constexpr int kBookNf4 = 0;
constexpr int kBookInt4 = 1;

// ---------------------------------------------------------------------------
// Small PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Record the first device-side error of a call (never clears an earlier one).
__device__ __forceinline__ void set_status(int32_t *status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// ---- mbarrier -------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

// Brings a tensor-map descriptor (a kernel parameter) into the cache of
// descriptors ahead of its first copy.
__device__ __forceinline__ void prefetch_tensormap(const void *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Adds `bytes` to the transaction count of the current phase without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended (not spinning, so it
// takes no issue slots from the other warps) until the phase completes or
// about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// A wait on one phase of an mbarrier that gives up after kWaitLimitNs: it then
// raises the CTA's abort flag and the call's TIMEOUT status and returns false.
// Every waiter also polls the abort flag so that one timed-out role brings the
// whole CTA down instead of leaving the others spinning.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

constexpr uint32_t kSuspendHintNs = 100000;                     // 100 us per suspended try

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendHintNs)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      set_status(status, 6 /* QLORA_ERR_TIMEOUT */);
      return false;
    }
  }
}

// ---- TMA ------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load of the box at element coordinates (x inner, y outer) into
// shared memory; completion is counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// As tma_load_2d, with an L2 cache policy (from l2_evict_first_policy).
__device__ __forceinline__ void tma_load_2d_hint(void *smem_dst, const CUtensorMap *map, uint64_t *bar,
                                                 int32_t x, int32_t y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// L2 policy for data read once: its lines are the first to be replaced.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// 3-D tiled load of the box at element coordinates (x, y, z).
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                            int32_t y, int32_t z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 2-D tiled store of a shared-memory box to global memory (elements outside
// the tensor are not written). Completion is tracked by bulk groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *smem_src, int32_t x,
                                             int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups are still reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Untiled bulk copy shared -> global of `bytes` (multiple of 16, both
// addresses 16-byte aligned), tracked by bulk groups.
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (multiple of 16, both addresses
// 16-byte aligned) that completes transaction bytes on an mbarrier of this CTA.
__device__ __forceinline__ void bulk_load(void *sdst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(sdst)),
               "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Orders this thread's completed async-proxy (bulk copy) writes to global
// memory before its later generic-proxy accesses, such as a release store.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Barrier over a subset of the CTA's warps (id 1..15, count a multiple of 32).
// bar.sync is an aligned barrier: every lane of a warp must arrive together,
// so the warp is reconverged first (lanes may come from a single-lane branch).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Atomic add at GPU scope that releases this thread's earlier writes (and
// those ordered before it by a barrier) and acquires the writes released by
// earlier adds to the same word; returns the old value.
__device__ __forceinline__ unsigned long long atom_add_acq_rel_gpu(unsigned long long *p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

// Flag publication between CTAs of one grid (global memory, GPU scope).
__device__ __forceinline__ void st_release_gpu_u64(uint64_t *p, uint64_t v) {
  asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_acquire_gpu_u64(const uint64_t *p) {
  uint64_t v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Generic-proxy shared-memory writes -> visible to the async proxy (tcgen05).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- clusters / distributed shared memory ----------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster (release / acquire). The barrier is
// aligned, so each warp is reconverged before it arrives.
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// ---- CTA pairs (cta_group::2) ----------------------------------------------
// Arrive once on an mbarrier of another CTA of the cluster (shared::cluster
// address from mapa_shared).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 2-D tiled load into this CTA's shared memory whose completion bytes are
// counted on an mbarrier of the pair's even CTA (`bar_cluster_addr`).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *map, uint32_t bar_cluster_addr,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (both CTAs' TMEM) (+)= A (both CTAs' smem, split by M) * B (both CTAs'
// smem, split by N)^T; issued by one thread of the even CTA.
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on the mbarrier at the same shared-memory offset in both CTAs of the
// pair once the pair's tcgen05 ops issued so far are done.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// ---- warp-level matrix fragments ------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Byte offset inside a TMA-swizzled tile (rows of `span` = 32, 64 or 128 bytes,
// tile aligned to the swizzle atom): the 16-byte chunk index is XORed with the
// row bits above it.
__device__ __forceinline__ uint32_t swizzle_off(uint32_t off, uint32_t span) {
  return off ^ (((off >> 7) & ((span >> 4) - 1u)) << 4);
}

// ---- tcgen05 ----------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- UMMA descriptors ---------------------------------------------------------
// Shared-memory matrix descriptor (sm_100 format, version 1): start address,
// leading- and stride-dimension byte offsets (all >> 4), swizzle layout code.
enum : uint32_t { kLayoutNone = 0, kLayoutSW128 = 2, kLayoutSW64 = 4, kLayoutSW32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor: kind::f16 with bf16 A and B, fp32 D, shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, bool a_mn_major,
                                                  bool b_mn_major) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | ((a_mn_major ? 1u : 0u) << 15) // A major
         | ((b_mn_major ? 1u : 0u) << 16) // B major
         | ((N >> 3) << 17)               // N / 8
         | ((M >> 4) << 24);              // M / 16
}

// ---------------------------------------------------------------------------
// NF4 block tables
//
// For one block with scale s, the 16 dequantised values are
// T[c] = bf16_rn(fp32_rn(level[c] * s)). They are held as two byte planes of
// four 32-bit registers each: lo[i] holds the low bytes of T[4i..4i+3], hi[i]
// the high bytes. A code nibble then selects its bytes with PRMT.
// ---------------------------------------------------------------------------
struct Nf4Table {
  uint32_t lo[4];
  uint32_t hi[4];
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

template <uint32_t LUT>
__device__ __forceinline__ uint32_t lop3(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
  return d;
}

// Two fp32 values -> packed bf16x2 (round to nearest even): low half = lo.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Block scale s = fp32_rn(q8 * d): the product is rounded once.
__device__ __forceinline__ float block_scale(uint32_t q8, float d) {
  return __fmul_rn(static_cast<float>(q8), d);
}

__device__ __forceinline__ Nf4Table table_from_levels(const float (&L)[16], float s) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__fmul_rn(L[2 * i], s), __fmul_rn(L[2 * i + 1], s));
  Nf4Table t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // pk[2i] bytes: lo(T4i) hi(T4i) lo(T4i+1) hi(T4i+1); pk[2i+1]: same for T4i+2, T4i+3
    t.lo[i] = prmt(pk[2 * i], pk[2 * i + 1], 0x6420u);
    t.hi[i] = prmt(pk[2 * i], pk[2 * i + 1], 0x7531u);
  }
  return t;
}

template <int BOOK>
__device__ __forceinline__ Nf4Table make_table_book(float s) {
  if constexpr (BOOK == kBookInt4) {
    constexpr float L[16] = QLORA_INT4_LEVELS;
    return table_from_levels(L, s);
  } else {
    constexpr float L[16] = QLORA_NF4_LEVELS;
    return table_from_levels(L, s);
  }
}

__device__ __forceinline__ Nf4Table make_table(float s) { return make_table_book<kBookNf4>(s); }

// Expand one 32-bit word of packed codes (8 weights, element 2j in the high
// nibble of byte j) into 8 bf16 values, returned as 4 words of bf16 pairs in
// element order (word 0 = elements 0 and 1, element 0 in the low half).
__device__ __forceinline__ void expand8(const Nf4Table &t, uint32_t w, uint32_t (&out)[4]) {
  // Nibble k of w (bits 4k..4k+3) holds element k^1. PRMT reads 4 selector
  // nibbles; bit 3 of a selector means "replicate sign", so selectors are
  // masked to 3 bits and the upper half of the codebook is chosen with a mask.
  const uint32_t sel = w & 0x77777777u;
  const uint32_t sel_hi = sel >> 16;
  const uint32_t w4 = w << 4;
  // 0xFF in byte k when bit 3 of nibble k is set (the sign bit of the byte that
  // holds it, taken from w for odd nibbles and from w << 4 for even ones).
  const uint32_t m_lo = prmt(w, w4, 0x9D8Cu);
  const uint32_t m_hi = prmt(w, w4, 0xBFAEu);
  // bytes for nibbles 0..3 (elements 1, 0, 3, 2) and 4..7 (elements 5, 4, 7, 6)
  const uint32_t lo_a = lop3<0xD8>(prmt(t.lo[0], t.lo[1], sel), prmt(t.lo[2], t.lo[3], sel), m_lo);
  const uint32_t hi_a = lop3<0xD8>(prmt(t.hi[0], t.hi[1], sel), prmt(t.hi[2], t.hi[3], sel), m_lo);
  const uint32_t lo_b =
      lop3<0xD8>(prmt(t.lo[0], t.lo[1], sel_hi), prmt(t.lo[2], t.lo[3], sel_hi), m_hi);
  const uint32_t hi_b =
      lop3<0xD8>(prmt(t.hi[0], t.hi[1], sel_hi), prmt(t.hi[2], t.hi[3], sel_hi), m_hi);
  // interleave low and high bytes into bf16 pairs in element order
  out[0] = prmt(lo_a, hi_a, 0x4051u);
  out[1] = prmt(lo_a, hi_a, 0x6273u);
  out[2] = prmt(lo_b, hi_b, 0x4051u);
  out[3] = prmt(lo_b, hi_b, 0x6273u);
}

}  // namespace qlora
