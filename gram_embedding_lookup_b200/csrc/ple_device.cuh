// Device-side building blocks for libple on sm_100a: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM allocation, MMA issue, commit, loads),
// the shared-memory matrix descriptor for K-major SWIZZLE_128B tiles and the
// instruction descriptor of tcgen05.mma kind::f16.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "ple.h"

namespace ple {

// Sticky device status: the first error wins.
__device__ __forceinline__ void set_status(int32_t* status, int32_t code) {
  atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ per-token metadata
// Written by the prepare kernel, read by the epilogues.
struct __align__(16) TokMeta {
  float g;        // sigmoid(w_gate . h_t)
  int32_t seq;    // sequence index
  int32_t pos;    // position inside the sequence (-1: no token)
  int32_t flags;  // kFlagLast: last token of its sequence
};
constexpr int32_t kFlagLast = 1;

// ------------------------------------------------------------------ programmatic dependent launch
// launch_dependents lets the next kernel in the stream (launched with
// programmatic stream serialization) start once every CTA of this grid has
// issued it; wait blocks until the previous grid has completed and its memory
// is visible. Data the previous kernel writes is read only after the wait.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ smem address helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Bounded waits: about one second of SM clock at B200 frequencies.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// The same test with cluster-scope acquire: for barriers on which threads of
// the peer CTA of a pair arrive with release at cluster scope.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete. Returns false if the
// wait ran out after `limit` SM cycles (the caller records PLE_ERR_TIMEOUT and
// abandons its work).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit = kWaitLimitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long start = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - start > limit) return false;
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Adds `bytes` to the transaction count of the barrier's current phase, with no
// arrival: a later mbar_arrive by the same thread completes its part.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled load global -> shared, completion counted on `bar` (bytes).
// x is the innermost coordinate (elements), y the row. One destination CTA.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// 2-D tiled store shared -> global (bulk-group completion). Rows or columns
// outside the tensor are not written. The start coordinates must not be negative.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until at most N of this thread's bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
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

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp gets lane (base + i).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major operand stored as 128-byte rows
// (64 fp16 of K) with the 128-byte swizzle, 8-row groups 1024 bytes apart
// (the layout a TMA load with CU_TENSOR_MAP_SWIZZLE_128B produces).
//   bits  0-13 start address >> 4      bits 16-29 leading byte offset >> 4 (1, unused)
//   bits 32-45 stride byte offset >> 4 bits 46-47 descriptor version (1 on sm_100)
//   bits 61-63 layout: 2 = SWIZZLE_128B
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------ CTA pairs (clusters of 2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
  return out;
}

// Arrive on an mbarrier given by a shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// The same arrive with the default (CTA-scope) release: for a producer whose
// data sits in its own CTA's shared memory and is read there by the pair's
// tensor core, once a proxy fence has made it visible to the async proxy. The
// cluster-scope release above costs about a third of a microsecond per use.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// All threads of both CTAs of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Tiled load into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in the peer CTA of the pair (shared::cluster address).
// One destination CTA.
// A 3-D box {x, y, z} into this CTA's shared memory, completion on its barrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

// The same for a 3-D box {x, y, z}: the projection's K-major operands as
// {64 elements, rows, K-blocks}, two K-blocks per copy.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 int32_t z, uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster)
      : "memory");
}

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

// Pair MMA issued by the even CTA: A rows [0, M/2) and B rows [0, N/2) come from
// its shared memory, the other halves from the same offsets in the odd CTA;
// each CTA's TMEM receives its M/2 rows of D.
__device__ __forceinline__ void mma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at `bar_cluster` (either CTA of the pair) when the
// pair MMAs issued so far complete.
__device__ __forceinline__ void mma_commit_pair(uint32_t bar_cluster) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
               : "memory");
}

// ------------------------------------------------------------------ asynchronous copies global -> shared
// (non-bulk cp.async: generic proxy, no registers held; completion tracked by an mbarrier)
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier receives one arrive when every cp.async this thread issued so far
// has completed; the arrive is part of the barrier's expected count.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// ------------------------------------------------------------------ shared-memory loads and stores
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ float2 ld_shared_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ------------------------------------------------------------------ named barriers
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// The same barrier, returning whether pred held for any of the threads: a
// decision every thread of the group then takes alike.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------ E4M3 dequantisation
// e = fp16(a * s0 + b * s1) for 16 codes of two table rows (a, b): each code is
// decoded exactly (E4M3 -> fp16 -> fp32 conversions; NaN codes stay NaN), the
// sum is fmaf(a, s0, b * s1) in fp32, rounded to nearest even. Every kernel of
// the library dequantises through this function.
__device__ __forceinline__ float2 e4m3x2_cvt(uint32_t two_codes) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two_codes & 0xFFFFu),
                                                     __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&hr));
}

__device__ __forceinline__ uint32_t deq2(uint32_t wa, uint32_t wb, int shift, float s0, float s1) {
  const float2 a = e4m3x2_cvt(wa >> shift);
  const float2 b = e4m3x2_cvt(wb >> shift);
  const __half2 r = __floats2half2_rn(fmaf(a.x, s0, b.x * s1), fmaf(a.y, s0, b.y * s1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// o0 = outputs of codes 0..7 (words a.x, a.y), o1 = codes 8..15.
__device__ __forceinline__ void deq16(const uint4& a, const uint4& b, float s0, float s1, uint4& o0, uint4& o1) {
  o0.x = deq2(a.x, b.x, 0, s0, s1);
  o0.y = deq2(a.x, b.x, 16, s0, s1);
  o0.z = deq2(a.y, b.y, 0, s0, s1);
  o0.w = deq2(a.y, b.y, 16, s0, s1);
  o1.x = deq2(a.z, b.z, 0, s0, s1);
  o1.y = deq2(a.z, b.z, 16, s0, s1);
  o1.z = deq2(a.w, b.w, 0, s0, s1);
  o1.w = deq2(a.w, b.w, 16, s0, s1);
}

// One row on its own (the multi-head layout): e = fp16(a * s) for 16 codes,
// the product in fp32, rounded to nearest even.
__device__ __forceinline__ uint32_t deq2_one(uint32_t wa, int shift, float s) {
  const float2 a = e4m3x2_cvt(wa >> shift);
  const __half2 r = __floats2half2_rn(a.x * s, a.y * s);
  return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ void deq16_one(const uint4& a, float s, uint4& o0, uint4& o1) {
  o0.x = deq2_one(a.x, 0, s);
  o0.y = deq2_one(a.x, 16, s);
  o0.z = deq2_one(a.y, 0, s);
  o0.w = deq2_one(a.y, 16, s);
  o1.x = deq2_one(a.z, 0, s);
  o1.y = deq2_one(a.z, 16, s);
  o1.z = deq2_one(a.w, 0, s);
  o1.w = deq2_one(a.w, 16, s);
}

// NVFP4 rows: e = fp16(a' * s0 + b' * s1) for 16 elements of two rows, where a'
// is an FP4 E2M1 code times its block's E4M3 scale. Codes come two per byte,
// the low nibble first (8 bytes per 16 elements); one block scale covers the
// 16. The product of an E2M1 value (at most 2 significant bits, magnitude
// 0.5 .. 6) and an E4M3 value (4 bits, 2^-9 .. 448) has at most 6 significant
// bits and lies in [2^-10, 2688], so it is exact in fp16. Then fmaf in fp32
// and RNE to fp16 as for FP8 rows. NaN block scales stay NaN.
__device__ __forceinline__ __half2 e2m1x2_cvt(uint32_t byte) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(r) : "r"(byte & 0xFFu));
  return *reinterpret_cast<const __half2*>(&r);
}

__device__ __forceinline__ uint32_t deq2_nv(uint32_t wa, uint32_t wb, int shift, __half2 ba, __half2 bb, float s0,
                                            float s1) {
  const float2 a = __half22float2(__hmul2(e2m1x2_cvt(wa >> shift), ba));
  const float2 b = __half22float2(__hmul2(e2m1x2_cvt(wb >> shift), bb));
  const __half2 r = __floats2half2_rn(fmaf(a.x, s0, b.x * s1), fmaf(a.y, s0, b.y * s1));
  return *reinterpret_cast<const uint32_t*>(&r);
}

// ca, cb: the 8 code bytes of each row (16 elements); bsa, bsb: the block-scale bytes.
__device__ __forceinline__ void deq16_nv(const uint2& ca, const uint2& cb, uint32_t bsa, uint32_t bsb, float s0,
                                         float s1, uint4& o0, uint4& o1) {
  const float2 bs = e4m3x2_cvt((bsa & 0xFFu) | ((bsb & 0xFFu) << 8));
  const __half2 ba = __float2half2_rn(bs.x);          // exact: an E4M3 value is an fp16 value
  const __half2 bb = __float2half2_rn(bs.y);
  o0.x = deq2_nv(ca.x, cb.x, 0, ba, bb, s0, s1);
  o0.y = deq2_nv(ca.x, cb.x, 8, ba, bb, s0, s1);
  o0.z = deq2_nv(ca.x, cb.x, 16, ba, bb, s0, s1);
  o0.w = deq2_nv(ca.x, cb.x, 24, ba, bb, s0, s1);
  o1.x = deq2_nv(ca.y, cb.y, 0, ba, bb, s0, s1);
  o1.y = deq2_nv(ca.y, cb.y, 8, ba, bb, s0, s1);
  o1.z = deq2_nv(ca.y, cb.y, 16, ba, bb, s0, s1);
  o1.w = deq2_nv(ca.y, cb.y, 24, ba, bb, s0, s1);
}

// ------------------------------------------------------------------ table row chunks
// Streaming loads of data read once (no L1 allocation).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream_u16(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_stream_u8(const void* p) {
  uint16_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u8 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// One 16-element chunk of a table row: E4M3 codes (16 bytes), or NVFP4 codes
// (8 bytes) and the chunk's block-scale byte.
template <bool NV> struct RowChunk;
template <> struct RowChunk<false> { uint4 c; };
template <> struct RowChunk<true> { uint2 c; uint32_t b; };

// Chunk j (16 elements) of global row `row` (sub-table offset already added):
// codes at row * cs, block scales at row * bs, both strides in bytes. E4M3:
// cs = D. NVFP4 in separate arrays: cs = D/2, bs = D/16; NVFP4 rows (codes and
// block scales side by side, blocks = codes + D/2): cs = bs = 9D/16.
template <bool NV>
__device__ __forceinline__ RowChunk<NV> load_chunk(const uint8_t* codes, const uint8_t* blocks, int64_t row,
                                                   int32_t cs, int32_t bs, int j) {
  RowChunk<NV> r;
  if constexpr (NV) {
    r.c = ld_stream_v2(codes + row * cs + 8 * j);
    r.b = ld_stream_u8(blocks + row * bs + j);
  } else {
    (void)blocks;
    (void)bs;
    r.c = ld_stream_v4(codes + row * cs + 16 * j);
  }
  return r;
}

template <bool NV>
__device__ __forceinline__ void deq_chunk(const RowChunk<NV>& a, const RowChunk<NV>& b, float s0, float s1,
                                          uint4& o0, uint4& o1) {
  if constexpr (NV) deq16_nv(a.c, b.c, a.b, b.b, s0, s1, o0, o1);
  else deq16(a.c, b.c, s0, s1, o0, o1);
}

// ------------------------------------------------------------------ the gate
constexpr int kEmbedH4 = 10;    // uint4 of h per lane held in registers (hidden <= 2560)

// g = sigmoid(w_gate . h_t) for one token, by one warp, in fp32: lane l adds
// up the 8-element groups j = l, l + 32, l + 64, ... in that order (the first
// kEmbedH4 of them already loaded into hv), then a butterfly reduction across
// the lanes. Every kernel that computes a gate (prefill embed, gate, decode)
// goes through these functions, which all take the sums in this order, so all
// paths give the same bits for a token.
__device__ __forceinline__ void gate_dot8(float& acc, const uint4& hq, const uint4& wq) {
  const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hq);
  const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&wq);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 hf = __bfloat1622float2(h2[q]);
    const float2 wf = __bfloat1622float2(w2[q]);
    acc = fmaf(hf.x, wf.x, acc);
    acc = fmaf(hf.y, wf.y, acc);
  }
}

__device__ __forceinline__ float gate_finish(float acc) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return 1.0f / (1.0f + expf(-acc));
}

__device__ __forceinline__ float gate_warp(const uint4 (&hv)[kEmbedH4], const uint4* hrow, const uint4* wg, int H8,
                                           int lane) {
  float acc = 0.f;
#pragma unroll
  for (int r = 0; r < kEmbedH4; ++r) {
    const int j = lane + 32 * r;
    if (j < H8) gate_dot8(acc, hv[r], __ldg(wg + j));
  }
  for (int j = lane + 32 * kEmbedH4; j < H8; j += 32) gate_dot8(acc, ld_stream_v4(hrow + j), __ldg(wg + j));
  return gate_finish(acc);
}

// The same gate with the first kEmbedH4 groups of w_gate loaded as well (wv):
// a caller can load the weights before it waits for the previous kernel.
__device__ __forceinline__ float gate_warp_pre(const uint4 (&hv)[kEmbedH4], const uint4 (&wv)[kEmbedH4],
                                               const uint4* hrow, const uint4* wg, int H8, int lane) {
  float acc = 0.f;
#pragma unroll
  for (int r = 0; r < kEmbedH4; ++r) {
    const int j = lane + 32 * r;
    if (j < H8) gate_dot8(acc, hv[r], wv[r]);
  }
  for (int j = lane + 32 * kEmbedH4; j < H8; j += 32) gate_dot8(acc, ld_stream_v4(hrow + j), __ldg(wg + j));
  return gate_finish(acc);
}

// The same gate with the row loaded in two halves of kEmbedH4 / 2 (fewer
// registers held at once); the sums are taken in the same order.
__device__ __forceinline__ float gate_warp_halves(const uint4* hrow, const uint4* wg, int H8, int lane) {
  constexpr int kHalf = kEmbedH4 / 2;
  float acc = 0.f;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint4 hv[kHalf];
#pragma unroll
    for (int r = 0; r < kHalf; ++r) {
      const int j = lane + 32 * (half * kHalf + r);
      if (j < H8) hv[r] = ld_stream_v4(hrow + j);
    }
#pragma unroll
    for (int r = 0; r < kHalf; ++r) {
      const int j = lane + 32 * (half * kHalf + r);
      if (j < H8) gate_dot8(acc, hv[r], __ldg(wg + j));
    }
  }
  for (int j = lane + 32 * kEmbedH4; j < H8; j += 32) gate_dot8(acc, ld_stream_v4(hrow + j), __ldg(wg + j));
  return gate_finish(acc);
}

// The gate of token row hrow (H8 = hidden / 8 groups of 8), loads included.
__device__ __forceinline__ float gate_warp_row(const uint4* hrow, const uint4* wg, int H8, int lane) {
  uint4 hv[kEmbedH4];
#pragma unroll
  for (int r = 0; r < kEmbedH4; ++r) {
    const int j = lane + 32 * r;
    if (j < H8) hv[r] = ld_stream_v4(hrow + j);
  }
  return gate_warp(hv, hrow, wg, H8, lane);
}

// ------------------------------------------------------------------ L2 prefetch
// Asks for `bytes` (a multiple of 16, 16-byte aligned address) to be brought
// into L2; no completion is tracked.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
               : "memory");
}

// ------------------------------------------------------------------ bulk copies shared -> global
// One contiguous copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned) in the calling thread's current bulk group.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}

// Orders this thread's global accesses in the async proxy (bulk copies) with
// its generic ones, both ways.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ------------------------------------------------------------------ bulk copies global -> shared
// One contiguous copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

}  // namespace ple
