// tcgen05 (5th-generation tensor core) and tensor-map TMA helpers shared by
// the tensor-core kernels: the 128-byte-swizzled shared-memory layouts the MMA
// descriptors describe, the descriptors themselves, MMA issue and completion,
// tensor-memory allocation and read-back, and the tiled bulk tensor load
// (never with cluster multicast).
#pragma once

#include <cuda.h>  // CUtensorMap

#include "common.cuh"

namespace cta {

constexpr int kSwRowBytes = 128;  // one swizzle-atom row: 64 bf16
constexpr int kSwAtomBytes = 1024;  // 8 rows of 128 bytes

// Byte offset of 16-byte piece c of row r in a 128-byte-swizzled tile of
// `rows` rows: column atoms of rows x 128 B (piece c lies in atom c / 8), each
// made of 8-row groups of 1024 B in which piece c of row r sits at c ^ (r % 8).
// A K-major operand stores its M or N index as the row and K as the piece; an
// MN-major one stores K as the row and 8 consecutive M or N elements per piece.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c, int rows) {
  const int atom = c >> 3, cc = c & 7;
  return (uint32_t)(atom * rows * kSwRowBytes + (r >> 3) * kSwAtomBytes + (r & 7) * kSwRowBytes +
                    ((cc ^ (r & 7)) << 4));
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups
// 1024 B apart (stride byte offset), leading byte offset 16 (unused), version 1.
__device__ __forceinline__ unsigned long long desc_kmajor(uint32_t saddr) {
  return (unsigned long long)((saddr >> 4) & 0x3FFFu) | (1ull << 16) |
         ((unsigned long long)(kSwAtomBytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// MN-major, 128-byte swizzle: 8-deep K groups 1024 B apart (stride byte
// offset), 64-element MN blocks `lbo` bytes apart (leading byte offset).
__device__ __forceinline__ unsigned long long desc_mnmajor(uint32_t saddr, uint32_t lbo) {
  return (unsigned long long)((saddr >> 4) & 0x3FFFu) |
         ((unsigned long long)((lbo >> 4) & 0x3FFFu) << 16) |
         ((unsigned long long)(kSwAtomBytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: A and B bf16, D fp32, M x N; a_mn / b_mn
// select the MN-major (transposed) layout of that operand.
constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Generic-proxy writes to shared memory, made visible to the tensor cores and TMA.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A * B, issued by one thread.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, unsigned long long a, unsigned long long b,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on bar when every MMA this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (the warp reads the
// 32 lanes of its lane quarter).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Tensor-memory allocation by one whole warp; the base address lands in *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(slot)), "r"(cols) : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
               : "memory");
}

// Tiled 3-D tensor load global -> this CTA's shared memory (no multicast),
// completing on bar.  The innermost coordinate x times the element size must
// be a multiple of 16 bytes; dst is 1024-byte aligned for the 128-byte swizzle.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            unsigned long long* bar, unsigned long long policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(z),
        "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Named barrier over `count` threads that also ORs a predicate across them.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " barrier.cta.red.or.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0u;
}
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("barrier.cta.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

}  // namespace cta
