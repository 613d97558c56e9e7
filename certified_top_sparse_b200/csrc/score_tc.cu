// Phase 1 for the all-query case on the 5th-generation tensor cores:
// S = Q K^T for 128 query rows of one KV group at a time.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): the attention distribution of every
// query row is the softmax of its scores q.k_i / sqrt(d); this kernel writes
// the unscaled dot products u_i = q.k_i (the scale is folded into the weights).
//
// When every query of a head is a row (self-attention: m = n), QK^T is a dense
// contraction, so it runs as tcgen05.mma (bf16 x bf16 -> fp32): one CTA of 256
// threads per (KV group, 128-row tile); Q (128 x d) and each 256-key chunk of K
// (256 x d) are staged in shared memory in the 128-byte-swizzled K-major layout
// the MMA descriptors describe; the 128 x 256 fp32 product accumulates in 256
// tensor-memory columns; each row (TMEM lane) is read back by two threads, one
// per warpgroup and half of the columns, with tcgen05.ld and written to the
// logit buffer.  Exact products (bf16 x bf16
// fits fp32) accumulated in fp32, like the CUDA-core score kernel (the order
// of the d-term sum differs).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace cta {

namespace {

constexpr int kTcRows = 128;     // M: query rows per CTA (one per thread and TMEM lane)
constexpr int kTcN = 256;        // N: keys per MMA chunk (TMEM columns)
constexpr int kTcThreads = 256;  // two warpgroups: same TMEM lanes (rows), half the columns each

// Stages rows [0, rows) of a row-major [*, D] bf16 matrix into the swizzled tile.
template <int D>
__device__ __forceinline__ void stage_sw128(unsigned char* tile, const __nv_bfloat16* src, int rows) {
  constexpr int P = D / 8;  // 16-byte pieces per row
  for (int x = threadIdx.x; x < rows * P; x += kTcThreads) {
    const int r = x / P, c = x % P;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)r * D) + c);
    *reinterpret_cast<uint4*>(tile + sw128_offset(r, c, rows)) = v;
  }
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
score_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ K,
                float* __restrict__ u, Plan p, uint32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-byte aligned tiles (the swizzle pattern repeats every 1024 bytes)
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* qs = base;                              // [D/64][128 rows][128 B]
  unsigned char* ks = base + kTcRows * D * 2;            // [D/64][256 rows][128 B]
  __shared__ unsigned long long mma_done;
  __shared__ uint32_t tmem_slot;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;            // warpgroup: which half of the columns it reads back
  const int rr = threadIdx.x & (kTcRows - 1);  // row (TMEM lane) of this thread
  const int tiles = p.gm / kTcRows;
  const int group = blockIdx.x / tiles, tile = blockIdx.x % tiles;
  const int64_t row0 = (int64_t)group * p.gm + (int64_t)tile * kTcRows;

  if (warp == 0) tmem_alloc(&tmem_slot, kTcN);
  if (threadIdx.x == 0) {
    mbar_init(&mma_done, 1);
    mbar_fence_init();
  }
  stage_sw128<D>(qs, q + row0 * D, kTcRows);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  const __nv_bfloat16* Kg = K + (int64_t)group * p.n * D;
  float* urow = u + (row0 + rr) * p.ustride;
  constexpr uint32_t idesc = idesc_bf16(kTcRows, kTcN, false, false);
  bool ok = true;

  const int nchunks = (int)(p.n / kTcN);
  for (int c = 0; c < nchunks; ++c) {
    stage_sw128<D>(ks, Kg + (int64_t)c * kTcN * D, kTcN);
    fence_proxy_async();  // generic-proxy writes -> visible to the tensor core
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        // k-step s: atom s / 4, 32-byte slice s % 4 of each 128-byte row
        const uint32_t off = (uint32_t)((s & 3) * 32);
        const uint32_t qa = smem_u32(qs) + (uint32_t)((s >> 2) * kTcRows * kSwRowBytes) + off;
        const uint32_t ka = smem_u32(ks) + (uint32_t)((s >> 2) * kTcN * kSwRowBytes) + off;
        tc_mma(tmem, desc_kmajor(qa), desc_kmajor(ka), idesc, s > 0);
      }
      tc_commit(&mma_done);
    }
    if (!mbar_wait(&mma_done, (unsigned)c & 1u)) {
      if (lane == 0) atomicOr(status, CTA_DEV_TIMEOUT);
      ok = false;
    }
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int cb = wg * (kTcN / 64); cb < (wg + 1) * (kTcN / 64); ++cb) {
        uint32_t v[32];
        tc_ld32(lane_addr + (uint32_t)(cb * 32), v);
        float4* dst = reinterpret_cast<float4*>(urow + (int64_t)c * kTcN + cb * 32);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                               __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
      }
    }
    tc_fence_before();
    // the K tile and the accumulator columns are free again; stop on a timeout
    if (__syncthreads_or(ok ? 0 : 1)) break;
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTcN);
}

template <int D>
size_t score_tc_smem() {
  return 1024 + (size_t)(kTcRows + kTcN) * D * 2;
}

}  // namespace

bool score_tc_applies(const Plan& p, int dtype) {
  return dtype == kDtypeBF16 && (p.d == 64 || p.d == 128) && p.gm % kTcRows == 0 &&
         p.n % kTcN == 0 && p.n <= (int64_t)kShortMaxN;
}

cudaError_t launch_score_tc(const void* q, const void* K, float* u, const Plan& p,
                            uint32_t* status, cudaStream_t st) {
  const unsigned grid = (unsigned)(p.groups * (p.gm / kTcRows));
  if (p.d == 64) {
    const size_t smem = std::max<size_t>(score_tc_smem<64>(), 100 * 1024);  // <= 2 CTAs per SM
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    score_tc_kernel<64><<<grid, kTcThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(K), u, p, status);
  } else {
    const size_t smem = std::max<size_t>(score_tc_smem<128>(), 100 * 1024);
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    score_tc_kernel<128><<<grid, kTcThreads, smem, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(K), u, p, status);
  }
  return cudaGetLastError();
}

}  // namespace cta
