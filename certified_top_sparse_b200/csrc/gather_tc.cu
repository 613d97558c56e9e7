// Phases 3 and 4 for decode-shaped problems (bf16 values, d = 128) on the
// 5th-generation tensor cores.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the exact head-tail
// decomposition Attn = H mu_head + tau mu_tail, the truncated output is mu_head
// and the error needs mu_tail, i.e. per row the kept sum sum_{kept} w_i v_i
// and the dropped sum sum_{dropped} w_i v_i over all n value rows.
//
// For the (at most four) query rows of a row tile, which share one KV head,
// these sums are one contraction per stage of 128 keys:
//     S[dim][c] += sum_key V[key][dim] W[c][key],
// column c running over (kept, dropped) x (three bf16 parts of the fp32
// weight) x row.  The parts hi = bf16(w), mid = bf16(w - hi), lo = bf16(w -
// hi - mid) carry the fp32 weight to about 2^-24 relative, and bf16 x bf16
// products are exact in the fp32 accumulator, so the sums match fp32
// multiply-adds up to the order of addition.  The CUDA cores only turn logits
// into weights; value rows go from HBM to shared memory by TMA and from there
// into tcgen05.mma as the MN-major A operand (M = 128 dimensions), the weights
// are the K-major B operand (N = 32, unused columns zero), and the sums
// accumulate in tensor memory over the whole key range of a work item.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0     TMA: each stage is two 64-dimension boxes of 128 keys (128-byte
//              swizzle) into a ring of kGStages slots;
//   warp 1     MMA: 8 MMAs (K = 16) per stage, whose commit frees the slot; at
//              the end of an item a commit hands the accumulator over; owns
//              the tensor memory (two accumulators, so an item's epilogue
//              overlaps the next item's stream);
//   warp 0     also brings the stage's logits of the tile's rows (bulk copies
//              on the same barrier), so the weight warps read shared memory only;
//   warps 2-5  weights: warp r writes row r's part of the stage's W tile;
//   warps 6-9  epilogue: read the accumulator, add the parts in fp64, write
//              the range partial.
// Work items are (KV group, key range, row tile) with ranges cut in stages so
// that every SM gets about the same number of stages.  A second, row-parallel
// kernel (one CTA per row, all range partials loaded at once) forms the
// outputs; it is launched as a programmatic dependent so that its launch
// overlaps the tail of this one.
#include <algorithm>

#include "common.cuh"
#include "finalize.cuh"  // single_gap_bound
#include "kernels.cuh"
#include "umma.cuh"

namespace cta {

namespace {

constexpr int kGD = 128;              // head dimension: MMA M, one TMEM lane per dimension
constexpr int kGK = 128;              // keys per stage
constexpr int kGN = 32;               // MMA N: weight columns, zero padded
constexpr int kGStages = 5;
constexpr int kGBox = 64;             // dimensions per TMA box: 128 bytes of bf16
constexpr int kGV = kGK * kGD * 2;    // value bytes per stage (32 KB)
constexpr int kGW = kGN * kGK * 2;    // weight-tile bytes per stage (8 KB)
constexpr int kGU = 4 * kGK * 4;      // logit bytes per stage: up to four rows of kGK fp32 (2 KB)
constexpr int kGWarps = 10;
constexpr int kGThreads = kGWarps * kWarp;
constexpr int kGWeightWarp0 = 2;
constexpr int kGEpiWarp0 = 6;
constexpr int kGEpiThreads = 4 * kWarp;
constexpr int kGEpiBar = 1;           // named barrier of the epilogue warps
constexpr uint32_t kGTmemCols = 2 * kGN;
constexpr size_t kGSmem = 1024 + (size_t)kGStages * (kGV + kGW + kGU);
static_assert(kGK % 64 == 0 && kGK <= 256, "a stage is whole 64-key swizzle atoms, one TMA box");
static_assert(kGSmem <= 227 * 1024, "shared memory");

struct GItem {
  int tile, range, group;
};
__device__ __forceinline__ GItem gitem_of(int it, const Plan& p) {
  GItem g;
  g.tile = it % p.tiles_out;
  const int rest = it / p.tiles_out;
  g.range = rest % p.nranges;
  g.group = rest / p.nranges;
  return g;
}

// Column of the accumulator / row of the W tile: a = 0 kept, 1 dropped;
// part 0, 1, 2 = hi, mid, lo; r = row of the tile.
template <int RT>
__device__ __forceinline__ int wcol(int a, int part, int r) {
  return (a * 3 + part) * RT + r;
}

// w ~ hi + mid + lo in bf16 (each remainder is exact in fp32).
__device__ __forceinline__ void split3(float w, uint32_t* part) {
  const __nv_bfloat16 h = __float2bfloat16_rn(w);
  const float r1 = __fsub_rn(w, __bfloat162float(h));
  const __nv_bfloat16 m = __float2bfloat16_rn(r1);
  const float r2 = __fsub_rn(r1, __bfloat162float(m));
  const __nv_bfloat16 l = __float2bfloat16_rn(r2);
  part[0] = __bfloat16_as_ushort(h);
  part[1] = __bfloat16_as_ushort(m);
  part[2] = __bfloat16_as_ushort(l);
}

__device__ __forceinline__ bool aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}

template <int RT, bool ERR>
__global__ void __launch_bounds__(kGThreads, 1)
gather_tc_kernel(const __grid_constant__ CUtensorMap vmap, const float* __restrict__ u,
                 const RowSel* __restrict__ sel, float* __restrict__ acc_out, Plan p,
                 uint32_t* __restrict__ status) {
  // the finalisation kernel may be scheduled now; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* vring = base;                          // [kGStages][2 boxes][kGK keys][128 B]
  unsigned char* wring = base + kGStages * kGV;         // [kGStages][kGK / 64][kGN rows][128 B]
  float* uring = reinterpret_cast<float*>(wring + kGStages * kGW);  // [kGStages][4 rows][kGK]
  __shared__ unsigned long long vfull[kGStages], wfull[kGStages], empty[kGStages];
  __shared__ unsigned long long accfull[2], accempty[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nitems = p.tiles_out * p.nranges * p.groups;
  const int spu = (int)((p.n + kGK - 1) / kGK);  // stages per (KV group, row tile)

  // W columns that no row writes stay zero
  for (int x = threadIdx.x; x < kGStages * kGW / 16; x += kGThreads)
    reinterpret_cast<uint4*>(wring)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();
  __syncwarp();
  if (warp == 1) tmem_alloc(&tmem_slot, kGTmemCols);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&wfull[s], RT);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kGEpiThreads);
    }
    mbar_init(&drain, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const unsigned long long pol = (p.tiles_out == 1) ? policy_evict_first() : policy_evict_last();
      const unsigned long long pol_u = policy_evict_first();
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(&vmap))
                   : "memory");
      int t = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const GItem g = gitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
        const int nrows = min(RT, p.gm - g.tile * RT);
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kGStages;
          if (t >= kGStages && !mbar_wait(&empty[slot], (unsigned)(t / kGStages - 1) & 1u)) {
            ok = false;
            break;
          }
          if (aborted(&s_abort)) {
            ok = false;
            break;
          }
          // the rows' logits of the stage's keys below n, in whole 16-byte pieces
          // (the logit rows are padded to a multiple of 64 keys)
          const int64_t key0 = (int64_t)sg * kGK;
          const unsigned ub = (unsigned)((min((int64_t)kGK, p.n - key0) + 3) / 4) * 16u;
          unsigned char* dst = vring + slot * kGV;
          mbar_arrive_expect_tx(&vfull[slot], (unsigned)kGV + ub * (unsigned)nrows);
          tma_load_3d(dst, &vmap, 0, (int)key0, g.group, &vfull[slot], pol);
          tma_load_3d(dst + kGV / 2, &vmap, kGBox, (int)key0, g.group, &vfull[slot], pol);
          for (int r = 0; r < nrows; ++r)
            bulk_load(uring + (slot * 4 + r) * kGK, u + (row0 + r) * p.ustride + key0, ub,
                      &vfull[slot], pol_u);
        }
      }
      if (!ok) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
        // the copies still in flight land before the CTA may exit (bounded)
        for (int t2 = max(0, t - kGStages); t2 < t; ++t2)
          mbar_wait(&vfull[t2 % kGStages], (unsigned)(t2 / kGStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kGD, kGN, /*a_mn=*/true, /*b_mn=*/false);
      int t = 0, j = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++j) {
        const GItem g = gitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        const int b = j & 1;
        if (j >= 2 && !mbar_wait(&accempty[b], (unsigned)((j >> 1) - 1) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * kGN);
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kGStages;
          const unsigned ph = (unsigned)(t / kGStages) & 1u;
          if (!mbar_wait(&vfull[slot], ph) || !mbar_wait(&wfull[slot], ph) || aborted(&s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v0 = smem_u32(vring + slot * kGV), w0 = smem_u32(wring + slot * kGW);
#pragma unroll
          for (int s = 0; s < kGK / 16; ++s)
            tc_mma(d, desc_mnmajor(v0 + (uint32_t)(s * 16 * kSwRowBytes), (uint32_t)(kGV / 2)),
                   desc_kmajor(w0 + (uint32_t)((s >> 2) * kGN * kSwRowBytes + (s & 3) * 32)), idesc,
                   (sg > s_lo || s > 0) ? 1u : 0u);
          tc_commit(&empty[slot]);
        }
        if (!ok) break;
        tc_commit(&accfull[b]);
      }
      if (!ok) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
      }
      tc_commit(&drain);  // every MMA issued has finished before the CTA exits (bounded)
      mbar_wait(&drain, 0u);
    }
  } else if (warp < kGEpiWarp0) {
    // ---------------- weights: warp r -> row r of the tile ----------------
    const int r = warp - kGWeightWarp0;
    if (r < RT) {
      int t = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const GItem g = gitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
        const bool row_ok = r < min(RT, p.gm - g.tile * RT);
        float M = 0.0f;
        uint32_t ks = 0u, is = 0u;
        // this kernel is a programmatic dependent of selection: its row results
        // are read only after that grid has finished
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (row_ok) {
          const RowSel* rs = sel + row0 + r;
          M = __ldg(&rs->M);
          ks = __ldg(&rs->kstar);
          is = (uint32_t)__ldg(&rs->istar);
        }
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kGStages;
          const int64_t k0 = (int64_t)sg * kGK + 4 * lane;  // this lane's four keys
          // the stage (values and logits) has landed; its slot's W tile is then
          // free too (the MMAs that last read the slot have finished)
          if (!mbar_wait(&vfull[slot], (unsigned)(t / kGStages) & 1u) || aborted(&s_abort)) ok = false;
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row_ok) x = reinterpret_cast<const float4*>(uring + (slot * 4 + r) * kGK)[lane];
          // weights of the four keys, split into kept / dropped and three parts
          uint32_t hp[4][3], tp[4][3];
          const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float w = 0.0f;
            bool kept = false;
            if (row_ok && k0 + i < p.n) {
              w = weight(xs[i], M, p.scale2);
              kept = is_kept(order_key(xs[i]), (uint32_t)(k0 + i), ks, is);
            }
            split3(kept ? w : 0.0f, hp[i]);
            if constexpr (ERR) split3(kept ? 0.0f : w, tp[i]);
          }
          unsigned char* wt = wring + slot * kGW;
          const int c = lane >> 1;  // 16-byte piece (8 keys) along K; this lane writes one half
          const uint32_t half = (uint32_t)(lane & 1) * 8u;
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            *reinterpret_cast<uint2*>(wt + sw128_offset(wcol<RT>(0, part, r), c, kGN) + half) =
                make_uint2(hp[0][part] | (hp[1][part] << 16), hp[2][part] | (hp[3][part] << 16));
            if constexpr (ERR)
              *reinterpret_cast<uint2*>(wt + sw128_offset(wcol<RT>(1, part, r), c, kGN) + half) =
                  make_uint2(tp[0][part] | (tp[1][part] << 16), tp[2][part] | (tp[3][part] << 16));
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) mbar_arrive(&wfull[slot]);
        }
      }
      if (!ok && lane == 0) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
      }
    }
  } else {
    // ---------------- epilogue ----------------
    const int tid = threadIdx.x - kGEpiWarp0 * kWarp;  // 0..127
    const int quarter = warp & 3;                      // TMEM lanes this warp may read
    const int dim = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    int j = 0;
    bool failed = false;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++j) {
      const GItem g = gitem_of(it, p);
      const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
      const int nrows = min(RT, p.gm - g.tile * RT);
      const int b = j & 1;
      const bool ok = mbar_wait(&accfull[b], (unsigned)(j >> 1) & 1u);
      if (bar_red_or(kGEpiBar, kGEpiThreads, !ok || aborted(&s_abort))) {
        failed = true;
        break;
      }
      tc_fence_after();
      __syncwarp();
      uint32_t c[32];
      tc_ld32(lane_addr + (uint32_t)(b * kGN), c);
      tc_fence_before();
      mbar_arrive(&accempty[b]);
      // range partial of each row: the three parts added in fp64, fixed order
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        if (r < nrows) {
#pragma unroll
          for (int a = 0; a < (ERR ? 2 : 1); ++a) {
            const double v = ((double)__uint_as_float(c[wcol<RT>(a, 0, r)]) +
                              (double)__uint_as_float(c[wcol<RT>(a, 1, r)])) +
                             (double)__uint_as_float(c[wcol<RT>(a, 2, r)]);
            acc_out[(((row0 + r) * p.nranges + g.range) * 2 + a) * kGD + dim] = (float)v;
          }
        }
      }
    }
    if (failed && tid == 0) {
      atomicOr(status, CTA_DEV_TIMEOUT);
      s_abort = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  __syncwarp();
  if (warp == 1) tmem_dealloc(tmem, kGTmemCols);
}

// Phase 4: one CTA per row, launched as a programmatic dependent of the value
// pass (it waits for that grid's results).  Thread (a, dim) sums the head
// (a = 0) or tail (a = 1) partials of one dimension over the ranges in a fixed
// order, sixteen loads in flight.  256 threads: the CTA fits beside a value-
// pass or logits CTA on an SM, so it neither waits for a free SM nor keeps the
// next call's logits pass off one.
constexpr int kFinThreads = 2 * kGD;

template <bool ERR>
__global__ void __launch_bounds__(kFinThreads)
finalize_tc_kernel(const float* __restrict__ acc_out, const RowSel* __restrict__ sel,
                   const float* __restrict__ gmax, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ err_out, float* __restrict__ kl_out,
                   float* __restrict__ gap_out, Plan p, uint32_t* __restrict__ status) {
  // The next call's logits pass may be scheduled now (it streams K at once
  // and waits for this grid before it writes the logits).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ double tail[kGD];
  __shared__ double sq[kGD];
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const int a = tid / kGD, dim = tid % kGD;
  // every load of the row is issued before the first use: the row's selection
  // result, its dropped-logit maxima and this thread's range partials
  const RowSel rs = sel[row];
  float gpart = kNegInf;  // warp 2 (which forms the gap bound) loads the partial maxima
  if (tid >= 2 * kWarp && tid - 2 * kWarp < p.gparts)
    gpart = __ldcg(gmax + row * kMaxGParts + (tid - 2 * kWarp));
  double s = 0.0;
  if (ERR || a == 0) {
    const float* src = acc_out + (row * p.nranges * 2 + a) * kGD + dim;
#pragma unroll 16
    for (int c = 0; c < p.nranges; ++c) s += (double)__ldcg(src + (int64_t)c * 2 * kGD);
  }
  if (a == 1) tail[dim] = s;
  __syncthreads();
  if (a == 0) {
    const double mu_h = s / rs.wh;
    out[row * kGD + dim] = __float2bfloat16_rn((float)mu_h);
    const double diff = (ERR && rs.wt > 0.0) ? tail[dim] / rs.wt - mu_h : 0.0;
    sq[dim] = diff * diff;
  }
  __syncthreads();
  if (tid < kWarp) {  // fixed-order tree over the dimensions
    double v = (sq[4 * tid] + sq[4 * tid + 1]) + (sq[4 * tid + 2] + sq[4 * tid + 3]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (tid == 0) {
      if (!(rs.wh > 0.0)) atomicOr(status, CTA_DEV_INTERNAL);
      if (err_out) err_out[row] = (float)(rs.C < rs.Z && rs.wt > 0.0 ? rs.tv * sqrt(v) : 0.0);
    }
  } else if (tid == kWarp) {
    if (kl_out) kl_out[row] = (float)log1p(rs.wt / rs.wh);
  } else if (tid >= 2 * kWarp && tid < 3 * kWarp && gap_out) {
    // the row's largest dropped logit over the selection CTAs' partial maxima
    float gm = __shfl_sync(0xffffffffu, gpart, 0);
    for (int c = 1; c < kMaxGParts; ++c) gm = fmaxf(gm, __shfl_sync(0xffffffffu, gpart, c));
    if (tid == 2 * kWarp)
      gap_out[row] = (float)single_gap_bound((double)key_value(rs.kstar), (double)gm, rs.k, p.n, kGD);
  }
}

template <int RT, bool ERR>
cudaError_t launch_t(const CUtensorMap& map, const float* u, const RowSel* sel, float* acc,
                     const Plan& p, uint32_t* status, cudaStream_t st) {
  auto kern = gather_tc_kernel<RT, ERR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGSmem);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const long long nitems = (long long)p.tiles_out * p.nranges * p.groups;
  const unsigned grid = (unsigned)std::min<long long>(nitems, sms);
  // programmatic dependent of selection: the value stream starts early
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kGThreads, 1, 1);
  cfg.dynamicSmemBytes = kGSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, u, sel, acc, p, status);
}

template <bool ERR>
cudaError_t launch_finalize(const float* acc, const RowSel* sel, const float* gmax, void* out,
                            float* err_out, float* kl_out, float* gap_out, const Plan& p,
                            uint32_t* status, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.rows, 1, 1);
  cfg.blockDim = dim3(kFinThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, finalize_tc_kernel<ERR>, acc, sel, gmax,
                            static_cast<__nv_bfloat16*>(out), err_out, kl_out, gap_out, p, status);
}

template <bool ERR>
cudaError_t launch_e(const CUtensorMap& map, const float* u, const RowSel* sel, float* acc,
                     const Plan& p, uint32_t* status, cudaStream_t st) {
  switch (p.rt_out) {
    case 1: return launch_t<1, ERR>(map, u, sel, acc, p, status, st);
    case 2: return launch_t<2, ERR>(map, u, sel, acc, p, status, st);
    case 4: return launch_t<4, ERR>(map, u, sel, acc, p, status, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

bool encode_kv_map(CUtensorMap* map, const void* base, const Plan& p) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc || p.d != kGD) return false;
  // [groups][n][128] bf16: dimensions innermost, boxes of 64 dimensions x kGK keys
  const cuuint64_t dims[3] = {(cuuint64_t)kGD, (cuuint64_t)p.n, (cuuint64_t)p.groups};
  const cuuint64_t strides[2] = {(cuuint64_t)kGD * 2, (cuuint64_t)p.n * kGD * 2};
  const cuuint32_t box[3] = {(cuuint32_t)kGBox, (cuuint32_t)kGK, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gather_tc_applies(const Plan& p, int dtype) {
  return dtype == kDtypeBF16 && p.d == kGD && p.n >= kGK && p.rt_out <= 4 && encode_tiled() != nullptr;
}

void set_ranges_tc(Plan* p, int sms) {
  const int64_t units = (int64_t)p->groups * p->tiles_out;
  const int64_t spu = (p->n + kGK - 1) / kGK;
  // range partials fit the workspace (one slot per chunk); at most 1024 ranges are tried
  const int64_t cap = std::min<int64_t>(std::min<int64_t>(spu, p->nchunks), 1024);
  constexpr int64_t kItemCost = 1;  // a stage's worth of hand-over per item
  // Every range count is scored by the busiest CTA's items times their length
  // (items go round-robin over the grid); the eight best are then simulated
  // exactly (the last range of a unit is shorter).
  constexpr int kTry = 8;
  int64_t cand[kTry], cscore[kTry];
  int ncand = 0;
  for (int64_t nr = 1; nr <= cap; ++nr) {
    const int64_t rs = (spu + nr - 1) / nr;
    const int64_t nranges = (spu + rs - 1) / rs;
    if (nranges != nr) continue;  // the same cut as a smaller count
    const int64_t items = units * nranges;
    const int64_t G = std::min<int64_t>(items, sms);
    const int64_t score = (items + G - 1) / G * (rs + kItemCost);
    int at;
    if (ncand < kTry) {
      at = ncand++;
    } else {
      if (score >= cscore[kTry - 1]) continue;
      at = kTry - 1;
    }
    cand[at] = nr;
    cscore[at] = score;
    while (at > 0 && cscore[at] < cscore[at - 1]) {  // keep the list sorted by score
      std::swap(cand[at], cand[at - 1]);
      std::swap(cscore[at], cscore[at - 1]);
      --at;
    }
  }
  int64_t best = -1, best_rs = spu, best_nr = 1;
  for (int c = 0; c < ncand; ++c) {
    const int64_t nranges = cand[c];
    const int64_t rs = (spu + nranges - 1) / nranges;
    const int64_t last = spu - (nranges - 1) * rs;
    const int64_t items = units * nranges;
    const int64_t G = std::min<int64_t>(items, sms);
    int64_t worst = 0;  // stages of the busiest CTA (items b, b + G, ... of the grid)
    for (int64_t b = 0; b < G; ++b) {
      int64_t w = 0;
      for (int64_t i = b; i < items; i += G)
        w += (((i / p->tiles_out) % nranges) == nranges - 1 ? last : rs) + kItemCost;
      worst = std::max(worst, w);
    }
    if (best < 0 || worst < best) {
      best = worst;
      best_rs = rs;
      best_nr = nranges;
    }
  }
  p->rstages = (int)best_rs;
  p->nranges = (int)best_nr;
}

cudaError_t launch_gather_tc(const void* V, const float* u, const RowSel* sel, float* acc,
                             const Plan& p, uint32_t* status, cudaStream_t st) {
  if (p.rstages < 1) return cudaErrorInvalidValue;
  CUtensorMap map;
  if (!encode_kv_map(&map, V, p)) return cudaErrorInvalidValue;
  return p.want_err ? launch_e<true>(map, u, sel, acc, p, status, st)
                    : launch_e<false>(map, u, sel, acc, p, status, st);
}

cudaError_t launch_finalize_tc(const float* acc, const RowSel* sel, const float* gmax, void* out,
                               float* err_out, float* kl_out, float* gap_out, const Plan& p,
                               uint32_t* status, cudaStream_t st) {
  return p.want_err
             ? launch_finalize<true>(acc, sel, gmax, out, err_out, kl_out, gap_out, p, status, st)
             : launch_finalize<false>(acc, sel, gmax, out, err_out, kl_out, gap_out, p, status, st);
}

}  // namespace cta
