// Phase 1 for decode-shaped problems (bf16 q and K, d = 128) on the
// 5th-generation tensor cores: u_i = q . k_i for the (at most four) query rows
// of a row tile, which share one KV head.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): the attention distribution of a query
// row is the softmax of its scores q.k_i / sqrt(d); this kernel writes the
// unscaled dot products (the scale is folded into the weights) and, per row
// and work range, the largest of them (selection takes the row maximum from
// those).
//
// Per stage of 128 keys the products are one MMA chain
//     S[key][r] = sum_dim K[key][dim] q[r][dim],
// with the K stage (K-major, 128-byte swizzled, as the TMA tensor load leaves
// it) as the A operand (M = 128 keys) and the row tile's queries as the B
// operand (N = 16, rows beyond the tile zero).  bf16 x bf16 products are exact
// in the fp32 accumulator; only the order of the sum over the dimensions
// differs from the CUDA-core kernel's.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0     TMA: K stages (two 64-dimension boxes of 128 keys) into a ring;
//   warp 1     stages the tile's queries once per work item (two buffers) and
//              issues 8 MMAs (K = 16) per stage into one of four tensor-memory
//              accumulators; owns the tensor memory;
//   warps 2-5  epilogue: each reads the scores of its 32 keys of the stage,
//              writes them to the logit rows (coalesced), tracks the rows'
//              maxima and non-finite values, and counts the keys per level
//              (key_level: 1/64 of a halving of the weight) in a shared-memory
//              histogram per row whose frame is fixed by the range's first
//              stage (its largest level, rounded up to a whole octave, plus
//              kHistHeadroom octaves; kHistOctaves octaves deep).  At the end
//              of a range the histogram goes to the workspace (RangeHist): the
//              fine counts and, per octave, the count and the count-weighted
//              sum of 2^(-j/64) over its 64 bins, from which the value pass
//              bounds every row's mass below any level without touching the
//              logits.
// Work items and key ranges are the ones the tensor-core value pass uses
// (Plan::rstages stages per range); the range maxima go to cmax[row][range].
//
// Ordering: the kernel is a programmatic dependent of the kernel before it on
// the stream (the caller's, or the previous call's last kernel).  Every
// thread waits for that grid (griddepcontrol.wait) before anything reads q or
// K or writes the workspace; only the tensor-memory allocation, the barrier
// set-up and the tensor-map prefetch come first.  It then lets the bracket
// kernel launch and zeroes the per-row counters and flags that the later
// kernels of the call use.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace cta {

namespace {

constexpr int kSD = 128;                   // head dimension: the contraction
constexpr int kSK = 128;                   // keys per stage: MMA M, one TMEM lane per key
constexpr int kSN = 16;                    // MMA N: query rows, zero padded
constexpr int kSStages = 5;
constexpr int kSAcc = 4;                   // TMEM accumulators: stages handed to the epilogue
constexpr int kSBox = 64;                  // dimensions per TMA box (128 bytes of bf16)
constexpr int kSStage = kSK * kSD * 2;     // K bytes per stage (32 KB)
constexpr int kSQ = kSN * kSD * 2;         // query tile (4 KB)
constexpr int kSThreads = 6 * kWarp;
constexpr int kSEpiWarp0 = 2;
constexpr int kSEpiThreads = 4 * kWarp;
constexpr int kSEpiBar = 1;                // named barrier of the epilogue warps
constexpr uint32_t kSTmemCols = kSAcc * kSN;
template <int RT>
constexpr size_t ssmem_bytes() {
  return 1024 + (size_t)kSStages * kSStage + 2 * (size_t)kSQ + (size_t)RT * kHistBins * 4;
}
static_assert(ssmem_bytes<4>() <= 227 * 1024, "shared memory");

struct SItem {
  int tile, range, group;
};
__device__ __forceinline__ SItem sitem_of(int it, const Plan& p) {
  SItem g;
  g.tile = it % p.tiles_score;
  const int rest = it / p.tiles_score;
  g.range = rest % p.nranges;
  g.group = rest / p.nranges;
  return g;
}

__device__ __forceinline__ bool aborted(const int* flag) {
  return *reinterpret_cast<const volatile int*>(flag) != 0;
}

template <int RT>
__global__ void __launch_bounds__(kSThreads, 1)
score_kv_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __nv_bfloat16* __restrict__ q,
                   float* __restrict__ u, float* __restrict__ cmax, TcBufs tb, Plan p,
                   uint32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* kring = base;                        // [kSStages][2 boxes][kSK keys][128 B]
  unsigned char* qbuf = base + kSStages * kSStage;    // [2][kSD / 64][kSN rows][128 B]
  uint32_t* hist = reinterpret_cast<uint32_t*>(qbuf + 2 * kSQ);  // [RT][kHistBins]
  __shared__ unsigned long long kfull[kSStages], kempty[kSStages];
  __shared__ unsigned long long accfull[kSAcc], accempty[kSAcc], qfree[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int s_abort;
  __shared__ float red[4][RT];
  __shared__ float pow_j[kLevelsPerOctave];  // 2^(-j/64)
  __shared__ uint32_t hist_below[RT], hist_flags;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nitems = p.tiles_score * p.nranges * p.groups;
  const int spu = (int)((p.n + kSK - 1) / kSK);  // stages per (KV group, row tile)

  for (int x = threadIdx.x; x < RT * kHistBins; x += kSThreads) hist[x] = 0u;
  if (threadIdx.x < kLevelsPerOctave)
    pow_j[threadIdx.x] = exp2f(-(float)threadIdx.x / (float)kLevelsPerOctave);
  if (threadIdx.x < RT) hist_below[threadIdx.x] = 0u;
  if (threadIdx.x == 0) hist_flags = 0u;
  __syncwarp();
  if (warp == 1) tmem_alloc(&tmem_slot, kSTmemCols);
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSStages; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int a = 0; a < kSAcc; ++a) {
      mbar_init(&accfull[a], 1);
      mbar_init(&accempty[a], 4);  // one arrival per epilogue warp
    }
    mbar_init(&qfree[0], 1);
    mbar_init(&qfree[1], 1);
    mbar_init(&drain, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  if (threadIdx.x == 0)
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(&kmap))
                 : "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // The previous grid on the stream (a caller's kernel may write q or K) has
  // completed and its writes are visible from here on.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  for (int64_t i = (int64_t)blockIdx.x * kSThreads + threadIdx.x; i < p.rows;
       i += (int64_t)gridDim.x * kSThreads) {
    tb.cand_cnt[i] = 0u;
    tb.ticket[i] = 0u;
    tb.brk_ready[i] = 0u;
  }

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const unsigned long long pol = (p.tiles_score == 1) ? policy_evict_first() : policy_evict_last();
      int t = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const SItem g = sitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kSStages;
          if (t >= kSStages && !mbar_wait(&kempty[slot], (unsigned)(t / kSStages - 1) & 1u)) {
            ok = false;
            break;
          }
          if (aborted(&s_abort)) {
            ok = false;
            break;
          }
          unsigned char* dst = kring + slot * kSStage;
          mbar_arrive_expect_tx(&kfull[slot], (unsigned)kSStage);
          tma_load_3d(dst, &kmap, 0, sg * kSK, g.group, &kfull[slot], pol);
          tma_load_3d(dst + kSStage / 2, &kmap, kSBox, sg * kSK, g.group, &kfull[slot], pol);
        }
      }
      if (!ok) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
        for (int t2 = max(0, t - kSStages); t2 < t; ++t2)  // copies in flight land (bounded)
          mbar_wait(&kfull[t2 % kSStages], (unsigned)(t2 / kSStages) & 1u);
      }
    }
  } else if (warp == 1) {
    // ---------------- queries and MMA issue ----------------
    constexpr uint32_t idesc = idesc_bf16(kSK, kSN, /*a_mn=*/false, /*b_mn=*/false);
    int t = 0, j = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++j) {
      const SItem g = sitem_of(it, p);
      const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
      const int nrows = min(RT, p.gm - g.tile * RT);
      const int b = j & 1;
      // the MMAs that last read this query buffer (item j - 2) have finished
      if (lane == 0 && j >= 2) ok = mbar_wait(&qfree[b], (unsigned)((j >> 1) - 1) & 1u);
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
        ok = false;
        break;
      }
      unsigned char* qb = qbuf + b * kSQ;
      for (int x = lane; x < kSN * (kSD / 8); x += kWarp) {
        const int r = x / (kSD / 8), c = x % (kSD / 8);
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (r < nrows) v = __ldg(reinterpret_cast<const uint4*>(q + (row0 + r) * kSD) + c);
        *reinterpret_cast<uint4*>(qb + sw128_offset(r, c, kSN)) = v;
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        const uint32_t q0 = smem_u32(qb);
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kSStages, acc = t % kSAcc;
          if (!mbar_wait(&kfull[slot], (unsigned)(t / kSStages) & 1u) ||
              (t >= kSAcc && !mbar_wait(&accempty[acc], (unsigned)(t / kSAcc - 1) & 1u)) ||
              aborted(&s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k0 = smem_u32(kring + slot * kSStage);
#pragma unroll
          for (int s = 0; s < kSD / 16; ++s)
            tc_mma(tmem + (uint32_t)(acc * kSN),
                   desc_kmajor(k0 + (uint32_t)((s >> 2) * (kSStage / 2) + (s & 3) * 32)),
                   desc_kmajor(q0 + (uint32_t)((s >> 2) * kSN * kSwRowBytes + (s & 3) * 32)), idesc,
                   s > 0 ? 1u : 0u);
          tc_commit(&kempty[slot]);
          tc_commit(&accfull[acc]);
        }
        if (ok) tc_commit(&qfree[b]);
      }
      if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
        ok = false;
        break;
      }
    }
    if (lane == 0) {
      if (!ok) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
      }
      tc_commit(&drain);  // every MMA issued has finished before the CTA exits (bounded)
      mbar_wait(&drain, 0u);
    }
  } else {
    // ---------------- epilogue ----------------
    const int tid = threadIdx.x - kSEpiWarp0 * kWarp;  // 0..127
    const int quarter = warp & 3;                      // TMEM lanes (keys) this warp may read
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sc = p.scale2;
    int t = 0;
    bool failed = false;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
      const SItem g = sitem_of(it, p);
      const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
      const int nrows = min(RT, p.gm - g.tile * RT);
      const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
      float mx[RT];
      int top[RT];
      uint32_t below[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        mx[r] = kNegInf;
        top[r] = 0;
        below[r] = 0u;
      }
      bool bad = false;
      uint32_t above = 0u;  // bit r: a key of row r lay above the histogram frame
      for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
        const int acc = t % kSAcc;
        const bool ok = mbar_wait(&accfull[acc], (unsigned)(t / kSAcc) & 1u) && !aborted(&s_abort);
        const bool okw = __all_sync(0xffffffffu, ok);
        // a failed warp leaves at once, except at the first stage of a range,
        // whose barrier every epilogue warp must reach
        if (!okw && sg != s_lo) {
          failed = true;
          break;
        }
        uint32_t c[16];
        if (okw) {
          tc_fence_after();
          tc_ld16(lane_addr + (uint32_t)(acc * kSN), c);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&accempty[acc]);
        }
        const int64_t key = (int64_t)sg * kSK + quarter * 32 + lane;
        const bool in = okw && key < p.n;
        if (sg == s_lo) {
          // the frame of this range's histograms: the first stage's largest
          // level per row, rounded up to an octave, plus the headroom
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            float v = (in && r < nrows) ? __uint_as_float(c[r]) : kNegInf;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) red[quarter][r] = v;
          }
          if (bar_red_or(kSEpiBar, kSEpiThreads, !okw)) {
            failed = true;
            break;
          }
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            const float m0 = fmaxf(fmaxf(red[0][r], red[1][r]), fmaxf(red[2][r], red[3][r]));
            float x0 = __fmul_rn(m0, sc);
            x0 = fminf(fmaxf(x0, -1.0e6f), 1.0e6f);  // -inf (no key) and NaN stay finite
            top[r] = (__float2int_ru(x0) + kHistHeadroom) * kLevelsPerOctave;
          }
          bar_sync(kSEpiBar, kSEpiThreads);  // red is free again
        }
        if (in) {
#pragma unroll
          for (int r = 0; r < RT; ++r) {
            if (r < nrows) {
              const float x = __uint_as_float(c[r]);
              u[(row0 + r) * p.ustride + key] = x;
              mx[r] = fmaxf(mx[r], x);
              bad |= !isfinite(x);
              const int i = top[r] - key_level(x, sc);
              if (i < 0) above |= 1u << r;
              else if (i >= kHistBins) ++below[r];
              else atomicAdd(&hist[r * kHistBins + i], 1u);
            }
          }
        }
      }
      // the range maxima of the tile's rows over the four warps
      if (bar_red_or(kSEpiBar, kSEpiThreads, failed)) {
        failed = true;
        break;
      }
      above = __reduce_or_sync(0xffffffffu, above);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        float v = mx[r];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[quarter][r] = v;
        const uint32_t bsum = __reduce_add_sync(0xffffffffu, below[r]);
        if (lane == 0 && bsum) atomicAdd(&hist_below[r], bsum);
      }
      if (lane == 0 && above) atomicOr(&hist_flags, above);
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, CTA_DEV_NONFINITE);
      bar_sync(kSEpiBar, kSEpiThreads);
      if (tid < nrows)
        cmax[(row0 + tid) * p.nchunks + g.range] =
            fmaxf(fmaxf(red[0][tid], red[1][tid]), fmaxf(red[2][tid], red[3][tid]));
      // the histograms to the workspace: octave summaries first (they read
      // every bin), then the fine counts, zeroing the bins for the next range
      RangeHist* rec0 = tb.hist + row0 * p.nranges + g.range;
      for (int x = tid; x < nrows * kHistOctaves; x += kSEpiThreads) {
        const int r = x / kHistOctaves, o = x % kHistOctaves;
        const uint32_t* hb = hist + r * kHistBins + o * kLevelsPerOctave;
        uint32_t cn = 0u;
        float ms = 0.0f;
#pragma unroll 8
        for (int j = 0; j < kLevelsPerOctave; ++j) {
          const uint32_t v = hb[j];
          cn += v;
          ms = fmaf((float)v, pow_j[j], ms);
        }
        RangeHist* rec = rec0 + (int64_t)r * p.nranges;
        rec->ocnt[o] = cn;
        rec->omass[o] = ms;
      }
      bar_sync(kSEpiBar, kSEpiThreads);
      uint32_t sat = 0u;
      for (int x = tid; x < nrows * (kHistBins / 2); x += kSEpiThreads) {
        const int r = x / (kHistBins / 2), i = 2 * (x % (kHistBins / 2));
        uint32_t* hb = hist + r * kHistBins + i;
        const uint32_t a = hb[0], b = hb[1];
        hb[0] = 0u;
        hb[1] = 0u;
        if ((a | b) > 0xffffu) sat |= 1u << r;
        const uint32_t packed = min(a, 0xffffu) | (min(b, 0xffffu) << 16);
        *reinterpret_cast<uint32_t*>(&(rec0 + (int64_t)r * p.nranges)->fine[i]) = packed;
      }
      sat = __reduce_or_sync(0xffffffffu, sat);
      if (lane == 0 && sat) atomicOr(&hist_flags, sat << 8);
      bar_sync(kSEpiBar, kSEpiThreads);
      if (tid < nrows) {
        RangeHist* rec = rec0 + (int64_t)tid * p.nranges;
        const uint32_t fl = hist_flags;
        rec->top = top[tid];
        rec->flags = (((fl >> tid) & 1u) ? kHistAbove : 0u) | (((fl >> (8 + tid)) & 1u) ? kHistSaturated : 0u);
        rec->below = hist_below[tid];
        hist_below[tid] = 0u;
      }
      bar_sync(kSEpiBar, kSEpiThreads);  // red, hist_flags and hist_below are free again
      if (tid == 0) hist_flags = 0u;
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
  if (warp == 1) tmem_dealloc(tmem, kSTmemCols);
}

template <int RT>
cudaError_t launch_t(const CUtensorMap& map, const void* q, float* u, float* cmax,
                     const TcBufs& tb, const Plan& p, uint32_t* status, cudaStream_t st) {
  auto kern = score_kv_tc_kernel<RT>;
  constexpr size_t smem = ssmem_bytes<RT>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const long long nitems = (long long)p.tiles_score * p.nranges * p.groups;
  const unsigned grid = (unsigned)std::min<long long>(nitems, sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kSThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see "Ordering" above
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, static_cast<const __nv_bfloat16*>(q), u, cmax, tb, p,
                            status);
}

}  // namespace

cudaError_t launch_score_kv_tc(const void* q, const void* K, float* u, float* cmax,
                               const TcBufs& tb, const Plan& p, uint32_t* status,
                               cudaStream_t st) {
  if (p.rstages < 1 || p.tiles_score != p.tiles_out || p.rt_score != p.rt_out)
    return cudaErrorInvalidValue;
  CUtensorMap map;
  if (!encode_kv_map(&map, K, p)) return cudaErrorInvalidValue;
  switch (p.rt_score) {
    case 1: return launch_t<1>(map, q, u, cmax, tb, p, status, st);
    case 2: return launch_t<2>(map, q, u, cmax, tb, p, status, st);
    case 4: return launch_t<4>(map, q, u, cmax, tb, p, status, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace cta
