// Phase 1: logits.  For every row the unscaled logit u_i = q . k_i of every key
// (fp32, fixed summation order), written to the workspace, and the largest
// logit of each (row, chunk).
//
// Method: certified Top-k attention, "A Mathematical Theory of Top-k Sparse
// Attention via Total Variation Distance" (arXiv 2512.07647), abstract: the
// truncation acts on one attention distribution P = softmax(s) with
// s_i = q.k_i / sqrt(d).  The scale is applied later; ranking uses u.
//
// Persistent CTAs walk a list of items (row tile, key chunk, KV group).  All
// rows of a tile read the same KV head, so every K row is read once per tile
// (once per GQA group in decode).  Each item's K rows, contiguous in memory,
// stream into a ring of four 16 KB shared-memory stages by bulk copies (TMA,
// cp.async.bulk, completion on mbarriers) that one thread issues four tiles
// ahead; eight warps compute from shared memory.  LPK lanes share one key, each
// lane owning 32 bytes of it and the matching q values in registers (its two
// 16-byte pieces are read in a lane-dependent order that spreads a warp's
// reads evenly over the shared-memory banks).  Products accumulate with packed
// f32x2 FMAs; a select-free transposed butterfly (each lane holds its rows in
// a lane-dependent order) combines the LPK partial sums.  Logits are
// staged per item in shared memory and written out coalesced with the chunk
// maxima.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kWarps = 8;
constexpr int kScoreThreads = kWarps * kWarp;
constexpr int kStageBytes = 32768;  // K rows per stage: 128 keys of 256 B
constexpr int kStages = 2;

template <typename T, int D, int RT>
struct ScoreCfg {
  static constexpr int ROWB = D * (int)sizeof(T);     // bytes per key row
  static constexpr int LPK = ROWB / 32;               // lanes per key (32 bytes each)
  static constexpr int KPI = kWarp / LPK;             // keys per warp step
  static constexpr int EPC = 16 / (int)sizeof(T);     // elements per 16-byte piece
  static constexpr int TK = kStageBytes / ROWB;       // keys per stage
  static constexpr int NOUT = RT >= LPK ? RT / LPK : 1;  // rows each lane holds after the butterfly
  static_assert(LPK >= 1 && LPK <= kWarp && kWarp % LPK == 0, "bad key width");
  static_assert(TK % (2 * kWarps * KPI) == 0, "a stage must split into pairs of warp steps");
  static constexpr int PAIRS = TK / (2 * kWarps * KPI);  // pairs of key steps per warp and stage
};

// Widen one 16-byte piece to EPC/2 packed fp32 pairs (64-bit registers).
template <typename T> __device__ __forceinline__ void widen_pairs(const uint4& r, unsigned long long* f);
template <>
__device__ __forceinline__ void widen_pairs<__nv_bfloat16>(const uint4& r, unsigned long long* f) {
  f[0] = pack2(r.x << 16, r.x & 0xffff0000u);
  f[1] = pack2(r.y << 16, r.y & 0xffff0000u);
  f[2] = pack2(r.z << 16, r.z & 0xffff0000u);
  f[3] = pack2(r.w << 16, r.w & 0xffff0000u);
}
template <> __device__ __forceinline__ void widen_pairs<float>(const uint4& r, unsigned long long* f) {
  f[0] = pack2(r.x, r.y);
  f[1] = pack2(r.z, r.w);
}

struct Item {
  int tile, chunk, group;
};
__device__ __forceinline__ Item item_of(int it, const Plan& p) {
  Item r;
  r.tile = it % p.tiles_score;
  const int rest = it / p.tiles_score;
  r.chunk = rest % p.nchunks;
  r.group = rest / p.nchunks;
  return r;
}

// Walks this CTA's (item, stage tile) sequence for the copy issuer.
struct TileIter {
  int it, j, nk;
  int64_t key0;
  int group;
  __device__ void start(int first, int nitems, const Plan& p) {
    it = first;
    j = 0;
    load(nitems, p);
  }
  __device__ void load(int nitems, const Plan& p) {
    if (it >= nitems) return;
    const Item I = item_of(it, p);
    key0 = (int64_t)I.chunk * p.chunk;
    nk = (int)min((int64_t)p.chunk, p.n - key0);
    group = I.group;
  }
  __device__ bool valid(int nitems) const { return it < nitems; }
  __device__ void next(int tk, int nitems, const Plan& p) {
    if ((j + 1) * tk < nk) { ++j; return; }
    it += gridDim.x;
    j = 0;
    load(nitems, p);
  }
};

template <typename T, int D, int RT>
__global__ void __launch_bounds__(kScoreThreads, 2)
score_kernel(const T* __restrict__ q, const T* __restrict__ K, float* __restrict__ u,
             float* __restrict__ cmax, Plan p, uint32_t* __restrict__ status) {
  using C = ScoreCfg<T, D, RT>;
  constexpr int NP = C::EPC / 2;  // fp32 pairs per 16-byte piece

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* stage = smem_raw;                                        // [kStages][32 KB]
  float* su = reinterpret_cast<float*>(smem_raw + kStages * kStageBytes);  // [RT][su_stride]
  // Row stride of the staged logits: chunk + KPI puts the rows of one warp
  // step in different banks (chunk is a multiple of 256).
  const int su_stride = p.chunk + C::KPI;
  __shared__ unsigned long long full[kStages];
  __shared__ int done_cnt[kStages];  // warps finished with each stage (cumulative)
  __shared__ float red[kWarps][RT];
  // Copy issuer state: the last warp to release a stage refills it, so the
  // state lives in shared memory.
  __shared__ TileIter prod;
  __shared__ int issued;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nitems = p.tiles_score * p.nchunks * p.groups;
  const unsigned long long pol = (p.tiles_score == 1) ? policy_evict_first() : policy_evict_last();

  // Bulk copies run kStages tiles ahead of consumption; whichever warp is the
  // last to release a stage issues its refill.
  auto issue_next = [&]() {
    if (!prod.valid(nitems)) return;
    const int s = issued % kStages;
    const int keys = min(C::TK, prod.nk - prod.j * C::TK);
    const unsigned bytes = (unsigned)(keys * C::ROWB);
    const unsigned char* src = reinterpret_cast<const unsigned char*>(
        K + ((int64_t)prod.group * p.n + prod.key0 + (int64_t)prod.j * C::TK) * D);
    mbar_arrive_expect_tx(&full[s], bytes);
    bulk_load(stage + s * kStageBytes, src, bytes, &full[s], pol);
    ++issued;
    prod.next(C::TK, nitems, p);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      done_cnt[s] = 0;
    }
    mbar_fence_init();
    issued = 0;
    prod.start(blockIdx.x, nitems, p);
    for (int s = 0; s < kStages; ++s) issue_next();
  }
  __syncthreads();

  // The lane's 32 bytes are pieces part and part + LPK of the key row.  Shared
  // memory serves 16-byte reads per 8 lanes: with LPK >= 8 those 8 lanes read
  // 8 consecutive pieces; with LPK = 4 (two keys per 8 lanes) the second key
  // starts from the other half, so every 8 lanes hit 8 different bank groups.
  const int part = lane % C::LPK;
  const int slot = lane / C::LPK;
  const int h = (C::LPK < 8) ? (slot & 1) : 0;
  const int ca = part + C::LPK * h;        // first 16-byte piece
  const int cb = part + C::LPK * (1 - h);  // second piece
  const int mask = row_mask<RT, C::LPK>(part);  // slot s of this lane holds row s ^ mask
  const bool writer = (RT >= C::LPK) || (part % (C::LPK / RT)) == 0;

  int t = 0;
  for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
    const Item I = item_of(it, p);
    const int64_t row0 = (int64_t)I.group * p.gm + (int64_t)I.tile * RT;
    const int nrows = min(RT, p.gm - I.tile * RT);
    const int64_t key0 = (int64_t)I.chunk * p.chunk;
    const int nk = (int)min((int64_t)p.chunk, p.n - key0);

    // q values of this lane's two pieces, for every row of the tile
    unsigned long long qa[RT][NP], qb[RT][NP];
#pragma unroll
    for (int sl = 0; sl < RT; ++sl) {
      const int r = sl ^ mask;
      if (r < nrows) {
        const uint4* qr = reinterpret_cast<const uint4*>(q + (row0 + r) * D);
        widen_pairs<T>(qr[ca], qa[sl]);
        widen_pairs<T>(qr[cb], qb[sl]);
      } else {
#pragma unroll
        for (int e = 0; e < NP; ++e) { qa[sl][e] = 0ull; qb[sl][e] = 0ull; }
      }
    }

    for (int j = 0; j * C::TK < nk; ++j, ++t) {
      const int s = t % kStages;
      const unsigned ph = (unsigned)(t / kStages) & 1u;
      // Every warp waits on the same barriers, so a copy that never lands
      // times all of them out at the same tile, before any item-end barrier.
      if (!mbar_wait(&full[s], ph)) {
        if (lane == 0) atomicOr(status, CTA_DEV_TIMEOUT);
        return;
      }
      const int nkt = min(C::TK, nk - j * C::TK);
      const uint4* st = reinterpret_cast<const uint4*>(stage + s * kStageBytes);
      (void)ph;
      // Pairs of key steps per warp: both dot products first, then both
      // butterflies, so the two shuffle chains overlap.
#pragma unroll
      for (int hp = 0; hp < C::PAIRS; ++hp) {
      const int kbase = hp * 2 * kWarps * C::KPI;
      float acc[2][RT];
#pragma unroll
      for (int u2 = 0; u2 < 2; ++u2) {
        const int key = kbase + warp * C::KPI + u2 * kWarps * C::KPI + slot;  // < TK
        unsigned long long ka[NP], kb[NP];
        widen_pairs<T>(st[key * (C::ROWB / 16) + ca], ka);
        widen_pairs<T>(st[key * (C::ROWB / 16) + cb], kb);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          unsigned long long a2 = 0ull;  // (+0, +0)
#pragma unroll
          for (int e = 0; e < NP; ++e) a2 = fma2p(qa[r][e], ka[e], a2);
#pragma unroll
          for (int e = 0; e < NP; ++e) a2 = fma2p(qb[r][e], kb[e], a2);
          acc[u2][r] = sum2(a2);
        }
      }
      XorReduce<RT, C::LPK / 2>::run(acc[0]);
      XorReduce<RT, C::LPK / 2>::run(acc[1]);
#pragma unroll
      for (int u2 = 0; u2 < 2; ++u2) {
        const int key = kbase + warp * C::KPI + u2 * kWarps * C::KPI + slot;
        if (writer && key < nkt) {
#pragma unroll
          for (int o = 0; o < C::NOUT; ++o) {
            const int r = o ^ mask;
            if (r < nrows) su[r * su_stride + j * C::TK + key] = acc[u2][o] + 0.0f;  // folds -0 into +0
          }
        }
      }
      }  // pairs of key steps
      __syncwarp();
      if (lane == 0) {
        // the last of the kWarps warps to release this fill refills it with
        // tile t + kStages
        __threadfence_block();
        const int done = atomicAdd(&done_cnt[s], 1);
        if (done == kWarps * (t / kStages) + kWarps - 1) {
          __threadfence_block();
          issue_next();
          __threadfence_block();
        }
      }
    }

    // item done: coalesced write-out, chunk maxima, non-finite check
    __syncthreads();
    float mx[RT];
    bool bad = false;
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      mx[r] = kNegInf;
      if (r < nrows) {
        float* dst = u + (row0 + r) * p.ustride + key0;
        for (int i = threadIdx.x; i < nk; i += kScoreThreads) {
          const float x = su[r * su_stride + i];
          dst[i] = x;
          bad |= !isfinite(x);
          mx[r] = fmaxf(mx[r], x);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      float v = mx[r];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (lane == 0) red[warp][r] = v;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(status, CTA_DEV_NONFINITE);
    __syncthreads();
    if (threadIdx.x < nrows) {
      float v = red[0][threadIdx.x];
      for (int w = 1; w < kWarps; ++w) v = fmaxf(v, red[w][threadIdx.x]);
      cmax[(row0 + threadIdx.x) * p.nchunks + I.chunk] = v;
    }
    __syncthreads();  // su and red are free again
  }
}

template <typename T, int D, int RT>
cudaError_t launch_score_t(const void* q, const void* K, float* u, float* cmax, const Plan& p,
                           uint32_t* status, cudaStream_t st) {
  const size_t smem = (size_t)kStages * kStageBytes +
                      sizeof(float) * RT * (p.chunk + ScoreCfg<T, D, RT>::KPI);
  auto kern = score_kernel<T, D, RT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kScoreThreads, smem);
  if (e != cudaSuccess) return e;
  const long long nitems = (long long)p.tiles_score * p.nchunks * p.groups;
  const long long grid = std::min<long long>(nitems, (long long)std::max(per_sm, 1) * sm_count());
  kern<<<(unsigned)grid, kScoreThreads, smem, st>>>(static_cast<const T*>(q),
                                                    static_cast<const T*>(K), u, cmax, p, status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_score_d(const void* q, const void* K, float* u, float* cmax, const Plan& p,
                           uint32_t* status, cudaStream_t st) {
  switch (p.rt_score) {
    case 1: return launch_score_t<T, D, 1>(q, K, u, cmax, p, status, st);
    case 2: return launch_score_t<T, D, 2>(q, K, u, cmax, p, status, st);
    case 4: return launch_score_t<T, D, 4>(q, K, u, cmax, p, status, st);
    case 8:
      if constexpr (sizeof(T) == 4) return launch_score_t<T, D, 8>(q, K, u, cmax, p, status, st);
      else return cudaErrorInvalidValue;  // bf16 tiles have at most 4 rows
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_score(int dtype, const void* q, const void* K, float* u, float* cmax,
                         const Plan& p, uint32_t* status, cudaStream_t st) {
  if (dtype == kDtypeF32) {
    return p.d == 64 ? launch_score_d<float, 64>(q, K, u, cmax, p, status, st)
                     : launch_score_d<float, 128>(q, K, u, cmax, p, status, st);
  }
  return p.d == 64 ? launch_score_d<__nv_bfloat16, 64>(q, K, u, cmax, p, status, st)
                   : launch_score_d<__nv_bfloat16, 128>(q, K, u, cmax, p, status, st);
}

}  // namespace cta
