// Phase 1: logits.  For every row the unscaled logit u_i = q . k_i of every key
// (fp32, fixed summation order), written to the workspace, and the largest
// logit of each (row, chunk).
//
// Method: certified Top-k attention, "A Mathematical Theory of Top-k Sparse
// Attention via Total Variation Distance" (arXiv 2512.07647), abstract: the
// truncation acts on one attention distribution P = softmax(s) with
// s_i = q.k_i / sqrt(d).  The scale is applied later; ranking uses u.
//
// Mapping: one CTA per (row tile, key chunk, KV group).  All rows of a tile
// read the same KV head, so every K row is loaded once per tile (once per
// GQA group when the tile covers the whole group, as in decode).  Each warp
// streams whole K rows with 16-byte coalesced loads: LPK lanes share one key,
// each lane owns a fixed d-slice (so its q slice lives in registers) and the
// LPK partial dot products are combined with a transposed butterfly.  Logits
// are staged in shared memory and written out coalesced.
#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / kWarp;
constexpr int kUnroll = 8;

template <typename T, int D, int RT>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(const T* __restrict__ q, const T* __restrict__ K, float* __restrict__ u,
             float* __restrict__ cmax, Plan p, uint32_t* __restrict__ status) {
  constexpr int EPL = Elem<T>::EPL;
  constexpr int LPK = D / EPL;     // lanes per key
  constexpr int KPI = kWarp / LPK; // keys per warp-wide load
  static_assert(RT <= LPK, "tile rows must not exceed lanes per key");
  static_assert(LPK <= kWarp && (kWarp % LPK) == 0, "bad key width");

  extern __shared__ float su[];    // [RT][chunk]
  __shared__ float red[kScoreWarps][RT];

  const int tile = blockIdx.x;
  const int chunk = blockIdx.y;
  const int group = blockIdx.z;
  const int lane = threadIdx.x & (kWarp - 1);
  const int warp = threadIdx.x >> 5;
  const int part = lane % LPK;
  const int slot = lane / LPK;

  const int64_t row0 = (int64_t)group * p.gm + (int64_t)tile * RT;
  const int nrows = min(RT, p.gm - tile * RT);
  const int64_t key0 = (int64_t)chunk * p.chunk;
  const int nk = (int)min((int64_t)p.chunk, p.n - key0);
  const T* Kc = K + ((int64_t)group * p.n + key0) * D;

  // q slices of the tile's rows; rows past the group's end contribute zeros.
  float qr[RT][EPL];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    if (r < nrows) {
      const uint4 raw = *reinterpret_cast<const uint4*>(q + (row0 + r) * D + part * EPL);
      Elem<T>::unpack(raw, qr[r]);
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) qr[r][e] = 0.f;
    }
  }

  const unsigned long long pol = (p.tiles_score == 1) ? policy_evict_first() : policy_evict_last();
  const int stride = kScoreWarps * KPI;            // keys per CTA-wide step
  const int row_of_lane = part / (LPK / RT);       // row held after the butterfly
  const bool writer = (part % (LPK / RT)) == 0;

  for (int base = warp * KPI; base < nk; base += stride * kUnroll) {
    uint4 raw[kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int key = base + j * stride + slot;
      raw[j] = (key < nk) ? ld_stream_once(Kc + (int64_t)key * D + part * EPL, pol)
                          : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      float kv[EPL];
      Elem<T>::unpack(raw[j], kv);
      float acc[RT];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a = fmaf(qr[r][e], kv[e], a);
        acc[r] = a;
      }
      TransposeReduce<RT, LPK / 2>::run(acc, lane);
      const int key = base + j * stride + slot;
      if (writer && key < nk && row_of_lane < nrows) {
        su[row_of_lane * p.chunk + key] = acc[0] + 0.0f;  // folds -0 into +0
      }
    }
  }
  __syncthreads();

  // Coalesced write-out, chunk maxima and a non-finite check.
  float mx[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) mx[r] = kNegInf;
  bool bad = false;
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    if (r < nrows) {
      float* dst = u + (row0 + r) * p.n + key0;
      for (int i = threadIdx.x; i < nk; i += kScoreThreads) {
        const float x = su[r * p.chunk + i];
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
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(status, CTA_DEV_NONFINITE);
  if (threadIdx.x < RT && threadIdx.x < nrows) {
    float v = red[0][threadIdx.x];
    for (int w = 1; w < kScoreWarps; ++w) v = fmaxf(v, red[w][threadIdx.x]);
    cmax[(row0 + threadIdx.x) * p.nchunks + chunk] = v;
  }
}

template <typename T, int D, int RT>
cudaError_t launch_score_t(const void* q, const void* K, float* u, float* cmax, const Plan& p,
                           uint32_t* status, cudaStream_t st) {
  const size_t smem = sizeof(float) * RT * p.chunk;
  auto kern = score_kernel<T, D, RT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.tiles_score, p.nchunks, p.groups);
  kern<<<grid, kScoreThreads, smem, st>>>(static_cast<const T*>(q), static_cast<const T*>(K), u,
                                          cmax, p, status);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_score_d(const void* q, const void* K, float* u, float* cmax, const Plan& p,
                           uint32_t* status, cudaStream_t st) {
  switch (p.rt_score) {
    case 1: return launch_score_t<T, D, 1>(q, K, u, cmax, p, status, st);
    case 2: return launch_score_t<T, D, 2>(q, K, u, cmax, p, status, st);
    case 4: return launch_score_t<T, D, 4>(q, K, u, cmax, p, status, st);
    case 8: return launch_score_t<T, D, 8>(q, K, u, cmax, p, status, st);
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
