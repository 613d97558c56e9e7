// Dense reference attention Attn(q, K, V) = sum_i softmax(s)_i v_i over every
// key, s_i = q.k_i / sqrt(d): the full output that the truncation error
// ||Attn - Attn_k||_2 ("A Mathematical Theory of Top-k Sparse Attention via
// Total Variation Distance", arXiv 2512.07647, abstract) is measured against.
//
// Deliberately independent of the certified path: one CTA per row, single
// pass, online softmax (running max and rescaled sums) per lane group, fp32
// arithmetic, lane groups merged in a fixed order at the end.  Not tuned.
#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kDenseThreads = 256;
constexpr int kDenseWarps = kDenseThreads / kWarp;

template <typename T, int D>
__global__ void __launch_bounds__(kDenseThreads)
dense_kernel(const T* __restrict__ q, const T* __restrict__ K, const T* __restrict__ V,
             T* __restrict__ out, int64_t n, int gm, float scale) {
  constexpr int EPL = Elem<T>::EPL;
  constexpr int LPK = D / EPL;
  constexpr int KPI = kWarp / LPK;
  constexpr int SLOTS = kDenseWarps * KPI;
  __shared__ float s_m[SLOTS], s_z[SLOTS];
  __shared__ float s_acc[SLOTS][D];

  const int64_t row = blockIdx.x;
  const int64_t group = row / gm;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int part = lane % LPK, slot = lane / LPK;
  const int gslot = warp * KPI + slot;
  const T* Kg = K + group * n * D;
  const T* Vg = V + group * n * D;

  float qv[EPL];
  Elem<T>::unpack(*reinterpret_cast<const uint4*>(q + row * D + part * EPL), qv);

  float m = kNegInf, z = 0.f, acc[EPL];
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;

  // Every lane of a warp runs the same number of iterations (shuffles below).
  for (int64_t base = 0; base < n; base += SLOTS) {
    const int64_t i = base + gslot;
    const bool valid = i < n;
    float kv[EPL], vv[EPL];
    Elem<T>::unpack(valid ? ld_stream(Kg + i * D + part * EPL) : make_uint4(0u, 0u, 0u, 0u), kv);
    Elem<T>::unpack(valid ? ld_stream(Vg + i * D + part * EPL) : make_uint4(0u, 0u, 0u, 0u), vv);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) dot = fmaf(qv[e], kv[e], dot);
#pragma unroll
    for (int o = LPK / 2; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (valid) {
      const float s = dot * scale;
      const float mn = fmaxf(m, s);
      const float c = expf(m - mn);   // 0 on the first key (m = -inf)
      const float w = expf(s - mn);
      z = z * c + w;
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] = fmaf(w, vv[e], acc[e] * c);
      m = mn;
    }
  }
  if (part == 0) { s_m[gslot] = m; s_z[gslot] = z; }
#pragma unroll
  for (int e = 0; e < EPL; ++e) s_acc[gslot][part * EPL + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float M = kNegInf;
    for (int g = 0; g < SLOTS; ++g) M = fmaxf(M, s_m[g]);
    float Z = 0.f, A = 0.f;
    for (int g = 0; g < SLOTS; ++g) {
      if (s_m[g] == kNegInf) continue;  // lane group saw no key
      const float c = expf(s_m[g] - M);
      Z += s_z[g] * c;
      A += s_acc[g][threadIdx.x] * c;
    }
    Elem<T>::store1(out + row * D + threadIdx.x, A / Z);
  }
}

template <typename T>
cudaError_t launch_dense_t(const void* q, const void* K, const void* V, void* out, int64_t n, int d,
                           int64_t rows, int gm, cudaStream_t st) {
  const float scale = (float)(1.0 / sqrt((double)d));
  if (d == 64)
    dense_kernel<T, 64><<<(unsigned)rows, kDenseThreads, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(K), static_cast<const T*>(V),
        static_cast<T*>(out), n, gm, scale);
  else
    dense_kernel<T, 128><<<(unsigned)rows, kDenseThreads, 0, st>>>(
        static_cast<const T*>(q), static_cast<const T*>(K), static_cast<const T*>(V),
        static_cast<T*>(out), n, gm, scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dense(int dtype, const void* q, const void* K, const void* V, void* out,
                         int64_t n, int d, int64_t rows, int gm, cudaStream_t st) {
  if (dtype == kDtypeF32) return launch_dense_t<float>(q, K, V, out, n, d, rows, gm, st);
  return launch_dense_t<__nv_bfloat16>(q, K, V, out, n, d, rows, gm, st);
}

}  // namespace cta
