// Device-side building blocks shared by the libcta kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cta {

constexpr int kWarp = 32;
#define kNegInf (__int_as_float(0xff800000))

// Launch plan, computed once on the host per call and passed by value.
struct Plan {
  int64_t n;            // keys per KV head
  int64_t rows;         // batch * n_heads * m
  int d;                // head dimension
  int gm;               // rows sharing one KV head: (n_heads / n_kv_heads) * m
  int groups;           // batch * n_kv_heads
  int chunk;            // keys per chunk (score / output passes)
  int nchunks;          // ceil(n / chunk)
  int rt_score;         // rows per score tile
  int tiles_score;      // ceil(gm / rt_score)
  int rt_out;           // rows per output-pass tile
  int tiles_out;        // ceil(gm / rt_out)
  float scale2;         // log2(e)/sqrt(d), rounded to fp32: weights are 2^(-scale2 (M - u))
  float two_s;          // 2^mass_shift, the fixed-point scale of the masses
  int mass_shift;
  double eps;
  int want_err;         // 1: also accumulate the dropped keys' value rows
  int sel_cluster;      // CTAs (a thread-block cluster) per row in the selection pass
};

// Per-row result of the selection pass.
struct RowSel {
  float M;                  // largest logit of the row (unscaled dot product)
  uint32_t kstar;           // order key of the last kept logit
  int32_t istar;            // key index of the last kept key
  int32_t k;                // k_eps
  unsigned long long Z;     // total fixed-point mass
  unsigned long long C;     // kept fixed-point mass
  double tv;                // (Z - C) / Z
};

// Per (row, chunk) record of the output pass.
struct Partial {
  double wh;                // sum of kept weights
  double wt;                // sum of dropped weights
};

constexpr float kBinsPerOctave = 64.0f;  // selection bins per halving of the weight
constexpr int kBins = 2048;               // selection bins (32 octaves; the last one is open)

// ---------------------------------------------------------------------------
// order-preserving 32-bit key of an fp32 logit: a > b  <=>  key(a) > key(b)
// (after -0 has been folded into +0).

__device__ __forceinline__ uint32_t order_key(float u) {
  uint32_t b = __float_as_uint(u);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(b);
}

// Composite key: logit order in the high word, lower key index ranks higher
// in the low word, so descending composite order is (logit desc, index asc).
__device__ __forceinline__ unsigned long long composite(uint32_t key, uint32_t idx) {
  return ((unsigned long long)key << 32) | (unsigned long long)(0xffffffffu - idx);
}

// A key is kept iff its composite key is >= the threshold's.
__device__ __forceinline__ bool is_kept(uint32_t key, uint32_t idx, uint32_t kstar, uint32_t istar) {
  return key > kstar || (key == kstar && idx <= istar);
}

// Softmax numerator relative to the row max: w = 2^(-a) with
// a = (M - u) * log2(e)/sqrt(d) >= 0, i.e. exp((u - M)/sqrt(d)).  The
// subtraction and product are rounded explicitly so that every kernel computes
// bit-identical exponents (and so weights and bins) for the same logit.
__device__ __forceinline__ float weight_arg(float u, float M, float scale2) {
  return __fmul_rn(__fsub_rn(M, u), scale2);
}
__device__ __forceinline__ float weight(float u, float M, float scale2) {
  return exp2f(-weight_arg(u, M, scale2));
}
// Selection bin of a logit: floor(64 a), so bin b holds weights in
// (2^-(b+1)/64, 2^-b/64] up to exp2f's rounding; non-finite values stay in range.
__device__ __forceinline__ int weight_bin(float a) {
  return (int)fminf(fmaxf(a * kBinsPerOctave, 0.0f), (float)(kBins - 1));
}

// Fixed-point mass of a weight (exact integer sums, order independent).
__device__ __forceinline__ unsigned long long fixed_mass(float w, float two_s) {
  return __float2ull_rn(__fmul_rn(fmaxf(w, 0.0f), two_s));  // NaN weights count as 0
}

// The certificate test in fp64: discarded mass / total <= eps.
__device__ __forceinline__ bool certified(unsigned long long Z, unsigned long long C, double eps) {
  return (double)(Z - C) / (double)Z <= eps;
}

// ---------------------------------------------------------------------------
// 16-byte streaming load (read-only path, no L1 allocation).

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Streaming load with an L2 evict-first policy (data read exactly once).
__device__ __forceinline__ uint4 ld_stream_once(const void* p, unsigned long long pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(pol));
  return r;
}

__device__ __forceinline__ unsigned long long policy_evict_first() {
  unsigned long long pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ unsigned long long policy_evict_last() {
  unsigned long long pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Element traits: 16 bytes hold EPL elements; unpack widens them to fp32.
template <typename T> struct Elem;

template <> struct Elem<float> {
  static constexpr int EPL = 4;
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  __device__ __forceinline__ static float load1(const float* p) { return *p; }
  __device__ __forceinline__ static void store1(float* p, float v) { *p = v; }
};

template <> struct Elem<__nv_bfloat16> {
  static constexpr int EPL = 8;
  __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
    // bf16 is the upper half of an fp32 word: widening is exact.
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ static float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void store1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

// ---------------------------------------------------------------------------
// Transposed butterfly reduction across the LPK lanes that share one key.
// On entry each lane holds CNT partial sums (one per row of a tile); on exit
// a[0] holds the full sum of row (lane % LPK) / (LPK / CNT).  Uses
// CNT - 1 + log2(LPK / CNT) shuffles instead of CNT * log2(LPK).
template <int CNT, int O>
struct TransposeReduce {
  __device__ __forceinline__ static void run(float* a, int lane) {
    if constexpr (O >= 1) {
      if constexpr (CNT > 1) {
        constexpr int H = CNT / 2;
        const bool upper = (lane & O) != 0;
#pragma unroll
        for (int i = 0; i < H; ++i) {
          const float send = upper ? a[i] : a[i + H];
          const float keep = upper ? a[i + H] : a[i];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
        }
        TransposeReduce<H, O / 2>::run(a, lane);
      } else {
        a[0] += __shfl_xor_sync(0xffffffffu, a[0], O);
        TransposeReduce<1, O / 2>::run(a, lane);
      }
    }
  }
};

}  // namespace cta
