// Device-side building blocks shared by the libcta kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

namespace cta {

constexpr int kWarp = 32;
#define kNegInf (__int_as_float(0xff800000))

// Launch plan, computed once on the host per call and passed by value.
struct Plan {
  int64_t n;            // keys per KV head
  int64_t ustride;      // row stride of the logit buffer: n rounded up to 64
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
  int nranges;          // output pass: chunk ranges per (KV group, row tile)
  int range_len;        // chunks per range
  int gparts;           // partial maxima of the dropped logits per row (one per selection CTA)
  int rstages;          // tensor-core output pass: 128-key stages per range (0: not used)
  int nmax;             // partial row maxima per row in cmax (per chunk, or per range of
                        // the tensor-core logits pass); row stride nchunks
  int settle_group;     // tensor-core decode path: value-pass ranges per CTA of the last kernel
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
  double wh;                // sum of the kept keys' weights (fp64, fixed order)
  double wt;                // sum of the dropped keys' weights
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
// Tensor-core decode path: exact masses in 128-bit fixed point, key levels and
// the records the three kernels of that path exchange through the workspace.

// Unsigned 128-bit integer (two 64-bit words) for exact mass sums: every
// weight w in [0, 1] becomes round(w * 2^62), so any number of them adds up
// without overflow and without depending on the order of the additions.
struct U128 {
  unsigned long long lo, hi;
};
constexpr int kMass62 = 62;
__device__ __forceinline__ U128 u128_zero() { return U128{0ull, 0ull}; }
__device__ __forceinline__ void u128_add(U128& a, unsigned long long x) {
  asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(a.lo), "+l"(a.hi) : "l"(x));
}
__device__ __forceinline__ void u128_add(U128& a, const U128& b) {
  asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, %3;" : "+l"(a.lo), "+l"(a.hi) : "l"(b.lo), "l"(b.hi));
}
__device__ __forceinline__ U128 u128_sub(U128 a, const U128& b) {
  asm("sub.cc.u64 %0, %0, %2;\n\tsubc.u64 %1, %1, %3;" : "+l"(a.lo), "+l"(a.hi) : "l"(b.lo), "l"(b.hi));
  return a;
}
__device__ __forceinline__ bool u128_lt(const U128& a, const U128& b) {
  return a.hi < b.hi || (a.hi == b.hi && a.lo < b.lo);
}
__device__ __forceinline__ double u128_to_double(const U128& a) {
  return (double)a.hi * 18446744073709551616.0 + (double)a.lo;
}
// Sum over the 32 lanes of a warp (butterfly: every lane ends with the total).
__device__ __forceinline__ U128 u128_warp_sum(U128 a) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    U128 b;
    b.lo = __shfl_xor_sync(0xffffffffu, a.lo, o);
    b.hi = __shfl_xor_sync(0xffffffffu, a.hi, o);
    u128_add(a, b);
  }
  return a;
}
// The weight w (fp32, 0 <= w <= 1) in units of 2^-62.
__device__ __forceinline__ unsigned long long mass62(float w) {
  return __float2ull_rn(__fmul_rn(fmaxf(w, 0.0f), 4.611686018427387904e18f));
}
// The certificate test on exact masses: (Z - C) / Z <= eps, in fp64.
__device__ __forceinline__ bool certified128(const U128& Z, const U128& C, double eps) {
  return u128_to_double(u128_sub(Z, C)) / u128_to_double(Z) <= eps;
}

// Level of a logit: ceil(64 x) with x = u * log2(e)/sqrt(d) rounded to fp32,
// i.e. the key's position on a grid of 1/64 of a halving of the weight.  It is
// a non-decreasing function of u, so a level interval is an interval of the
// ranking; every kernel computes it with these exact operations.  NaN and
// huge values are clamped (their rows are flagged non-finite).
constexpr int kLevelsPerOctave = 64;
__device__ __forceinline__ int key_level(float u, float scale2) {
  float x = __fmul_rn(u, scale2);
  x = fminf(fmaxf(x, -1.0e6f), 1.0e6f);
  return __float2int_ru(x * (float)kLevelsPerOctave);
}

// Per (row, key range) level histogram written by the tensor-core logits pass.
// Fine bin i counts the range's keys of level top - i; octave o of the frame
// is bins 64 o .. 64 o + 63.  top is a multiple of 64 set from the range's
// first stage (its largest level rounded up, plus kHistHeadroom octaves).
constexpr int kHistOctaves = 48;
constexpr int kHistHeadroom = 16;                        // octaves above the first stage's max
constexpr int kHistBins = kHistOctaves * kLevelsPerOctave;  // 3072
constexpr uint32_t kHistAbove = 0x1u;   // a key lay above the frame: the record is unusable
constexpr uint32_t kHistSaturated = 0x2u;  // a fine count exceeded 65535
struct RangeHist {
  int32_t top;                  // level of fine bin 0 (multiple of 64)
  uint32_t flags;               // kHistAbove | kHistSaturated
  uint32_t below;               // keys below the frame (level <= top - kHistBins)
  uint32_t pad;
  uint32_t ocnt[kHistOctaves];  // keys per octave
  float omass[kHistOctaves];    // per octave: sum over its bins j of count * 2^(-j/64)
  uint16_t fine[kHistBins];     // keys per fine bin (saturating)
};
static_assert(sizeof(RangeHist) % 16 == 0, "records are read with 16-byte loads");

// Per row: the level bracket of the cut that the value pass used.  Keys with
// level >= lhi are kept for certain, keys with level < llo dropped for certain,
// the window llo <= level < lhi is settled once the exact cut is known.
struct RowBracket {
  float M;        // largest logit of the row
  int32_t llo, lhi;
  uint32_t pad;
};

// Per (row, key range): what the value pass accumulated over the range's keys.
struct RangeRec {
  U128 mh, mt, mw;   // exact masses (2^-62 units) of the kept, dropped and window keys
  double wh, wt;     // weight sums of the kept and dropped keys (window keys excluded),
                     // fp32 per stage and lane, fp64 above: an independent reduction for KL
  uint32_t nh, nw;   // kept and window key counts
  float tmax;        // largest logit among the dropped keys (-inf if none)
  uint32_t pad;
};
static_assert(sizeof(RangeRec) % 16 == 0, "16-byte records");

// Per (row, key range) after the last kernel has settled the range's window keys.
struct SegRec {
  double wh, wt;     // weight sums (for KL) of the kept and dropped keys of the range
  float tmax;        // largest dropped logit of the range
  uint32_t pad[3];
};

constexpr int kCandCap = 2048;   // window keys per row kept as candidates for the exact cut

// Workspace regions of the tensor-core decode path (device pointers, set per call).
struct TcBufs {
  RangeHist* hist;       // [rows][nranges]
  RangeRec* rrec;        // [rows][nranges]
  SegRec* srec;          // [rows][nranges]
  RowBracket* brk;       // [rows]
  unsigned long long* cand;  // [rows][kCandCap] composite keys of window keys
  uint32_t* cand_cnt;    // [rows] window keys seen (zeroed by the logits pass)
  uint32_t* ticket;      // [rows] ranges settled (zeroed by the logits pass)
  uint32_t* brk_ready;   // [rows] 1 once the row's bracket is written (zeroed by the logits pass)
  uint32_t* hmask;       // [rows][mask_words] bit j of word w: key 32 w + j kept for certain
  int64_t mask_words;    // words per row: 4 per 128-key stage
};

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
// Packed fp32 pair FMA (Blackwell f32x2): d = a * b + c on both lanes, each
// with a single IEEE round-to-nearest like fmaf.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n .reg .b64 ra, rb, rc, rd;\n"
      " mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rc, {%6, %7};\n"
      " fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// The same on packed pairs held in 64-bit registers (no repacking per FMA).
__device__ __forceinline__ unsigned long long fma2p(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long pack2(uint32_t lo, uint32_t hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float sum2(unsigned long long v) {
  float x, y;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(x), "=f"(y) : "l"(v));
  return x + y;
}

// bf16 pair (one 32-bit word, element 0 in the low half) widened to fp32.
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// ---------------------------------------------------------------------------
// mbarrier and bulk-copy (TMA, non-multicast) helpers.  Every wait is bounded
// by wall time: on expiry it reports failure instead of spinning forever.

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(unsigned long long* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}
// Wait for the phase with the given parity to complete; false after ~2 s.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, unsigned parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}
// 1-D bulk copy global -> this CTA's shared memory, completing on bar.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, unsigned bytes,
                                          unsigned long long* bar, unsigned long long policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ---------------------------------------------------------------------------
// Transposed butterfly reduction across the LPK lanes that share one key,
// without selects.  Each lane holds CNT partial sums, slot s holding row
// s ^ mask where mask = row_mask<CNT, LPK>(part), part = lane % LPK (the
// caller arranges its rows that way).  At the level with xor offset O the two
// partner lanes differ in the mask bit of that level, so the row a lane keeps
// is always in its low half and the row its partner needs is always in its
// high half: a[i] += shfl_xor(a[i + H], O).  On exit a[0..max(1, CNT/LPK))
// hold full sums of rows i ^ mask, i.e. row part / (LPK / CNT) when
// CNT <= LPK and rows i + (CNT / LPK) * part otherwise.
template <int CNT, int LPK>
__device__ __forceinline__ int row_mask(int part) {
  if constexpr (CNT >= LPK) {
    return (CNT / LPK) * part;
  } else {
    int shift = 0;
    while ((LPK >> shift) > CNT) ++shift;  // log2(LPK / CNT)
    return part >> shift;
  }
}

template <int CNT, int O>
struct XorReduce {
  __device__ __forceinline__ static void run(float* a) {
    if constexpr (O >= 1) {
      if constexpr (CNT > 1) {
        constexpr int H = CNT / 2;
#pragma unroll
        for (int i = 0; i < H; ++i) a[i] += __shfl_xor_sync(0xffffffffu, a[i + H], O);
        XorReduce<H, O / 2>::run(a);
      } else {
        a[0] += __shfl_xor_sync(0xffffffffu, a[0], O);
        XorReduce<1, O / 2>::run(a);
      }
    }
  }
};

}  // namespace cta
