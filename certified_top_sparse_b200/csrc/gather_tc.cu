// Kernels 2 and 3 of the decode path (bf16 values, d = 128): the row brackets
// and the value pass on the 5th-generation tensor cores, which needs only a
// bracket of the cut, not the cut itself.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): certified Top-k keeps the minimal
// k_eps keys whose discarded softmax tail mass TV is <= eps; with the exact
// head-tail decomposition Attn = H mu_head + tau mu_tail the truncated output
// is mu_head and the error needs mu_tail, i.e. per row the kept sum
// sum_{kept} w_i v_i and the dropped sum sum_{dropped} w_i v_i.
//
// The bracket.  From the level histograms of the logits pass (RangeHist) the
// bracket kernel bounds, for every level boundary, the mass of the keys below it
// from above and from below (a level is 1/64 of a halving of the weight, so
// every key's weight is known within a factor 2^(1/64) from its level alone),
// and the total mass likewise.  The cut lies where the mass below reaches eps
// of the total, so every key whose level is certainly above that point is
// kept (level >= lhi) and every key certainly below is dropped (level < llo);
// the keys between (the window, typically a few hundred per row) are left to
// the last kernel, which finds the exact cut among them.  Octave totals of the
// histograms locate the octave(s) of the cut; only their fine bins are read.
//
// The value sums.  For the (at most four) query rows of a row tile, which
// share one KV head, the kept and dropped sums are one contraction per stage
// of 128 keys:
//     S[dim][c] += sum_key V[key][dim] W[c][key],
// column c running over (kept, dropped) x (three bf16 parts of the fp32
// weight) x row.  The parts hi = bf16(w), mid = bf16(w - hi), lo = bf16(w -
// hi - mid) carry the fp32 weight to about 2^-24 relative, and bf16 x bf16
// products are exact in the fp32 accumulator.  Window keys get weight 0 in
// both columns.  The value stages (V) come from HBM by TMA as the MN-major A
// operand (M = 128 dimensions), the weights are the K-major B operand (N = 32,
// unused columns zero), and the sums accumulate in tensor memory over the
// whole key range of a work item.
//
// The exact masses.  Alongside, every key's weight becomes an integer in units
// of 2^-62 (mass62) and is added, in 128 bits, to the kept, dropped or window
// mass of its row and range: exact and order-independent, so the last kernel's
// certificate test is exact too.  Window keys also go to a per-row candidate
// list (composite key: logit order, then index).  Per range the pass writes a
// RangeRec: the three masses, fp64 weight sums of the kept and dropped keys,
// their counts and the largest dropped logit.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0     TMA: each stage is two 64-dimension boxes of 128 keys (128-byte
//              swizzle) into a ring of kGStages slots, and the stage's logits
//              of the tile's rows (bulk copies on a barrier of their own);
//   warp 1     MMA: 8 MMAs (K = 16) per stage, whose commit frees the slot; at
//              the end of an item a commit hands the accumulator over; owns
//              the tensor memory (two accumulators);
//   warps 2-9  weights: warp 2 + r + 4 h writes row r's part of the W tile
//              and its masses in the stages of parity h (so two stages are in
//              the works at once), after its row's bracket is out; at the end
//              of an item the eight warps read the accumulator (each the
//              tensor-memory lane quarter of its warp % 4), add the parts in
//              fp64 and write the range partials.
// Work items are (KV group, key range, row tile) with ranges cut in stages so
// that every SM gets about the same number of stages.
//
// Ordering: logits pass -> bracket kernel -> value pass, each a programmatic
// dependent of the one before.  The bracket kernel lets the value pass launch
// only after its own wait for the logits pass, so when a value-pass CTA starts,
// the logits pass (and the caller's kernels before it) have completed: the
// producer streams value rows and logits at once, and the weight warps wait
// only for their own row's bracket (a flag per row, bounded wait).
#include <algorithm>
#include <climits>

#include "common.cuh"
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
constexpr int kGWeightWarps = 8;
constexpr int kGEpiThreads = kGWeightWarps * kWarp;  // the weight warps also read the accumulator
constexpr int kGEpiBar = 1;           // named barrier of the weight warps
constexpr uint32_t kGTmemCols = 2 * kGN;
constexpr int kCandBuf = 128;         // window keys a weight warp buffers (>= 128: one stage's)
constexpr size_t kGSmem = 1024 + (size_t)kGStages * (kGV + kGW + kGU) + kGWeightWarps * kCandBuf * 8;
static_assert(kGK % 64 == 0 && kGK <= 256, "a stage is whole 64-key swizzle atoms, one TMA box");
static_assert(kGSmem <= 227 * 1024, "shared memory");

constexpr int kMergeOct = 64;         // octaves of the merged per-row frame (two per lane)
constexpr int kFineOctMax = 4;        // window octaves refined with the fine counts

// A weight warp's part of a range record, handed to its partner warp.
struct RecPart {
  U128 mz, mh, mt;
  double wh, wt;
  uint32_t nh, nw;
  float tmax;
};

__device__ __forceinline__ RowBracket ld_cg_bracket(const RowBracket* b) {
  const int4 v = __ldcg(reinterpret_cast<const int4*>(b));
  return RowBracket{__int_as_float(v.x), v.y, v.z, (uint32_t)v.w};
}

// A row's bracket is handed from the bracket kernel to the value pass through
// a flag per row (zeroed by the logits pass of the same call): the value pass
// starts a row as soon as its bracket is out, not when every row's is.
__device__ __forceinline__ void publish_bracket(RowBracket* b, uint32_t* ready, const RowBracket& v) {
  *b = v;
  __threadfence();
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(ready), "r"(1u) : "memory");
}
// Lane 0 waits (bounded) for the flag; true once it is set.
__device__ __forceinline__ bool wait_bracket(const uint32_t* ready) {
  const int lane = threadIdx.x & 31;
  uint32_t ok = 1u;
  if (lane == 0) {
    auto seen = [&]() {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ready) : "memory");
      return v != 0u;
    };
    if (!seen()) {
      const unsigned long long t0 = global_ns();
      ok = 0u;
      while (global_ns() - t0 <= kWaitLimitNs) {
        if (seen()) {
          ok = 1u;
          break;
        }
      }
    }
  }
  // the warp barrier orders lane 0's acquire before every lane's reads of the bracket
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok, 0) != 0u;
}

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

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Appends a warp's buffered window keys buf[0, nb) to the row's candidate list
// (all are counted; keys beyond the list's capacity are dropped, which the
// last kernel detects from the count).  Whole warp.
__device__ __forceinline__ void flush_cands(const unsigned long long* buf, uint32_t nb,
                                            unsigned long long* cand, uint32_t* cnt) {
  const int lane = threadIdx.x & 31;
  uint32_t base = 0u;
  if (lane == 0) base = atomicAdd(cnt, nb);
  base = __shfl_sync(0xffffffffu, base, 0);
  for (uint32_t i = lane; i < nb; i += 32)
    if (base + i < (uint32_t)kCandCap) cand[base + i] = buf[i];
  __syncwarp();
}

// 2^e in fp32, exactly, for -126 <= e <= 127 (0 below).
__device__ __forceinline__ float pow2f_int(int e) {
  return e < -126 ? 0.0f : __int_as_float((127 + min(e, 127)) << 23);
}

// Inclusive suffix sums across the lanes (lane l gets the sum over lanes >= l).
__device__ __forceinline__ float warp_suffix_sum_f(float v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_down_sync(0xffffffffu, v, o);
    v += (lane + o < 32) ? y : 0.0f;
  }
  return v;
}
__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// The bracket of each row's cut: one CTA of kBWarps warps per row, between the
// logits pass and the value pass.  Reads the row's range histograms and range
// maxima and writes the row's RowBracket (M, llo, lhi).
//
// Frame: T = 64 ceil(X_M), X_M = fl(M * scale2), so every key's level is <= T;
// merged fine index g = T - level, octave O = g / 64.  A key with fine index g
// has weight w = 2^-a with a within E of X_M - (T - g)/64 ... X_M - (T - g - 1)/64,
// i.e. 2^(delta - (g + 1)/64) <= w <= 2^(delta - g/64) up to the relative slack
// s, where delta = T/64 - X_M in [0, 1) and E covers the fp32 rounding of
// a = (M - u) * scale2 against X_M - x and exp2f's error; s also covers the
// fp32 arithmetic of the bounds themselves (sums of a few thousand terms in
// any order).
//
// Steps: (1) every warp loads the headers and octave sums of its ranges
// (range r to warp r % kBWarps, up to kBPre ranges per warp in flight) while
// the block reduces the row maximum; (2) each warp merges its ranges into the
// row frame (range r's octave o is merged octave o - sh_r, sh_r = (top_r - T)
// / 64), the warps' partial sums are added in warp order; (3) warp 0 bounds the
// mass below every octave boundary and finds the window octaves [Ohi, Olo);
// (4) every warp adds its ranges' fine counts of the window bins into shared
// counters (integers: order-free); (5) warp 0 refines the boundaries bin by bin.
// ---------------------------------------------------------------------------
constexpr int kBWarps = 8;
constexpr int kBThreads = kBWarps * kWarp;
constexpr int kBPre = 4;  // ranges per warp whose loads go out before the row maximum is known

struct RangeHead {
  int top;
  uint32_t flags, below;
  float oa, ob;  // octave sums o = lane and o = lane + 32 (0 past the frame)
};

__device__ __forceinline__ RangeHead load_head(const RangeHist* h) {
  const int lane = threadIdx.x & 31;
  RangeHead x;
  x.top = __ldcg(&h->top);
  x.flags = __ldcg(&h->flags);
  x.below = __ldcg(&h->below);
  x.oa = __ldcg(&h->omass[lane]);
  x.ob = lane + 32 < kHistOctaves ? __ldcg(&h->omass[lane + 32]) : 0.0f;
  return x;
}

// Adds one range to the warp's merged octave sums mu (octaves lane, lane + 32)
// and its deep mass (keys below the merged frame; summed on lane 0 only for
// the range's own below-frame count).
__device__ __forceinline__ void merge_range(const RangeHist* h, const RangeHead& x, int T,
                                            float p_delta, float (&mu)[2], float& deep, bool& bad) {
  const int lane = threadIdx.x & 31;
  bad |= x.flags != 0u || (x.top % kLevelsPerOctave) != 0;
  const int sh = (x.top - T) / kLevelsPerOctave;
  if (lane == 0) deep += (float)x.below * p_delta * pow2f_int(sh - kHistOctaves);
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int o = lane + 32 * k + sh;  // the range octave that merged octave O needs
    const float va = __shfl_sync(0xffffffffu, x.oa, o & 31);
    const float vb = __shfl_sync(0xffffffffu, x.ob, o & 31);
    mu[k] += (o >= 0 && o < kHistOctaves) ? (o < 32 ? va : vb) : 0.0f;
  }
  // rare: the range's frame reaches below the merged frame (sh <= -17)
  if (sh <= kHistOctaves - 1 - kMergeOct) {
    for (int o = max(kMergeOct + sh, 0) + lane; o < kHistOctaves; o += 32)
      deep += (float)__ldcg(&h->ocnt[o]) * p_delta * pow2f_int(sh - o);
  }
}

// Adds one range's fine counts of the window bins: lane l covers bin pairs
// 64 q + 2 l (q < nwo) of the window that starts at merged fine index g0.
__device__ __forceinline__ void fine_range(const RangeHist* h, int sh, int g0, int nwo,
                                           uint32_t (&c)[2 * kFineOctMax]) {
  const int lane = threadIdx.x & 31;
  uint32_t v[kFineOctMax];
#pragma unroll
  for (int q = 0; q < kFineOctMax; ++q) {
    const int gi = g0 + kLevelsPerOctave * q + 2 * lane + sh * kLevelsPerOctave;  // even
    const bool ok = q < nwo && gi >= 0 && gi + 1 < kHistBins;
    v[q] = ok ? __ldcg(reinterpret_cast<const unsigned int*>(&h->fine[gi])) : 0u;
  }
#pragma unroll
  for (int q = 0; q < kFineOctMax; ++q) {
    c[2 * q] += v[q] & 0xffffu;
    c[2 * q + 1] += v[q] >> 16;
  }
}

__global__ void __launch_bounds__(kBThreads)
bracket_tc_kernel(const RangeHist* __restrict__ hist, const float* __restrict__ cmax,
                  RowBracket* __restrict__ brk, uint32_t* __restrict__ ready, Plan p) {
  // the histograms and maxima are complete; the value pass may be scheduled
  // from here on (after the logits pass, and so after the caller's kernels)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float s_mu[kBWarps][kMergeOct];
  __shared__ float s_deep[kBWarps], s_max[kBWarps];
  __shared__ uint32_t s_cnt[kFineOctMax * kLevelsPerOctave];
  __shared__ int s_olo, s_ohi;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = blockIdx.x;
  const int nr = p.nranges;
  const RangeHist* rh = hist + row * nr;
  for (int i = threadIdx.x; i < kFineOctMax * kLevelsPerOctave; i += kBThreads) s_cnt[i] = 0u;

  // (1) loads of the first kBPre ranges of this warp, and the row maximum
  RangeHead pre[kBPre];
#pragma unroll
  for (int i = 0; i < kBPre; ++i) pre[i] = load_head(rh + min(warp + kBWarps * i, nr - 1));
  float M = kNegInf;
  for (int r = threadIdx.x; r < nr; r += kBThreads) M = fmaxf(M, __ldcg(cmax + row * p.nchunks + r));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) s_max[warp] = M;
  __syncthreads();
  M = s_max[0];
#pragma unroll
  for (int w = 1; w < kBWarps; ++w) M = fmaxf(M, s_max[w]);
  RowBracket out{M, INT_MIN, INT_MAX, 0u};  // default: every key is in the window
  const float XM = __fmul_rn(M, p.scale2);
  if (!(fabsf(XM) < 1.0e6f)) {  // non-finite rows: flagged by the logits pass
    if (threadIdx.x == 0) publish_bracket(brk + row, ready + row, out);
    return;
  }
  const int T = __float2int_ru(XM) * kLevelsPerOctave;
  const float delta = (float)((double)T / kLevelsPerOctave - (double)XM);  // in [0, 1)
  const float p_delta = exp2f(delta);

  // (2) merge this warp's ranges in range order
  bool bad = false;
  float mu[2] = {0.0f, 0.0f};
  float deep = 0.0f;  // upper bound of the mass of keys below the merged frame
#pragma unroll
  for (int i = 0; i < kBPre; ++i) {
    const int r = warp + kBWarps * i;
    if (r < nr) merge_range(rh + r, pre[i], T, p_delta, mu, deep, bad);
  }
  for (int r = warp + kBWarps * kBPre; r < nr; r += kBWarps)  // many ranges (large n)
    merge_range(rh + r, load_head(rh + r), T, p_delta, mu, deep, bad);
  s_mu[warp][lane] = mu[0];
  s_mu[warp][lane + 32] = mu[1];
  deep = warp_sum_f(deep);
  if (lane == 0) s_deep[warp] = deep;
  if (__syncthreads_or(bad)) {
    if (threadIdx.x == 0) publish_bracket(brk + row, ready + row, out);
    return;
  }

  // (3) warp 0: octave bounds and the window octaves
  const float slack = (fabsf(XM) + 2.0f * kMergeOct + 64.0f) * 0x1p-22f + 1.0e-4f;
  const float p_64 = exp2f(-1.0f / kLevelsPerOctave);
  const float eps = (float)p.eps;
  float loU = 0.0f, loL = 0.0f, upU = 0.0f, upL = 0.0f, ZU = 0.0f, ZL = 0.0f;
  int Olo = 0, Ohi = 0;
  if (warp == 0) {
    mu[0] = s_mu[0][lane];
    mu[1] = s_mu[0][lane + 32];
    deep = s_deep[0];
#pragma unroll
    for (int w = 1; w < kBWarps; ++w) {
      mu[0] += s_mu[w][lane];
      mu[1] += s_mu[w][lane + 32];
      deep += s_deep[w];
    }
    deep *= 1.0f + slack;
    // per-octave mass bounds; octave O holds weights 2^(delta - O - j/64) per unit of omass
    float hi_m[2], lo_m[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float f = p_delta * pow2f_int(-(lane + 32 * k));
      hi_m[k] = mu[k] * f * (1.0f + slack);
      lo_m[k] = mu[k] * f * p_64 * (1.0f - slack);
    }
    // suffix sums from the bottom of the frame: mass of octaves >= O
    upU = warp_suffix_sum_f(hi_m[1]);
    upL = warp_suffix_sum_f(lo_m[1]);
    const float totU1 = __shfl_sync(0xffffffffu, upU, 0), totL1 = __shfl_sync(0xffffffffu, upL, 0);
    loU = warp_suffix_sum_f(hi_m[0]) + totU1;
    loL = warp_suffix_sum_f(lo_m[0]) + totL1;
    ZU = __shfl_sync(0xffffffffu, loU, 0) + deep;
    ZL = __shfl_sync(0xffffffffu, loL, 0);
    // D+(O) <= eps ZL: the keys of octaves >= O are certainly dropped
    // D-(O) >  eps ZU: the keys of octaves <  O are certainly kept
    const uint32_t tail0 = __ballot_sync(0xffffffffu, loU + deep <= eps * ZL);
    const uint32_t tail1 = __ballot_sync(0xffffffffu, upU + deep <= eps * ZL);
    const uint32_t head0 = __ballot_sync(0xffffffffu, loL > eps * ZU);
    const uint32_t head1 = __ballot_sync(0xffffffffu, upL > eps * ZU);
    // smallest O with the tail condition (kMergeOct: only the deep keys;
    // kMergeOct + 1: none), largest O with the head condition (0 if none)
    Olo = tail0 ? __ffs(tail0) - 1 : tail1 ? 32 + __ffs(tail1) - 1
          : (deep <= eps * ZL ? kMergeOct : kMergeOct + 1);
    Ohi = head1 ? 32 + 31 - __clz(head1) : head0 ? 31 - __clz(head0) : 0;
    if (lane == 0) {
      s_olo = Olo;
      s_ohi = Ohi;
    }
  }
  __syncthreads();
  Olo = s_olo;
  Ohi = s_ohi;
  if (Olo <= Ohi) {  // cannot happen with consistent bounds; keep the default
    if (threadIdx.x == 0) publish_bracket(brk + row, ready + row, out);
    return;
  }
  int g_lo = kLevelsPerOctave * Olo, g_hi = kLevelsPerOctave * Ohi;  // the coarse result
  const int nwo = Olo - Ohi;
  const bool fine = Olo <= kMergeOct && nwo <= kFineOctMax;
  if (fine) {
    // (4) fine counts of the window bins [g0, g0 + 64 nwo)
    const int g0 = kLevelsPerOctave * Ohi;
    uint32_t c[2 * kFineOctMax];
#pragma unroll
    for (int b = 0; b < 2 * kFineOctMax; ++b) c[b] = 0u;
#pragma unroll
    for (int i = 0; i < kBPre; ++i) {
      const int r = warp + kBWarps * i;
      if (r < nr) fine_range(rh + r, (pre[i].top - T) / kLevelsPerOctave, g0, nwo, c);
    }
    for (int r = warp + kBWarps * kBPre; r < nr; r += kBWarps)
      fine_range(rh + r, (__ldcg(&rh[r].top) - T) / kLevelsPerOctave, g0, nwo, c);
#pragma unroll
    for (int q = 0; q < kFineOctMax; ++q) {
      if (q < nwo) {
        if (c[2 * q]) atomicAdd(&s_cnt[kLevelsPerOctave * q + 2 * lane], c[2 * q]);
        if (c[2 * q + 1]) atomicAdd(&s_cnt[kLevelsPerOctave * q + 2 * lane + 1], c[2 * q + 1]);
      }
    }
    __syncthreads();
    if (warp == 0) {
      // (5) lane l owns the B = 2 nwo consecutive window bins B l ... B l + B - 1
      const int B = 2 * nwo;
      const float baseU =
          (Olo < kMergeOct ? __shfl_sync(0xffffffffu, (Olo < 32 ? loU : upU), Olo & 31) : 0.0f) + deep;
      const float baseL =
          (Olo < kMergeOct) ? __shfl_sync(0xffffffffu, (Olo < 32 ? loL : upL), Olo & 31) : 0.0f;
      float bu[2 * kFineOctMax], bl[2 * kFineOctMax], su = 0.0f, sl = 0.0f;
#pragma unroll
      for (int b = 0; b < 2 * kFineOctMax; ++b) {
        const int g = g0 + B * lane + b;
        const float cnt = (b < B) ? (float)s_cnt[B * lane + b] : 0.0f;
        const float f = p_delta *
                        exp2f(-(float)(g & (kLevelsPerOctave - 1)) / (float)kLevelsPerOctave) *
                        pow2f_int(-(g / kLevelsPerOctave));
        bu[b] = cnt * f * (1.0f + slack);
        bl[b] = cnt * f * p_64 * (1.0f - slack);
        su += bu[b];
        sl += bl[b];
      }
      // mass of the window bins of the lanes above this one (larger g)
      const float aboveU = warp_suffix_sum_f(su) - su, aboveL = warp_suffix_sum_f(sl) - sl;
      // walk this lane's bins from its bottom (largest g) up
      float DU = baseU + aboveU, DL = baseL + aboveL;
      int my_lo = INT_MAX, my_hi = -1;
#pragma unroll
      for (int b = 2 * kFineOctMax - 1; b >= 0; --b) {
        DU += bu[b];
        DL += bl[b];
        const int g = g0 + B * lane + b;  // boundary at the top of bin g: keys with index >= g
        const bool in = b < B;
        my_lo = (in && DU <= eps * ZL) ? g : my_lo;
        my_hi = (in && DL > eps * ZU && my_hi < 0) ? g : my_hi;
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        my_lo = min(my_lo, __shfl_xor_sync(0xffffffffu, my_lo, o));
        my_hi = max(my_hi, __shfl_xor_sync(0xffffffffu, my_hi, o));
      }
      if (my_lo != INT_MAX) g_lo = min(g_lo, my_lo);
      if (my_hi >= 0) g_hi = max(g_hi, my_hi);
      if (g_lo <= g_hi) {  // inconsistent: fall back to the coarse window
        g_lo = kLevelsPerOctave * Olo;
        g_hi = kLevelsPerOctave * Ohi;
      }
    }
  }
  // keys with fine index >= g_lo (level <= T - g_lo) are dropped, keys with
  // fine index < g_hi (level > T - g_hi) are kept
  if (threadIdx.x == 0) {
    out.llo = (Olo > kMergeOct) ? INT_MIN : T - g_lo + 1;
    out.lhi = T - g_hi + 1;
    publish_bracket(brk + row, ready + row, out);
  }
}

template <int RT, bool ERR>
__global__ void __launch_bounds__(kGThreads, 1)
gather_tc_kernel(const __grid_constant__ CUtensorMap vmap, const float* __restrict__ u,
                 TcBufs tb, float* __restrict__ acc_out, Plan p,
                 uint32_t* __restrict__ status) {
  // the last kernel may be scheduled now; it waits for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* vring = base;                          // [kGStages][2 boxes][kGK keys][128 B]
  unsigned char* wring = base + kGStages * kGV;         // [kGStages][kGK / 64][kGN rows][128 B]
  float* uring = reinterpret_cast<float*>(wring + kGStages * kGW);  // [kGStages][4 rows][kGK]
  unsigned long long* cbuf_all =
      reinterpret_cast<unsigned long long*>(uring + kGStages * 4 * kGK);  // [8][kCandBuf]
  __shared__ unsigned long long vfull[kGStages], wfull[kGStages], empty[kGStages];
  // the logits of stage t land on ufull[t % 2][t % kGStages]: each of these
  // barriers serves one parity of stages, whose weight warps alone wait on it
  // and see every one of its phases (a parity wait is sound only then)
  __shared__ unsigned long long ufull[2][kGStages];
  __shared__ unsigned long long accfull[2], accempty[2], drain;
  __shared__ RecPart rpart[2][4];  // by item parity and row
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
      mbar_init(&ufull[0][s], 1);
      mbar_init(&ufull[1][s], 1);
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
      const unsigned long long pol_u = policy_evict_last();  // read again by the last kernel
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<unsigned long long>(&vmap))
                   : "memory");
      // The first ring of value stages goes out at once (the value rows do not
      // depend on the earlier kernels of the call).  (Prefetching the next
      // 6-24 stages into L2 as well made the step slower.)
      int nA = 0;
      for (int it = blockIdx.x; it < nitems && nA < kGStages; it += gridDim.x) {
        const GItem g = gitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        for (int sg = s_lo; sg < s_hi && nA < kGStages; ++sg, ++nA) {
          unsigned char* dst = vring + nA * kGV;
          mbar_arrive_expect_tx(&vfull[nA], (unsigned)kGV);
          tma_load_3d(dst, &vmap, 0, sg * kGK, g.group, &vfull[nA], pol);
          tma_load_3d(dst + kGV / 2, &vmap, kGBox, sg * kGK, g.group, &vfull[nA], pol);
        }
      }
      // (the logits are complete: see the weight warps)
      int t = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const GItem g = gitem_of(it, p);
        const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
        const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
        const int nrows = min(RT, p.gm - g.tile * RT);
        for (int sg = s_lo; sg < s_hi; ++sg, ++t) {
          const int slot = t % kGStages;
          if (t >= nA) {
            if (!mbar_wait(&empty[slot], (unsigned)(t / kGStages - 1) & 1u) || aborted(&s_abort)) {
              ok = false;
              break;
            }
            unsigned char* dst = vring + slot * kGV;
            mbar_arrive_expect_tx(&vfull[slot], (unsigned)kGV);
            tma_load_3d(dst, &vmap, 0, sg * kGK, g.group, &vfull[slot], pol);
            tma_load_3d(dst + kGV / 2, &vmap, kGBox, sg * kGK, g.group, &vfull[slot], pol);
          }
          // the rows' logits of the stage's keys below n, in whole 16-byte pieces
          // (the logit rows are padded to a multiple of 64 keys)
          const int64_t key0 = (int64_t)sg * kGK;
          const unsigned ub = (unsigned)((min((int64_t)kGK, p.n - key0) + 3) / 4) * 16u;
          unsigned long long* ub_bar = &ufull[t & 1][slot];
          mbar_arrive_expect_tx(ub_bar, ub * (unsigned)nrows);
          for (int r = 0; r < nrows; ++r)
            bulk_load(uring + (slot * 4 + r) * kGK, u + (row0 + r) * p.ustride + key0, ub,
                      ub_bar, pol_u);
        }
      }
      if (!ok) {
        atomicOr(status, CTA_DEV_TIMEOUT);
        s_abort = 1;
        // the copies still in flight land before the CTA may exit (bounded)
        for (int t2 = max(0, t - kGStages); t2 < t; ++t2) {
          mbar_wait(&vfull[t2 % kGStages], (unsigned)(t2 / kGStages) & 1u);
          mbar_wait(&ufull[t2 & 1][t2 % kGStages], (unsigned)(t2 / (2 * kGStages)) & 1u);
        }
        for (int t2 = t; t2 < nA; ++t2) mbar_wait(&vfull[t2], 0u);
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
  } else {
    // ---------------- weights (warps 2-9) and the accumulator ----------------
    // warp wi = warp - 2 serves row r = wi % 4 of the tile in the stages t of
    // parity h = wi / 4 (t counts the CTA's stages), so that two stages are in
    // the works at once; it reads tensor-memory lanes 32 (warp % 4) ... + 31.
    const int wi = warp - kGWeightWarp0;
    const int r = wi & 3, h = wi >> 2;
    const int quarter = warp & 3;
    const int dim = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    // No griddepcontrol.wait: this grid launches only after every bracket CTA
    // has passed its own wait for the logits pass, so the logits, histograms
    // and zeroed flags are complete; each row's bracket is waited for by flag.
    const float sc = p.scale2;
    int t = 0, jj = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++jj) {
      const GItem g = gitem_of(it, p);
      const int s_lo = g.range * p.rstages, s_hi = min(spu, s_lo + p.rstages);
      const int64_t row = (int64_t)g.group * p.gm + (int64_t)g.tile * RT + r;
      const int nrows = min(RT, p.gm - g.tile * RT);
      const bool row_ok = r < nrows;
      float M = 0.0f;
      int llo = INT_MIN, lhi = INT_MAX;
      if (row_ok) {
        if (!wait_bracket(tb.brk_ready + row)) ok = false;
        const RowBracket bk = ld_cg_bracket(tb.brk + row);
        M = bk.M;
        llo = bk.llo;
        lhi = bk.lhi;
      }
      U128 mz = u128_zero(), mh = u128_zero(), mt = u128_zero();
      double wh = 0.0, wt = 0.0;  // fp64 sums of per-stage fp32 weight sums (for KL only)
      uint32_t nh = 0u, nw = 0u;
      float tmax = kNegInf;
      unsigned long long* cand = tb.cand + row * kCandCap;
      unsigned long long* cbuf = cbuf_all + wi * kCandBuf;
      uint32_t nbuf = 0u;
      for (int sg = s_lo; sg < s_hi && ok; ++sg, ++t) {
        if (r >= RT || (t & 1) != h) continue;
        const int slot = t % kGStages;
        const int64_t k0 = (int64_t)sg * kGK + 4 * lane;  // this lane's four keys
        // the stage's logits have landed; its slot's W tile is then free too
        // (the MMAs that last read the slot have finished)
        if (!mbar_wait(&ufull[h][slot], (unsigned)(t / (2 * kGStages)) & 1u) || aborted(&s_abort))
          ok = false;
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          if (lane == 0) s_abort = 1;  // the other warps stop waiting too
          break;
        }
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row_ok) x = reinterpret_cast<const float4*>(uring + (slot * 4 + r) * kGK)[lane];
        uint32_t hp[4][3], tp[4][3];
        const float xs[4] = {x.x, x.y, x.z, x.w};
        uint32_t winmask = 0u, hbits = 0u;
        float sh_ = 0.0f, st_ = 0.0f;
        // branch-free: every key is kept (level >= lhi), dropped (< llo) or window
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const bool valid = row_ok && k0 + i < p.n;
          const float w = valid ? weight(xs[i], M, sc) : 0.0f;
          const int L = key_level(xs[i], sc);
          const bool head = valid && L >= lhi;
          const bool tail = valid && L < llo;
          const unsigned long long W = mass62(w);
          u128_add(mz, W);
          u128_add(mh, head ? W : 0ull);
          u128_add(mt, tail ? W : 0ull);
          nh += head ? 1u : 0u;
          hbits |= head ? (1u << i) : 0u;
          nw += (valid && !head && !tail) ? 1u : 0u;
          winmask |= (valid && !head && !tail) ? (1u << i) : 0u;
          sh_ += head ? w : 0.0f;
          st_ += tail ? w : 0.0f;
          tmax = fmaxf(tmax, tail ? xs[i] : kNegInf);
          uint32_t pt[3];
          split3(w, pt);
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            hp[i][part] = head ? pt[part] : 0u;
            if constexpr (ERR) tp[i][part] = tail ? pt[part] : 0u;
          }
        }
        wh += (double)sh_;
        wt += (double)st_;
        // the stage's kept-for-certain bits: lane l holds keys 4 l .. 4 l + 3,
        // i.e. bits 4 (l % 8) .. of word l / 8; eight lanes OR their nibbles
        {
          uint32_t wv = hbits << (4 * (lane & 7));
          wv |= __shfl_xor_sync(0xffffffffu, wv, 1);
          wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
          wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
          if (row_ok && (lane & 7) == 0) tb.hmask[row * tb.mask_words + 4 * (int64_t)sg + (lane >> 3)] = wv;
        }
        unsigned char* wtile = wring + slot * kGW;
        const int c = lane >> 1;  // 16-byte piece (8 keys) along K; this lane writes one half
        const uint32_t half = (uint32_t)(lane & 1) * 8u;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          *reinterpret_cast<uint2*>(wtile + sw128_offset(wcol<RT>(0, part, r), c, kGN) + half) =
              make_uint2(hp[0][part] | (hp[1][part] << 16), hp[2][part] | (hp[3][part] << 16));
          if constexpr (ERR)
            *reinterpret_cast<uint2*>(wtile + sw128_offset(wcol<RT>(1, part, r), c, kGN) + half) =
                make_uint2(tp[0][part] | (tp[1][part] << 16), tp[2][part] | (tp[3][part] << 16));
        }
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&wfull[slot]);
        // window keys to this warp's buffer (flushed to the row's list when
        // full and at the end of the item: one global atomic per flush)
        if (__any_sync(0xffffffffu, winmask != 0u)) {
          const uint32_t cnt = __popc(winmask);
          uint32_t pre = cnt;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, pre, o);
            if (lane >= o) pre += y;
          }
          const uint32_t total = __shfl_sync(0xffffffffu, pre, 31);
          if (nbuf + total > (uint32_t)kCandBuf) {
            flush_cands(cbuf, nbuf, cand, tb.cand_cnt + row);
            nbuf = 0u;
          }
          uint32_t at = nbuf + pre - cnt;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if (winmask & (1u << i)) cbuf[at++] = composite(order_key(xs[i]), (uint32_t)(k0 + i));
          }
          __syncwarp();
          nbuf += total;  // a stage adds at most 128 <= kCandBuf keys
        }
      }
      if (row_ok && __any_sync(0xffffffffu, nbuf > 0u)) {
        flush_cands(cbuf, nbuf, cand, tb.cand_cnt + row);
        nbuf = 0u;
      }
      // this warp's part of the range record (its stages); the warps of
      // parity 1 hand theirs over in shared memory
      const int b = jj & 1;
      mz = u128_warp_sum(mz);
      mh = u128_warp_sum(mh);
      mt = u128_warp_sum(mt);
      wh = warp_sum_d(wh);
      wt = warp_sum_d(wt);
      nh = __reduce_add_sync(0xffffffffu, nh);
      nw = __reduce_add_sync(0xffffffffu, nw);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      if (h == 1 && lane == 0) rpart[b][r] = RecPart{mz, mh, mt, wh, wt, nh, nw, tmax};
      // the accumulator of the item (all stages' MMAs done)
      const bool acc_ok = ok && mbar_wait(&accfull[b], (unsigned)(jj >> 1) & 1u) && !aborted(&s_abort);
      if (bar_red_or(kGEpiBar, kGEpiThreads, !acc_ok)) {
        ok = false;
        break;
      }
      if (h == 0 && row_ok && lane == 0) {
        const RecPart& o = rpart[b][r];
        u128_add(mz, o.mz);
        u128_add(mh, o.mh);
        u128_add(mt, o.mt);
        RangeRec rec;
        rec.mh = mh;
        rec.mt = mt;
        rec.mw = u128_sub(u128_sub(mz, mh), mt);
        rec.wh = wh + o.wh;
        rec.wt = wt + o.wt;
        rec.nh = nh + o.nh;
        rec.nw = nw + o.nw;
        rec.tmax = fmaxf(tmax, o.tmax);
        rec.pad = 0u;
        tb.rrec[row * p.nranges + g.range] = rec;
      }
      tc_fence_after();
      __syncwarp();
      uint32_t c[32];
      tc_ld32(lane_addr + (uint32_t)(b * kGN), c);
      tc_fence_before();
      mbar_arrive(&accempty[b]);
      // each warp of the lane quarter writes every other (row, kept/dropped) sum,
      // the three parts added in fp64, fixed order
      const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
      constexpr int NA = ERR ? 2 : 1;
#pragma unroll
      for (int x = 0; x < RT * NA; ++x) {
        const int rr = x / NA, a = x % NA;
        if ((x & 1) == h && rr < nrows) {
          const double v = ((double)__uint_as_float(c[wcol<RT>(a, 0, rr)]) +
                            (double)__uint_as_float(c[wcol<RT>(a, 1, rr)])) +
                           (double)__uint_as_float(c[wcol<RT>(a, 2, rr)]);
          acc_out[(((row0 + rr) * p.nranges + g.range) * 2 + a) * kGD + dim] = (float)v;
        }
      }
    }
    if (!ok && lane == 0) {
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

template <int RT, bool ERR>
cudaError_t launch_t(const CUtensorMap& map, const float* u, const TcBufs& tb,
                     float* acc, const Plan& p, uint32_t* status, cudaStream_t st) {
  auto kern = gather_tc_kernel<RT, ERR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGSmem);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const long long nitems = (long long)p.tiles_out * p.nranges * p.groups;
  const unsigned grid = (unsigned)std::min<long long>(nitems, sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kGThreads, 1, 1);
  cfg.dynamicSmemBytes = kGSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see "Ordering" above
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, u, tb, acc, p, status);
}

template <bool ERR>
cudaError_t launch_e(const CUtensorMap& map, const float* u, const TcBufs& tb,
                     float* acc, const Plan& p, uint32_t* status, cudaStream_t st) {
  switch (p.rt_out) {
    case 1: return launch_t<1, ERR>(map, u, tb, acc, p, status, st);
    case 2: return launch_t<2, ERR>(map, u, tb, acc, p, status, st);
    case 4: return launch_t<4, ERR>(map, u, tb, acc, p, status, st);
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

// The path depends on the shape and dtype alone, so that the workspace size
// is the same wherever it is computed; a missing tensor-map encoder makes the
// launch fail (CTA_ERR_CUDA) instead of choosing another path.
bool gather_tc_applies(const Plan& p, int dtype) {
  return dtype == kDtypeBF16 && p.d == kGD && p.n >= kGK && p.rt_out <= 4;
}

void set_ranges_tc(Plan* p, int sms) {
  const int64_t units = (int64_t)p->groups * p->tiles_out;
  const int64_t spu = (p->n + kGK - 1) / kGK;
  // range partials fit the workspace (one slot per chunk); at most 1024 ranges are tried
  const int64_t cap = std::min<int64_t>(std::min<int64_t>(spu, p->nchunks), 1024);
  // A work item ends with the accumulator hand-over and the range record
  // (about two stages of streaming), so the planner charges that much per item.
  constexpr int64_t kItemCost = 2;
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

cudaError_t launch_bracket_tc(const float* cmax, const TcBufs& tb, const Plan& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.rows, 1, 1);
  cfg.blockDim = dim3(kBThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bracket_tc_kernel, (const RangeHist*)tb.hist, cmax, tb.brk,
                            tb.brk_ready, p);
}

cudaError_t launch_gather_tc(const void* V, const float* u, const TcBufs& tb, float* acc,
                             const Plan& p, uint32_t* status, cudaStream_t st) {
  if (p.rstages < 1) return cudaErrorInvalidValue;
  CUtensorMap map;
  if (!encode_kv_map(&map, V, p)) return cudaErrorInvalidValue;
  return p.want_err ? launch_e<true>(map, u, tb, acc, p, status, st)
                    : launch_e<false>(map, u, tb, acc, p, status, st);
}

}  // namespace cta
