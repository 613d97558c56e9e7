// Phase 2 for short rows (n <= 1024, e.g. all-query self-attention): one warp
// per row, the row's logits in registers.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): certified Top-k keeps the minimal
// k_eps whose discarded softmax mass (Z - C_k) / Z is <= eps, keys ranked by
// logit (descending; ties by the lower index).
//
// The same exact arithmetic as the cluster selection: every weight w = 2^-a
// (see weight() in common.cuh) becomes a 64-bit fixed-point integer, so every
// mass sum is exact.  Per row:
//   1. M = the row maximum, Z, and per key its exponent a;
//   2. three levels of 64-bin histograms (bins floor(a), floor(64 a),
//      floor(4096 a): intervals of the ranking; counts and masses in shared
//      memory with 32-bit atomics, four copies against contention), each followed by a
//      warp scan that finds the bin holding the cut;
//   3. that bin's keys (almost always one or two) are taken in descending
//      composite order (logit, then lower index) by repeated warp maxima until
//      the kept mass is certified: that key is the last kept one (K*, I*);
//   4. the fp64 sums of the kept and dropped weights, the largest dropped
//      logit, and the kept indices, ascending, written with ballots of 32 keys.
#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kShortWarps = 8;
constexpr int kHist = 64;  // bins per histogram level

__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, v, o);
    v = y > v ? y : v;
  }
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <typename U>
__device__ __forceinline__ U warp_incl_scan(U v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const U y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

constexpr int kCopies = 4;  // histogram copies (lane % 4) against atomic contention
constexpr int kDigit = 21;  // masses are added as three 21-bit digits (32-bit atomics)

// One warp's histogram: per bin and copy, a count and three mass digits
// (copies of a bin in adjacent words, so they sit in different banks).  A
// digit sum over at most 1024 keys stays below 2^31.
struct Hist {
  unsigned int cnt[kHist][kCopies];
  unsigned int dig[3][kHist][kCopies];
};

__device__ __forceinline__ void hist_add(Hist& h, int bin, int cp, unsigned long long W) {
  constexpr unsigned long long mask = (1ull << kDigit) - 1ull;
  atomicAdd(&h.cnt[bin][cp], 1u);
  atomicAdd(&h.dig[0][bin][cp], (unsigned int)(W & mask));
  atomicAdd(&h.dig[1][bin][cp], (unsigned int)((W >> kDigit) & mask));
  atomicAdd(&h.dig[2][bin][cp], (unsigned int)(W >> (2 * kDigit)));
}


__device__ __forceinline__ void hist_bin(const Hist& h, int bin, unsigned long long* mass,
                                         unsigned long long* cnt) {
  unsigned long long d0 = 0ull, d1 = 0ull, d2 = 0ull, c = 0ull;
#pragma unroll
  for (int k = 0; k < kCopies; ++k) {
    c += h.cnt[bin][k];
    d0 += h.dig[0][bin][k];
    d1 += h.dig[1][bin][k];
    d2 += h.dig[2][bin][k];
  }
  *mass = d0 + (d1 << kDigit) + (d2 << (2 * kDigit));
  *cnt = c;
}

__device__ __forceinline__ void clear_hist(Hist& h, int lane) {
  unsigned int* w = &h.cnt[0][0];
  constexpr int words = (int)(sizeof(Hist) / sizeof(unsigned int));
#pragma unroll
  for (int i = lane; i < words; i += kWarp) w[i] = 0u;
}

// The bin (of kHist, two per lane in order) whose inclusion first certifies
// the kept mass, given the mass and count ranked above the histogram.  On
// return *before / *nbefore are the mass and count ranked above that bin.
__device__ __forceinline__ int cut_bin(const Hist& h, unsigned long long Z, double eps, int lane,
                                       unsigned long long* before, unsigned long long* nbefore) {
  unsigned long long m0, m1, c0, c1;
  hist_bin(h, 2 * lane, &m0, &c0);
  hist_bin(h, 2 * lane + 1, &m1, &c1);
  const unsigned long long incl = warp_incl_scan<unsigned long long>(m0 + m1, lane);
  const unsigned long long cincl = warp_incl_scan<unsigned long long>(c0 + c1, lane);
  const unsigned long long excl = *before + incl - m0 - m1;
  const unsigned long long cexcl = *nbefore + cincl - c0 - c1;
  const bool h0 = certified(Z, excl + m0, eps);
  const bool h1 = certified(Z, excl + m0 + m1, eps);
  const unsigned b1 = __ballot_sync(0xffffffffu, h1);
  const int L = b1 ? __ffs(b1) - 1 : 31;  // the last lane's bins always certify
  const bool first = __shfl_sync(0xffffffffu, h0, L);
  const unsigned long long ex = __shfl_sync(0xffffffffu, excl, L);
  const unsigned long long cx = __shfl_sync(0xffffffffu, cexcl, L);
  const unsigned long long mL0 = __shfl_sync(0xffffffffu, m0, L);
  const unsigned long long cL0 = __shfl_sync(0xffffffffu, c0, L);
  *before = first ? ex : ex + mL0;
  *nbefore = first ? cx : cx + cL0;
  return first ? 2 * L : 2 * L + 1;
}

// Latency-bound (a serial chain of scans and shuffles per row): as many rows
// in flight as registers allow, four CTAs per SM up to 16 keys per lane.
template <int NPL>
__global__ void __launch_bounds__(kShortWarps * kWarp, NPL <= 16 ? 4 : 1)
select_short_kernel(const float* __restrict__ u, RowSel* __restrict__ sel,
                    int32_t* __restrict__ k_out, float* __restrict__ tv_out,
                    int32_t* __restrict__ idx_out, float* __restrict__ gmax,
                    uint32_t* __restrict__ unit_cnt, Plan p, uint32_t* __restrict__ status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // as in the long-row kernel
  __shared__ Hist hist[kShortWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kShortWarps + warp;
  if (row >= p.rows) return;  // whole warps only; no block-wide barrier below
  const int n = (int)p.n;
  const float s2 = p.scale2, two_s = p.two_s;
  const float* ur = u + row * p.ustride;
  Hist& hw = hist[warp];
  const int cp = lane & (kCopies - 1);

  float x[NPL];
  float mx = kNegInf;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int i = j * kWarp + lane;
    x[j] = i < n ? ur[i] : kNegInf;
    mx = fmaxf(mx, x[j]);
  }
  const float M = warp_max_f(mx);
  const bool finite = isfinite(M);
  // the coarse histogram and Z in one loop (exponents recomputed where needed:
  // cheaper than holding them in registers)
  auto av = [&](int j) { return weight_arg(x[j], M, s2); };
  uint32_t live = 0u;  // bit j: key j * 32 + lane exists (later: lies in the current cut bin)
  clear_hist(hw, lane);
  __syncwarp();
  unsigned long long z = 0ull;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    if (j * kWarp + lane < n) {
      live |= 1u << j;
      const float a = av(j);
      const unsigned long long W = fixed_mass(exp2f(-a), two_s);
      z += W;
      hist_add(hw, (int)fminf(a, (float)(kHist - 1)), cp, W);  // a >= 0; NaN clamps too
    }
  }
  const unsigned long long Z = warp_sum_u64(z);
  __syncwarp();

  // ---- 1-2. three histogram levels narrow the cut to one bin of 1/4096 ------
  unsigned long long before = 0ull, nbefore = 0ull;
  if (finite && Z > 0ull) {
    const int b0 = cut_bin(hw, Z, p.eps, lane, &before, &nbefore);
    uint32_t in = 0u;
#pragma unroll
    for (int j = 0; j < NPL; ++j)
      if (((live >> j) & 1u) && (int)fminf(av(j), (float)(kHist - 1)) == b0) in |= 1u << j;
    live = in;
    // finer levels over the keys of the cut bin only: floor(64 a), floor(4096 a)
    int base = b0;
#pragma unroll 1
    for (int l = 1; l < 3; ++l) {
      const float scale = l == 1 ? (float)kHist : (float)(kHist * kHist);
      __syncwarp();
      clear_hist(hw, lane);
      __syncwarp();
#pragma unroll
      for (int j = 0; j < NPL; ++j)
        if ((live >> j) & 1u) {
          const float a = av(j);
          const int bb = min(max((int)(a * scale) - base * kHist, 0), kHist - 1);
          hist_add(hw, bb, cp, fixed_mass(exp2f(-a), two_s));
        }
      __syncwarp();
      const int bl = cut_bin(hw, Z, p.eps, lane, &before, &nbefore);
      in = 0u;
#pragma unroll
      for (int j = 0; j < NPL; ++j)
        if (((live >> j) & 1u) && min(max((int)(av(j) * scale) - base * kHist, 0), kHist - 1) == bl)
          in |= 1u << j;
      live = in;
      base = base * kHist + bl;
    }
  }

  // ---- 3. walk the cut bin in descending composite order -------------------
  const uint32_t inmask = live;  // bit j: key j * 32 + lane lies in the cut bin
  unsigned long long cum = before, kk = nbefore, last = ~0ull, K = 0ull;
  bool done = !(finite && Z > 0ull);
  for (int guard = 0; !done && guard < n; ++guard) {
    unsigned long long best = 0ull;
#pragma unroll
    for (int j = 0; j < NPL; ++j) {
      if ((inmask >> j) & 1u) {
        const unsigned long long ck = composite(order_key(x[j]), (uint32_t)(j * kWarp + lane));
        if (ck < last && ck > best) best = ck;
      }
    }
    best = warp_max_u64(best);
    if (best == 0ull) break;  // no key left: cannot happen for finite rows
    K = best;
    last = best;
    cum += fixed_mass(exp2f(-weight_arg(key_value((uint32_t)(best >> 32)), M, s2)), two_s);
    ++kk;
    done = certified(Z, cum, p.eps);
  }

  uint32_t kstar, istar;
  if (done && K != 0ull) {
    kstar = (uint32_t)(K >> 32);
    istar = 0xffffffffu - (uint32_t)(K & 0xffffffffull);
  } else {  // non-finite row: keep every key, flag it
    if (lane == 0) atomicOr(status, CTA_DEV_NONFINITE);
    kstar = 0u;
    istar = 0xffffffffu;
    kk = (unsigned long long)n;
    cum = Z;
  }

  // ---- 4. weight sums and the kept indices ---------------------------------
  double fh = 0.0, fd = 0.0;
  float dmax = kNegInf;  // the largest dropped logit
  int32_t* dst = idx_out + row * n;
  uint32_t pos = 0u;
#pragma unroll
  for (int j = 0; j < NPL; ++j) {
    const int i = j * kWarp + lane;
    bool kept = false;
    if (i < n) {
      kept = is_kept(order_key(x[j]), (uint32_t)i, kstar, istar);
      const double w = (double)exp2f(-av(j));
      if (kept) fh += w; else { fd += w; dmax = fmaxf(dmax, x[j]); }
    }
    const uint32_t m = __ballot_sync(0xffffffffu, kept);
    if (kept) {
      const uint32_t at = pos + __popc(m & ((1u << lane) - 1u));
      if (at < (uint32_t)n) dst[at] = (int32_t)i;
    }
    pos += __popc(m);
  }
  fh = warp_sum_f64(fh);
  fd = warp_sum_f64(fd);
  dmax = warp_max_f(dmax);
  if (lane == 0) {
    if (pos != (uint32_t)kk) atomicOr(status, CTA_DEV_INTERNAL);
    RowSel r;
    r.M = M;
    r.kstar = kstar;
    r.istar = (int32_t)istar;
    r.k = (int32_t)kk;
    r.Z = Z;
    r.C = cum;
    r.tv = Z ? (double)(Z - cum) / (double)Z : 0.0;
    r.wh = fh;
    r.wt = fd;
    sel[row] = r;
    k_out[row] = (int32_t)kk;
    tv_out[row] = (float)r.tv;
    gmax[row * kMaxGParts] = dmax;
    // the output pass counts finished ranges per (KV group, row tile)
    if ((row % p.gm) % p.rt_out == 0)
      unit_cnt[(row / p.gm) * p.tiles_out + (row % p.gm) / p.rt_out] = 0u;
  }
}

template <int NPL>
cudaError_t launch_short_t(const float* u, RowSel* sel, int32_t* k_out, float* tv_out,
                           int32_t* idx_out, float* gmax, uint32_t* unit_cnt, const Plan& p,
                           uint32_t* status, cudaStream_t st) {
  const unsigned grid = (unsigned)((p.rows + kShortWarps - 1) / kShortWarps);
  select_short_kernel<NPL><<<grid, kShortWarps * kWarp, 0, st>>>(u, sel, k_out, tv_out, idx_out,
                                                                 gmax, unit_cnt, p, status);
  return cudaGetLastError();
}

}  // namespace

bool select_short_applies(const Plan& p) { return p.n <= (int64_t)kShortMaxN; }

cudaError_t launch_select_short(const float* u, RowSel* sel, int32_t* k_out, float* tv_out,
                                int32_t* idx_out, float* gmax, uint32_t* unit_cnt, const Plan& p,
                                uint32_t* status, cudaStream_t st) {
  const int npl = (int)((p.n + kWarp - 1) / kWarp);
#define CTA_SHORT(N) launch_short_t<N>(u, sel, k_out, tv_out, idx_out, gmax, unit_cnt, p, status, st)
  if (npl <= 1) return CTA_SHORT(1);
  if (npl <= 2) return CTA_SHORT(2);
  if (npl <= 4) return CTA_SHORT(4);
  if (npl <= 8) return CTA_SHORT(8);
  if (npl <= 16) return CTA_SHORT(16);
  if (npl <= 32) return CTA_SHORT(32);
#undef CTA_SHORT
  return cudaErrorInvalidValue;
}

}  // namespace cta
