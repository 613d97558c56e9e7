// Phase 2: certified selection, one CTA per row.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): TV(P, P-hat) of the Top-k truncation
// equals the discarded softmax tail mass, and certified Top-k keeps the minimal
// k_eps with TV <= eps.  With the keys ranked by logit (descending; ties by
// the lower index), k_eps is the least k whose kept mass C_k satisfies
// (Z - C_k) / Z <= eps, Z the total mass.
//
// No sort of the row.  Every softmax numerator w_i = exp((u_i - max u) / sqrt d)
// becomes a 64-bit fixed-point integer W_i, so all mass sums are exact and do
// not depend on order.  Pass 1 builds a histogram of mass and count over value
// bins of the logit (bins are intervals of the ranking) and locates the bin
// that holds the cut.  Pass 2 gathers that bin's keys (normally a few hundred)
// and sorts them by (logit desc, index asc); a prefix sum of their masses
// gives the exact cut, i.e. the last kept key (K*, I*).  When the bin holds
// more keys than shared memory, 8-bit radix digits of the composite key
// (logit order, then index) narrow it first: this is exact for any input,
// including ties.  Pass 3 writes the kept indices in ascending order.
#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kBins = 2048;             // value bins per row
constexpr float kBinsPerUnit = 64.0f;   // bins per unit of scaled logit (range 32)
constexpr int kCap = 4096;              // candidates sorted in shared memory
constexpr int kItems = 8;               // keys per thread per compaction step
constexpr int kBinsPerThread = kBins / kSelThreads;
static_assert(kBins % kSelThreads == 0, "bins must split evenly over threads");
static_assert(kCap % kSelThreads == 0, "candidates must split evenly over threads");

struct SelShared {
  unsigned long long mass[kBins];
  unsigned int cnt[kBins];
  unsigned long long cand[kCap];
  unsigned long long warp_buf[kSelWarps];
  unsigned long long c_above;
  unsigned long long n_above;
  unsigned int n_in;
  unsigned int ncand;
  int bstar;
  int pos;
  float fbuf[kSelWarps];
};

__device__ __forceinline__ int value_bin(float x, float M, float binscale) {
  // (M - x) >= 0 for every finite logit.  The clamp keeps non-finite rows
  // (M = -inf, NaN differences) inside [0, kBins).
  const float t = __fmul_rn(__fsub_rn(M, x), binscale);
  return (int)fminf(fmaxf(t, 0.0f), (float)(kBins - 1));
}

// Exclusive scan of one 64-bit value per thread; *total gets the block sum.
__device__ unsigned long long block_scan_excl(unsigned long long v, unsigned long long* total,
                                              SelShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) S.warp_buf[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = (lane < kSelWarps) ? S.warp_buf[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kSelWarps) S.warp_buf[lane] = w;
  }
  __syncthreads();
  const unsigned long long before = warp ? S.warp_buf[warp - 1] : 0ull;
  *total = S.warp_buf[kSelWarps - 1];
  __syncthreads();
  return before + x - v;
}

__device__ float block_max(float v, SelShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) S.fbuf[warp] = v;
  __syncthreads();
  float r = S.fbuf[0];
  for (int w = 1; w < kSelWarps; ++w) r = fmaxf(r, S.fbuf[w]);
  __syncthreads();
  return r;
}

// Keys of the current candidate set: in bin bstar and, after `level` radix
// digits, with the top 8*level bits of the composite key equal to prefix.
__device__ __forceinline__ bool in_set(float x, unsigned long long ck, int b, int bstar, int level,
                                       unsigned long long prefix) {
  if (b != bstar) return false;
  return level == 0 || (ck >> (64 - 8 * level)) == prefix;
}

// Descending bitonic sort of S.cand[0, P), P a power of two <= kCap.
__device__ void bitonic_sort_desc(unsigned long long* a, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P / 2; i += kSelThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == desc) { a[lo] = y; a[hi] = x; }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const float* __restrict__ u, const float* __restrict__ cmax, RowSel* __restrict__ sel,
              int32_t* __restrict__ k_out, float* __restrict__ tv_out,
              int32_t* __restrict__ idx_out, Plan p, uint32_t* __restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelShared& S = *reinterpret_cast<SelShared*>(smem_raw);
  const int tid = threadIdx.x;
  const int64_t row = blockIdx.x;
  const int64_t n = p.n;
  const float* ur = u + row * n;

  // Row maximum from the per-chunk maxima of phase 1.
  float M = kNegInf;
  for (int c = tid; c < p.nchunks; c += kSelThreads) M = fmaxf(M, cmax[row * p.nchunks + c]);
  M = block_max(M, S);
  const float binscale = __fmul_rn(p.scale, kBinsPerUnit);

  // ---- pass 1: mass and count per value bin ---------------------------------
  for (int i = tid; i < kBins; i += kSelThreads) { S.mass[i] = 0ull; S.cnt[i] = 0u; }
  if (tid == 0) {
    S.bstar = kBins; S.pos = kCap; S.ncand = 0u;
    S.c_above = 0ull; S.n_above = 0ull; S.n_in = 0u;
  }
  __syncthreads();
  for (int64_t i = tid; i < n; i += kSelThreads) {
    const float x = ur[i];
    const int b = value_bin(x, M, binscale);
    atomicAdd(&S.mass[b], fixed_mass(weight(x, M, p.scale), p.two_s));
    atomicAdd(&S.cnt[b], 1u);
  }
  __syncthreads();

  unsigned long long Z;
  {
    unsigned long long m_loc[kBinsPerThread], m_tot = 0ull, c_tot = 0ull;
    unsigned int c_loc[kBinsPerThread];
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      m_loc[j] = S.mass[tid * kBinsPerThread + j];
      c_loc[j] = S.cnt[tid * kBinsPerThread + j];
      m_tot += m_loc[j];
      c_tot += c_loc[j];
    }
    unsigned long long n_tot;
    unsigned long long m_ex = block_scan_excl(m_tot, &Z, S);
    unsigned long long c_ex = block_scan_excl(c_tot, &n_tot, S);
    int found = -1;
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      if (found < 0 && certified(Z, m_ex + m_loc[j], p.eps)) found = j;
      if (found < 0) { m_ex += m_loc[j]; c_ex += c_loc[j]; }
    }
    if (found >= 0) atomicMin(&S.bstar, tid * kBinsPerThread + found);
    __syncthreads();
    if (found >= 0 && tid * kBinsPerThread + found == S.bstar) {
      S.c_above = m_ex;
      S.n_above = c_ex;
      S.n_in = c_loc[found];
    }
    __syncthreads();
  }
  const int bstar = S.bstar;  // kBins only if no bin passes: a non-finite row
  if (tid == 0 && bstar == kBins) atomicOr(status, CTA_DEV_NONFINITE);
  unsigned long long c_above = S.c_above;
  unsigned long long n_above = S.n_above;
  unsigned int n_in = S.n_in;
  __syncthreads();

  // ---- radix narrowing of an oversized boundary bin (exact, rare) ------------
  int level = 0;
  unsigned long long prefix = 0ull;
  while (n_in > (unsigned)kCap && level < 8) {
    for (int i = tid; i < 256; i += kSelThreads) { S.mass[i] = 0ull; S.cnt[i] = 0u; }
    if (tid == 0) S.pos = 256;
    __syncthreads();
    const int shift = 56 - 8 * level;
    for (int64_t i = tid; i < n; i += kSelThreads) {
      const float x = ur[i];
      const int b = value_bin(x, M, binscale);
      const unsigned long long ck = composite(order_key(x), (uint32_t)i);
      if (!in_set(x, ck, b, bstar, level, prefix)) continue;
      const int dig = (int)((ck >> shift) & 0xffull);
      atomicAdd(&S.mass[dig], fixed_mass(weight(x, M, p.scale), p.two_s));
      atomicAdd(&S.cnt[dig], 1u);
    }
    __syncthreads();
    // Digits in descending order: thread t < 256 owns digit 255 - t.
    const unsigned long long dm = (tid < 256) ? S.mass[255 - tid] : 0ull;
    const unsigned long long dc = (tid < 256) ? S.cnt[255 - tid] : 0ull;
    unsigned long long tmp;
    const unsigned long long m_ex = block_scan_excl(dm, &tmp, S);
    const unsigned long long c_ex = block_scan_excl(dc, &tmp, S);
    const bool hit = tid < 256 && certified(Z, c_above + m_ex + dm, p.eps) &&
                     !certified(Z, c_above + m_ex, p.eps);
    if (hit) {
      S.pos = 255 - tid;
      S.c_above = c_above + m_ex;
      S.n_above = n_above + c_ex;
      S.n_in = (unsigned int)dc;
    }
    __syncthreads();
    if (S.pos == 256) {  // cannot happen: the whole set satisfies the test
      if (tid == 0) atomicOr(status, CTA_DEV_INTERNAL);
      break;
    }
    prefix = (prefix << 8) | (unsigned long long)S.pos;
    c_above = S.c_above;
    n_above = S.n_above;
    n_in = S.n_in;
    ++level;
    __syncthreads();
  }

  // ---- pass 2: gather the candidate set, sort it, cut it ---------------------
  if (tid == 0) { S.ncand = 0u; S.pos = kCap; }
  __syncthreads();
  for (int64_t i = tid; i < n; i += kSelThreads) {
    const float x = ur[i];
    const int b = value_bin(x, M, binscale);
    if (b != bstar) continue;
    const unsigned long long ck = composite(order_key(x), (uint32_t)i);
    if (!in_set(x, ck, b, bstar, level, prefix)) continue;
    const unsigned int slot = atomicAdd(&S.ncand, 1u);
    if (slot < (unsigned)kCap) S.cand[slot] = ck;
  }
  __syncthreads();
  const int nc = (int)min(S.ncand, (unsigned)kCap);
  if (tid == 0 && S.ncand != n_in) atomicOr(status, CTA_DEV_INTERNAL);
  int P = 1;
  while (P < nc) P <<= 1;
  for (int i = nc + tid; i < P; i += kSelThreads) S.cand[i] = 0ull;  // below every real key
  __syncthreads();
  bitonic_sort_desc(S.cand, P);

  // Masses in rank order; each thread owns E consecutive candidates.
  constexpr int E = kCap / kSelThreads;
  unsigned long long wloc[E], wsum = 0ull;
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const int i = tid * E + j;
    unsigned long long w = 0ull;
    if (i < nc) w = fixed_mass(weight(key_value((uint32_t)(S.cand[i] >> 32)), M, p.scale), p.two_s);
    wloc[j] = w;
    wsum += w;
  }
  unsigned long long tmp;
  unsigned long long cum = c_above + block_scan_excl(wsum, &tmp, S);
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const int i = tid * E + j;
    if (i < nc && certified(Z, cum + wloc[j], p.eps) && !certified(Z, cum, p.eps)) {
      S.pos = i;
      S.c_above = cum + wloc[j];  // kept mass C_k
    }
    cum += wloc[j];
  }
  __syncthreads();
  int pos = S.pos;
  if (pos >= nc) {  // only for non-finite rows; keep every index in bounds
    if (tid == 0) atomicOr(status, bstar == kBins ? CTA_DEV_NONFINITE : CTA_DEV_INTERNAL);
    pos = nc > 0 ? nc - 1 : 0;  // cand[0] is the zero pad when nc == 0
  }
  const unsigned long long thr = S.cand[pos];
  const uint32_t kstar = (uint32_t)(thr >> 32);
  const uint32_t istar = 0xffffffffu - (uint32_t)(thr & 0xffffffffull);
  const unsigned long long C = (S.pos < nc) ? S.c_above : Z;
  long long k = (long long)n_above + pos + 1;
  if (k > n) k = n;
  if (tid == 0) {
    RowSel r;
    r.M = M;
    r.kstar = kstar;
    r.istar = (int32_t)istar;
    r.k = (int32_t)k;
    r.Z = Z;
    r.C = C;
    r.tv = (double)(Z - C) / (double)Z;
    sel[row] = r;
    k_out[row] = (int32_t)k;
    tv_out[row] = (float)r.tv;
  }

  // ---- pass 3: kept indices, ascending ---------------------------------------
  int32_t* dst = idx_out + row * n;
  unsigned long long written = 0ull;
  for (int64_t base = 0; base < n; base += (int64_t)kSelThreads * kItems) {
    const int64_t i0 = base + (int64_t)tid * kItems;
    unsigned int flags = 0u;
    int cnt = 0;
#pragma unroll
    for (int j = 0; j < kItems; ++j) {
      const int64_t i = i0 + j;
      if (i < n && is_kept(order_key(ur[i]), (uint32_t)i, kstar, istar)) {
        flags |= 1u << j;
        ++cnt;
      }
    }
    unsigned long long tot;
    unsigned long long off = written + block_scan_excl((unsigned long long)cnt, &tot, S);
#pragma unroll
    for (int j = 0; j < kItems; ++j)
      if (flags & (1u << j)) dst[off++] = (int32_t)(i0 + j);
    written += tot;
  }
  if (tid == 0 && written != (unsigned long long)k) atomicOr(status, CTA_DEV_INTERNAL);
}

}  // namespace

cudaError_t launch_select(const float* u, const float* cmax, RowSel* sel, int32_t* k_out,
                          float* tv_out, int32_t* idx_out, const Plan& p, uint32_t* status,
                          cudaStream_t st) {
  const size_t smem = sizeof(SelShared);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<<<(unsigned)p.rows, kSelThreads, smem, st>>>(u, cmax, sel, k_out, tv_out, idx_out,
                                                            p, status);
  return cudaGetLastError();
}

}  // namespace cta
