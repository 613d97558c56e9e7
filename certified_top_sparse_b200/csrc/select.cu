// Phase 2: certified selection.  One thread-block cluster per row.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): TV(P, P-hat) of the Top-k truncation
// equals the discarded softmax tail mass, and certified Top-k keeps the minimal
// k_eps with TV <= eps.  With the keys ranked by logit (descending; ties by
// the lower index), k_eps is the least k whose kept mass C_k satisfies
// (Z - C_k) / Z <= eps, Z the total mass.
//
// No sort of the row.  Every softmax numerator w = 2^-a (a >= 0, see weight()
// in common.cuh) becomes a 64-bit fixed-point integer W, so all mass sums are
// exact and independent of order and of how the row is split.  The row is
// split into CS contiguous segments (whole output chunks), one per CTA of a
// cluster (CS = 1..8); the CTAs exchange data through distributed shared
// memory with hardware cluster barriers only (no flag polling).
//   1. Counts per bin, bin = floor(64 a): bins are intervals of the ranking
//      and bin b holds weights in (2^-(b+1)/64, 2^-b/64], which bounds every
//      bin's mass from its count alone.
//   2. The merged counts bound the cumulative mass from above and below; the
//      cut lies in the window of bins [b1, b2] where the bounds do not decide.
//   3. One pass: exact Z, exact mass of the bins below the window (registers,
//      no atomics), the window's keys gathered as candidates, and per output
//      chunk the keys above the window (certainly kept).
//   4. CTA 0 takes every candidate, sums exact masses per sub-bin (1/64 of a
//      bin, still an interval of the ranking), finds the sub-bin that holds
//      the cut and sorts only its keys (logit desc, index asc); a prefix sum
//      of their exact masses gives the last kept key (K*, I*) and k_eps.
//   5. Per output chunk, the exclusive offset of its first kept index.
//   6. Each CTA writes the kept indices of its segment, ascending, from those
//      offsets (one warp per chunk, ballots of 32 keys), and its segment's
//      largest dropped logit (for the single-gap certificate).
// Alongside, the fp64 sums of the kept and of the dropped weights (the output
// normalisers): pass 3 sums the keys above and below the window, CTA 0 splits
// the window's candidates at the cut; every reduction has a fixed order.
// A window with more than 4096 keys (near-ties, e.g. all-equal logits) is
// first narrowed exactly by 8-bit radix digits of the composite key (logit
// order, then index); then the per-chunk counts come from a recount pass.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace cg = cooperative_groups;

namespace cta {

namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / kWarp;
constexpr int kCap = 4096;              // candidates sorted in shared memory
constexpr int kMaxCluster = 8;
constexpr int kSubPerBin = 64;          // sub-bins per bin: 4096 per halving of the weight
constexpr int kSub = 2048;              // sub-bins available (a window of up to 32 bins)
constexpr int kLocalChunks = 1024;      // per-CTA chunk counters kept in shared memory
constexpr int kIdxBatch = 20;           // 32-key words in flight per warp in the index pass
constexpr int kBinsPerThread = kBins / kSelThreads;
constexpr double kBoundSlack = 4e-6;    // covers exp2f's error (2 ulp) with margin
constexpr double kDecideSlack = 1e-9;   // covers fp64 rounding in the exact test
static_assert(kBins % kSelThreads == 0, "bins must split evenly over threads");
static_assert(kCap % kSelThreads == 0, "candidates must split evenly over threads");
static_assert(kSub % kSelThreads == 0, "sub-bins must split evenly over threads");
static_assert(kBins % kMaxCluster == 0, "bin slices must split evenly over the cluster");

struct SelShared {
  unsigned int cnt[kBins];          // this CTA's counts per bin
  unsigned int gcnt[kBins];         // the row's merged counts
  unsigned long long cand[kCap];    // this CTA's candidates; in CTA 0 later the sorted list
  unsigned long long mcand[kCap];   // CTA 0: the row's candidates
  unsigned long long sub_mass[kSub];  // CTA 0: exact mass per sub-bin of the window
  unsigned int sub_cnt[kSub];
  unsigned int lcc[kLocalChunks];   // certainly-kept keys per chunk of this segment
  unsigned long long dmass[256];    // radix narrowing: digit masses (this CTA)
  unsigned int dcnt[256];           //                  digit counts (this CTA)
  unsigned long long warp_buf[kSelWarps];
  unsigned long long warp_buf3[kSelWarps][3];
  double fwarp[kSelWarps][2];       // per-warp fp64 sums
  double fpart[2];                  // this CTA's fp64 weight sums: kept (above), dropped (below)
  double fsum[2];                   // block result of block_sum2
  unsigned long long zpart, tpart, wpart;  // this CTA's exact masses: all, below, window
  unsigned long long Z, T, Wn;      // the row's, summed over the cluster
  unsigned long long local_kept;    // kept keys in this CTA's segment (read by the cluster)
  unsigned long long offset;        // kept keys of the lower-ranked segments
  unsigned long long res_k;         // CTA 0: k_eps
  unsigned long long c_above, n_above, n_in_s;
  unsigned int res_kstar;           // CTA 0: order key of the last kept key
  unsigned int res_istar;           // CTA 0: its index
  unsigned int ncand;
  unsigned int n_in;
  unsigned int rcount[kMaxCluster + 1];  // CTA 0: candidate counts per rank, then prefix
  int b1, b2, pos;
  int row_shift;                    // fixed-point scale 2^row_shift of this row's exact masses
  float fbuf[kSelWarps];
};

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

// Exclusive scans of three 64-bit values per thread at once (three barriers);
// t[] gets the three block sums.
__device__ void block_scan_excl3(unsigned long long* v, unsigned long long* t, SelShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x[3] = {v[0], v[1], v[2]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, x[k], o);
      if (lane >= o) x[k] += y;
    }
  }
  if (lane == 31) {
#pragma unroll
    for (int k = 0; k < 3; ++k) S.warp_buf3[warp][k] = x[k];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      unsigned long long w = (lane < kSelWarps) ? S.warp_buf3[lane][k] : 0ull;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      if (lane < kSelWarps) S.warp_buf3[lane][k] = w;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    const unsigned long long before = warp ? S.warp_buf3[warp - 1][k] : 0ull;
    t[k] = S.warp_buf3[kSelWarps - 1][k];
    v[k] = before + x[k] - v[k];
  }
  __syncthreads();
}

__device__ unsigned long long block_sum(unsigned long long v, SelShared& S) {
  unsigned long long t;
  block_scan_excl(v, &t, S);
  return t;
}

// Fixed-order block sums of two fp64 values per thread (into S.fsum).
__device__ void block_sum2(double a, double b, SelShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
  if (lane == 0) { S.fwarp[warp][0] = a; S.fwarp[warp][1] = b; }
  __syncthreads();
  if (threadIdx.x == 0) {
    double x = 0.0, y = 0.0;
    for (int w = 0; w < kSelWarps; ++w) { x += S.fwarp[w][0]; y += S.fwarp[w][1]; }
    S.fsum[0] = x;
    S.fsum[1] = y;
  }
  __syncthreads();
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

__device__ __forceinline__ unsigned long long warp_sum(unsigned long long v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Visits the keys of [lo, hi) in warp-uniform groups: g(x[4], i, ok) gets four
// consecutive keys i..i+3 per lane (lane j of a warp holds keys 4j..4j+3 of a
// 128-key group; ok[e] says whether key i+e exists) with B 16-byte loads in
// flight per thread.  Every lane of a warp calls g the same number of times,
// so the lanes may vote; a group never straddles a 128-key boundary relative
// to lo.  Without 16-byte alignment each lane holds one key (x[1..3] absent).
template <int B, typename G>
__device__ __forceinline__ void for_each_quad(const float* __restrict__ ur, int64_t lo, int64_t hi,
                                              bool vec, G&& g) {
  if (vec) {
    const int64_t nv = (hi - lo) >> 2;
    const float4* p4 = reinterpret_cast<const float4*>(ur + lo);
    for (int64_t j0 = 0; j0 < nv; j0 += B * kSelThreads) {
      float4 x[B];
#pragma unroll
      for (int q = 0; q < B; ++q) {
        const int64_t j = j0 + q * kSelThreads + threadIdx.x;
        x[q] = (j < nv) ? p4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int q = 0; q < B; ++q) {
        const int64_t j = j0 + q * kSelThreads + threadIdx.x;
        const bool ok = j < nv;
        const float xs[4] = {x[q].x, x[q].y, x[q].z, x[q].w};
        const bool oks[4] = {ok, ok, ok, ok};
        g(xs, lo + 4 * j, oks);
      }
    }
    const int64_t t0 = lo + 4 * nv;  // < 4 leftover keys, one per lane of warp 0
    if (t0 < hi && threadIdx.x < 32) {
      const int64_t i = t0 + threadIdx.x;
      const float xs[4] = {i < hi ? ur[i] : 0.f, 0.f, 0.f, 0.f};
      const bool oks[4] = {i < hi, false, false, false};
      g(xs, i, oks);
    }
  } else {
    for (int64_t i0 = lo; i0 < hi; i0 += kSelThreads) {
      const int64_t i = i0 + threadIdx.x;
      const float xs[4] = {i < hi ? ur[i] : 0.f, 0.f, 0.f, 0.f};
      const bool oks[4] = {i < hi, false, false, false};
      g(xs, i, oks);
    }
  }
}

// Descending bitonic sort of a[0, P), P a power of two <= kCap.
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

// Rigorous fixed-point mass bounds of one key in bin b: 2^(shift - b/64) is
// evaluated with exp2f (exact argument: b/64 and shift are small dyadic
// numbers); the slack covers its 2-ulp error, the product's rounding and the
// weights' own exp2f error.
__device__ __forceinline__ unsigned long long bin_mass_hi(int b, int shift) {
  const float v = exp2f((float)shift - (float)b / kBinsPerOctave) * (float)(1.0 + kBoundSlack);
  return __float2ull_ru(v) + 1ull;
}
__device__ __forceinline__ unsigned long long bin_mass_lo(int b, int shift) {
  if (b >= kBins - 1) return 0ull;  // the last bin is open below
  const float v = exp2f((float)shift - (float)(b + 1) / kBinsPerOctave) * (float)(1.0 - kBoundSlack);
  const unsigned long long w = __float2ull_rd(v);
  return w > 0ull ? w - 1ull : 0ull;
}

__global__ void __launch_bounds__(kSelThreads, 2)
select_kernel(const float* __restrict__ u, const float* __restrict__ cmax, RowSel* __restrict__ sel,
              int32_t* __restrict__ k_out, float* __restrict__ tv_out,
              uint32_t* __restrict__ chunk_off, int32_t* __restrict__ idx_out,
              float* __restrict__ gmax, uint32_t* __restrict__ unit_cnt, Plan p,
              uint32_t* __restrict__ status) {
  // Launched as a programmatic dependent of the logits pass (which does not
  // trigger early, so this only saves the launch latency): wait for it, then
  // let the value pass launch (it streams values, which do not depend on this
  // kernel, and waits for its results before reading them).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelShared& S = *reinterpret_cast<SelShared*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int CS = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  SelShared* S0 = cluster.map_shared_rank(&S, 0);

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t row = blockIdx.x / CS;
  const int64_t n = p.n;
  const float* ur = u + row * p.ustride;
  // Segments are whole output chunks, so a chunk's count has one owner CTA.
  const int64_t seg = (((n + CS - 1) / CS + p.chunk - 1) / p.chunk) * p.chunk;
  const int64_t lo = min(n, (int64_t)rank * seg);
  const int64_t hi = min(n, lo + seg);
  const int c0 = (lo < hi) ? (int)(lo / p.chunk) : 0;  // an empty segment owns no chunk
  const int c1 = (lo < hi) ? (int)((hi + p.chunk - 1) / p.chunk) : 0;
  const bool local_cc = (c1 - c0) <= kLocalChunks;
  uint32_t* cc = chunk_off + row * p.nchunks;
  const bool vec = (n & 3) == 0;
  const float s2 = p.scale2;
  const uint32_t chunk = (uint32_t)p.chunk;

  // The output pass counts finished ranges per (KV group, row tile): zeroed
  // here by the tile's first row.
  if (rank == 0 && tid == 0 && (row % p.gm) % p.rt_out == 0)
    unit_cnt[(row / p.gm) * p.tiles_out + (row % p.gm) / p.rt_out] = 0u;

  // Row maximum from the partial maxima of phase 1 (same in every CTA).
  float M = kNegInf;
  for (int c = tid; c < p.nmax; c += kSelThreads) M = fmaxf(M, cmax[row * p.nchunks + c]);
  M = block_max(M, S);

  for (int i = tid; i < kBins; i += kSelThreads) S.cnt[i] = 0u;
  for (int c = tid; c < kLocalChunks; c += kSelThreads) S.lcc[c] = 0u;
  for (int c = c0 + tid; c < c1; c += kSelThreads) cc[c] = 0u;
  if (tid == 0) {
    S.ncand = 0u; S.n_in = 0u; S.b1 = kBins; S.b2 = kBins; S.pos = kCap;
    S.zpart = S.tpart = S.wpart = S.local_kept = 0ull;
  }
  __syncthreads();

  // ---- 1. counts per bin ------------------------------------------------------
  for_each_quad<8>(ur, lo, hi, vec, [&](const float* x, int64_t, const bool* ok) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (ok[e]) atomicAdd(&S.cnt[weight_bin(weight_arg(x[e], M, s2))], 1u);
  });
  cluster.sync();

  // ---- merge: slice r summed by CTA r, then gathered by everyone -------------
  const int per = kBins / CS;
  for (int b = rank * per + tid; b < (rank + 1) * per; b += kSelThreads) {
    unsigned int v[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) v[r] = (r < CS) ? cluster.map_shared_rank(&S, r)->cnt[b] : 0u;
    unsigned int c = 0u;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) c += v[r];
    S.gcnt[b] = c;
  }
  cluster.sync();
  {
    unsigned int v[kBinsPerThread];
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = tid + j * kSelThreads;
      const int owner = b / per;
      v[j] = (owner != rank) ? cluster.map_shared_rank(&S, owner)->gcnt[b] : 0u;
    }
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = tid + j * kSelThreads;
      if (b / per != rank) S.gcnt[b] = v[j];
    }
  }
  __syncthreads();

  // ---- 2. window of bins [b1, b2] that holds the cut --------------------------
  {
    unsigned long long lo_m[kBinsPerThread], hi_m[kBinsPerThread], cn[kBinsPerThread];
    unsigned long long lsum = 0ull, hsum = 0ull, csum = 0ull;
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = tid * kBinsPerThread + j;
      cn[j] = S.gcnt[b];
      lo_m[j] = cn[j] * bin_mass_lo(b, p.mass_shift);
      hi_m[j] = cn[j] * bin_mass_hi(b, p.mass_shift);
      lsum += lo_m[j];
      hsum += hi_m[j];
      csum += cn[j];
    }
    unsigned long long sc[3] = {lsum, hsum, csum}, tot[3];
    block_scan_excl3(sc, tot, S);
    const unsigned long long ZL = tot[0], ZU = tot[1];
    // The exact masses below use the scale 2^row_shift with Z * 2^row_shift
    // <= 2^62: every sum fits 64 bits and the rounding of the n weights moves
    // the total by at most n * 2^-(row_shift + 1) <= n * 2^-62 * Z_upper, a
    // relative error of at most n * 2^-61 (<= 2^-33 for n <= 2^28), whatever
    // the spread of the weights.  (One scale for every row, fixed by n alone,
    // would lose up to n^2 * 2^-63 of the mass.)
    if (tid == 0) {
      const int e = ilogb((double)ZU * ldexp(1.0, -p.mass_shift)) + 1;  // Z_upper < 2^e
      S.row_shift = min(62, 62 - max(e, 0));
    }
    unsigned long long CL = sc[0], CU = sc[1], CN = sc[2];
    const double e_hi = p.eps * (1.0 - kDecideSlack), e_lo = p.eps * (1.0 + kDecideSlack);
    unsigned long long cn_before[kBinsPerThread];
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = tid * kBinsPerThread + j;
      cn_before[j] = CN;
      CN += cn[j];
      CL += lo_m[j];
      CU += hi_m[j];
      const double TL = (double)(ZL - CL), TU = (double)(ZU - CU);
      // TV after bin b lies in [TL / (CU + TL), TU / (CL + TU)]
      if (TU <= e_hi * ((double)CL + TU)) atomicMin(&S.b2, b);          // certainly certified
      if (!(TL > e_lo * ((double)CU + TL))) atomicMin(&S.b1, b);        // not certainly uncertified
    }
    __syncthreads();
    const int b2 = min(S.b2, kBins - 1);
    const int b1 = min(S.b1, b2);
#pragma unroll
    for (int j = 0; j < kBinsPerThread; ++j) {
      const int b = tid * kBinsPerThread + j;
      if (b == b1) S.n_above = cn_before[j];                 // keys in bins above b1
      if (b == b2) S.n_in_s = cn_before[j] + cn[j];          // keys in bins up to b2
    }
    __syncthreads();
  }
  const int b2 = min(S.b2, kBins - 1);
  const int b1 = min(S.b1, b2);
  unsigned long long n_above = S.n_above;
  unsigned long long n_in = S.n_in_s - n_above;
  const float two_s = ldexpf(1.0f, S.row_shift);
  const bool direct = n_in <= (unsigned long long)kCap;

  // ---- 3. exact masses, candidates, certainly-kept counts per chunk -----------
  {
    unsigned long long z = 0ull, t = 0ull, wn = 0ull;
    double fa = 0.0, fb = 0.0;  // fp64 weight sums above / below the window
    for_each_quad<4>(ur, lo, hi, vec, [&](const float* x, int64_t i, const bool* ok) {
      unsigned int above = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = weight_arg(x[e], M, s2);
        const int b = weight_bin(a);
        const float w = ok[e] ? exp2f(-a) : 0.0f;
        const unsigned long long W = fixed_mass(w, two_s);
        z += W;
        if (b > b2) { t += W; fb += (double)w; }
        else if (b >= b1) wn += W;
        else fa += (double)w;
        if (direct && ok[e]) {
          if (b < b1) ++above;
          else if (b <= b2) {
            const unsigned int slot = atomicAdd(&S.ncand, 1u);
            if (slot < (unsigned)kCap) S.cand[slot] = composite(order_key(x[e]), (uint32_t)(i + e));
          }
        }
      }
      if (direct) {
        const unsigned int tot = __reduce_add_sync(0xffffffffu, above);
        if (lane == 0 && tot) {
          const uint32_t c = (uint32_t)i / chunk;  // the whole group lies in this chunk
          if (local_cc) atomicAdd(&S.lcc[c - c0], tot);
          else atomicAdd(&cc[c], tot);
        }
      }
    });
    z = warp_sum(z);
    t = warp_sum(t);
    wn = warp_sum(wn);
    if (lane == 0) {
      atomicAdd(&S.zpart, z);
      atomicAdd(&S.tpart, t);
      atomicAdd(&S.wpart, wn);
    }
    block_sum2(fa, fb, S);
    if (tid == 0) { S.fpart[0] = S.fsum[0]; S.fpart[1] = S.fsum[1]; }
    if (direct && local_cc)
      for (int c = c0 + tid; c < c1; c += kSelThreads) cc[c] = S.lcc[c - c0];
  }
  cluster.sync();
  if (warp == 0) {
    unsigned long long z = 0ull, t = 0ull, wn = 0ull;
    if (lane < CS) {
      const SelShared* R = cluster.map_shared_rank(&S, lane);
      z = R->zpart;
      t = R->tpart;
      wn = R->wpart;
    }
    z = warp_sum(z);
    t = warp_sum(t);
    wn = warp_sum(wn);
    if (lane == 0) { S.Z = z; S.T = t; S.Wn = wn; }
  }
  __syncthreads();
  const unsigned long long Z = S.Z;
  unsigned long long c_above = Z - S.T - S.Wn;  // exact mass of the bins above the window

  // ---- radix narrowing of an oversized window (exact, rare) -------------------
  int level = 0;
  unsigned long long prefix = 0ull;
  if (!direct) {
    while (n_in > (unsigned long long)kCap && level < 8) {
      cluster.sync();  // the previous digit histograms have been read
      for (int i = tid; i < 256; i += kSelThreads) { S.dmass[i] = 0ull; S.dcnt[i] = 0u; }
      if (tid == 0) S.pos = 256;
      __syncthreads();
      const int shift = 56 - 8 * level;
      for_each_quad<4>(ur, lo, hi, vec, [&](const float* x, int64_t i, const bool* ok) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = weight_arg(x[e], M, s2);
          const int b = weight_bin(a);
          if (!ok[e] || b < b1 || b > b2) continue;
          const unsigned long long ck = composite(order_key(x[e]), (uint32_t)(i + e));
          if (level > 0 && (ck >> (64 - 8 * level)) != prefix) continue;
          const int dig = (int)((ck >> shift) & 0xffull);
          atomicAdd(&S.dmass[dig], fixed_mass(exp2f(-a), two_s));
          atomicAdd(&S.dcnt[dig], 1u);
        }
      });
      cluster.sync();
      // digits in descending order: thread t < 256 owns digit 255 - t
      unsigned long long dm = 0ull, dc = 0ull;
      if (tid < 256) {
        for (int r = 0; r < CS; ++r) {
          const SelShared* R = cluster.map_shared_rank(&S, r);
          dm += R->dmass[255 - tid];
          dc += R->dcnt[255 - tid];
        }
      }
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
      if (S.pos == 256) {  // cannot happen for finite rows
        if (tid == 0 && rank == 0) atomicOr(status, CTA_DEV_INTERNAL);
        break;
      }
      prefix = (prefix << 8) | (unsigned long long)S.pos;
      c_above = S.c_above;
      n_above = S.n_above;
      n_in = S.n_in;
      ++level;
      __syncthreads();
    }
    for_each_quad<4>(ur, lo, hi, vec, [&](const float* x, int64_t i, const bool* ok) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int b = weight_bin(weight_arg(x[e], M, s2));
        if (!ok[e] || b < b1 || b > b2) continue;
        const unsigned long long ck = composite(order_key(x[e]), (uint32_t)(i + e));
        if (level > 0 && (ck >> (64 - 8 * level)) != prefix) continue;
        const unsigned int slot = atomicAdd(&S.ncand, 1u);
        if (slot < (unsigned)kCap) S.cand[slot] = ck;
      }
    });
    cluster.sync();
  }

  // ---- 4. CTA 0: narrow the candidates by sub-bin, sort, find the exact cut ----
  if (rank == 0) {
    // pull every CTA's candidates into mcand (parallel shared-memory reads)
    if (tid < CS) S.rcount[tid] = min(cluster.map_shared_rank(&S, tid)->ncand, (unsigned)kCap);
    __syncthreads();
    if (tid == 0) {
      unsigned int acc = 0u;
      for (int r = 0; r < CS; ++r) { const unsigned int c = S.rcount[r]; S.rcount[r] = acc; acc += c; }
      S.rcount[CS] = acc;
    }
    __syncthreads();
    const int nc = (int)min(S.rcount[CS], (unsigned)kCap);
    for (int i = tid; i < nc; i += kSelThreads) {
      int r = 0;
      while (r + 1 < CS && (unsigned)i >= S.rcount[r + 1]) ++r;
      S.mcand[i] = cluster.map_shared_rank(&S, r)->cand[i - S.rcount[r]];
    }
    if (tid == 0 && (unsigned long long)nc != n_in) atomicOr(status, CTA_DEV_INTERNAL);
    __syncthreads();  // every thread has read the candidate counts
    if (tid == 0) { S.ncand = 0u; S.pos = kSub; }
    __syncthreads();

    // The list to sort, and the mass and count of the keys ranked above it.
    const unsigned long long* src = S.mcand;
    unsigned long long* srt = S.cand;
    int m = nc;
    unsigned long long base_mass = c_above, base_cnt = n_above;
    double wk = 0.0, wd = 0.0;  // fp64 weights of the window's kept / dropped candidates
    const int nsub = (b2 - b1 + 1) * kSubPerBin;
    if (direct && nsub <= kSub) {
      for (int i = tid; i < nsub; i += kSelThreads) { S.sub_mass[i] = 0ull; S.sub_cnt[i] = 0u; }
      __syncthreads();
      const float top = (float)(b1 * kSubPerBin + nsub - 1);
      auto sub_of = [&](float a) {
        return max(0, (int)fminf(a * (kBinsPerOctave * kSubPerBin), top) - b1 * kSubPerBin);
      };
      for (int i = tid; i < nc; i += kSelThreads) {
        const float a = weight_arg(key_value((uint32_t)(S.mcand[i] >> 32)), M, s2);
        const int sb = sub_of(a);
        atomicAdd(&S.sub_mass[sb], fixed_mass(exp2f(-a), two_s));
        atomicAdd(&S.sub_cnt[sb], 1u);
      }
      __syncthreads();
      constexpr int SPT = kSub / kSelThreads;
      unsigned long long ms[SPT], msum = 0ull, csum = 0ull;
      unsigned int cs[SPT];
#pragma unroll
      for (int j = 0; j < SPT; ++j) {
        const int sb = tid * SPT + j;
        ms[j] = sb < nsub ? S.sub_mass[sb] : 0ull;
        cs[j] = sb < nsub ? S.sub_cnt[sb] : 0u;
        msum += ms[j];
        csum += cs[j];
      }
      unsigned long long sc[3] = {msum, csum, 0ull}, stot[3];
      block_scan_excl3(sc, stot, S);
      unsigned long long cum = c_above + sc[0];
      unsigned long long cnt_before = sc[1];
      // The certificate holds from one sub-bin on (the cumulative mass only
      // grows): only the thread whose sub-bins contain the change searches.
      if (!certified(Z, cum, p.eps) && certified(Z, cum + msum, p.eps)) {
#pragma unroll
        for (int j = 0; j < SPT; ++j) {
          const int sb = tid * SPT + j;
          if (sb < nsub && certified(Z, cum + ms[j], p.eps)) {
            S.pos = sb;
            S.c_above = cum;            // mass ranked above the sub-bin
            S.n_above = cnt_before;     // window keys ranked above it
            break;
          }
          cum += ms[j];
          cnt_before += cs[j];
        }
      }
      __syncthreads();
      const int sstar = S.pos;
      if (sstar < nsub) {
        base_mass = S.c_above;
        base_cnt = n_above + S.n_above;
        // keys of the cut sub-bin to sort; keys of the sub-bins above are kept
        for (int i = tid; i < nc; i += kSelThreads) {
          const unsigned long long ck = S.mcand[i];
          const float a = weight_arg(key_value((uint32_t)(ck >> 32)), M, s2);
          const int sb = sub_of(a);
          if (sb == sstar) {
            const unsigned int slot = atomicAdd(&S.ncand, 1u);
            S.cand[slot] = ck;
          } else if (sb < sstar) {
            atomicAdd(&cc[(0xffffffffu - (uint32_t)(ck & 0xffffffffull)) / chunk], 1u);
            wk += (double)exp2f(-a);
          } else {
            wd += (double)exp2f(-a);
          }
        }
        __syncthreads();
        m = (int)S.ncand;
        src = S.cand;
        srt = S.mcand;
      } else if (tid == 0) {
        atomicOr(status, CTA_DEV_NONFINITE);  // no sub-bin passes: only for non-finite rows
      }
      __syncthreads();
    }
    // sort src[0, m) into srt, descending (composite keys are unique)
    if (m <= 2 * kSelThreads) {
      unsigned long long v[2];
      int rk[2] = {0, 0};
#pragma unroll
      for (int h = 0; h < 2; ++h) v[h] = (tid + h * kSelThreads < m) ? src[tid + h * kSelThreads] : 0ull;
      for (int j = 0; j < m; ++j) {
        const unsigned long long c = src[j];
        rk[0] += c > v[0];
        rk[1] += c > v[1];
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (tid + h * kSelThreads < m) srt[rk[h]] = v[h];
    } else {
      int P = 1;
      while (P < m) P <<= 1;
      for (int i = tid; i < P; i += kSelThreads) srt[i] = i < m ? src[i] : 0ull;  // pad below all keys
      __syncthreads();
      bitonic_sort_desc(srt, P);
    }
    if (m == 0 && tid == 0) srt[0] = 0ull;
    if (tid == 0) S.pos = kCap;
    __syncthreads();

    constexpr int E = kCap / kSelThreads;  // consecutive sorted keys per thread
    unsigned long long wloc[E], wsum = 0ull;
    float wfl[E];
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const int i = tid * E + j;
      wfl[j] = (i < m) ? weight(key_value((uint32_t)(srt[i] >> 32)), M, s2) : 0.0f;
      wloc[j] = fixed_mass(wfl[j], two_s);
      wsum += wloc[j];
    }
    unsigned long long tmp;
    unsigned long long cum = base_mass + block_scan_excl(wsum, &tmp, S);
    // as for the sub-bins: the certificate changes once along the sorted keys
    if (!certified(Z, cum, p.eps) && certified(Z, cum + wsum, p.eps)) {
#pragma unroll
      for (int j = 0; j < E; ++j) {
        const int i = tid * E + j;
        if (i < m && certified(Z, cum + wloc[j], p.eps)) {
          S.pos = i;
          S.c_above = cum + wloc[j];  // kept mass C_k
          break;
        }
        cum += wloc[j];
      }
    }
    __syncthreads();
    int pos = S.pos;
    const bool ok = pos < m;
    if (!ok) {  // only for non-finite rows; keep every index in bounds
      if (tid == 0) atomicOr(status, CTA_DEV_NONFINITE);
      pos = m > 0 ? m - 1 : 0;  // srt[0] is the zero pad when m == 0
    }
    const unsigned long long thr = srt[pos];
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const int i = tid * E + j;
      if (i <= pos) wk += (double)wfl[j]; else wd += (double)wfl[j];
    }
    block_sum2(wk, wd, S);
    if (direct) {  // kept keys of the sorted list, per chunk
      for (int i = tid; i <= pos && i < m; i += kSelThreads) {
        const uint32_t idx = 0xffffffffu - (uint32_t)(srt[i] & 0xffffffffull);
        atomicAdd(&cc[idx / chunk], 1u);
      }
    }
    // the CTAs' fp64 sums of the weights above / below the window: loaded by
    // warp 0 in parallel, added in rank order
    double fa_row = 0.0, fb_row = 0.0;
    if (warp == 0) {
      double x0 = 0.0, x1 = 0.0;
      if (lane < CS) {
        const SelShared* R = cluster.map_shared_rank(&S, lane);
        x0 = R->fpart[0];
        x1 = R->fpart[1];
      }
      for (int q = 0; q < CS; ++q) {
        fa_row += __shfl_sync(0xffffffffu, x0, q);
        fb_row += __shfl_sync(0xffffffffu, x1, q);
      }
    }
    if (tid == 0) {
      long long k = (long long)base_cnt + pos + 1;
      if (k > n) k = n;
      const unsigned long long C = ok ? S.c_above : Z;
      S.res_kstar = (uint32_t)(thr >> 32);
      S.res_istar = 0xffffffffu - (uint32_t)(thr & 0xffffffffull);
      S.res_k = (unsigned long long)k;
      RowSel r;
      r.M = M;
      r.kstar = S.res_kstar;
      r.istar = (int32_t)S.res_istar;
      r.k = (int32_t)k;
      r.Z = Z;
      r.C = C;
      r.tv = Z ? (double)(Z - C) / (double)Z : 0.0;
      // kept = above the window + the window's kept candidates; dropped likewise
      // (an oversized window recomputes both in the recount pass below)
      r.wh = fa_row + S.fsum[0];
      r.wt = fb_row + S.fsum[1];
      sel[row] = r;
      k_out[row] = (int32_t)k;
      tv_out[row] = (float)r.tv;
    }
  }
  cluster.sync();

  // ---- 5. per-chunk offsets of the kept indices ------------------------------
  const uint32_t kstar = S0->res_kstar;
  const uint32_t istar = S0->res_istar;
  const unsigned long long k_total = S0->res_k;
  if (!direct) {  // recount: kept keys per chunk, and both weight sums, from the threshold
    double fk = 0.0, fd = 0.0;
    for_each_quad<4>(ur, lo, hi, vec, [&](const float* x, int64_t i, const bool* ok) {
      unsigned int kept = 0u;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (!ok[e]) continue;
        const bool k = is_kept(order_key(x[e]), (uint32_t)(i + e), kstar, istar);
        const double w = (double)weight(x[e], M, s2);
        if (k) { ++kept; fk += w; } else { fd += w; }
      }
      const unsigned int tot = __reduce_add_sync(0xffffffffu, kept);
      if (lane == 0 && tot) atomicAdd(&cc[(uint32_t)i / chunk], tot);
    });
    block_sum2(fk, fd, S);
    if (tid == 0) { S.fpart[0] = S.fsum[0]; S.fpart[1] = S.fsum[1]; }
    __syncthreads();
  }
  // exclusive scan over this CTA's chunks (in blocks of kSelThreads chunks)
  unsigned long long run = 0ull;
  for (int cb = c0; cb < c1; cb += kSelThreads) {
    const int c = cb + tid;
    const unsigned long long v = (c < c1) ? __ldcg(cc + c) : 0ull;
    run += block_sum(v, S);
  }
  if (tid == 0) S.local_kept = run;
  cluster.sync();
  if (warp == 0) {
    unsigned long long o = (lane < rank) ? cluster.map_shared_rank(&S, lane)->local_kept : 0ull;
    o = warp_sum(o);
    if (lane == 0) S.offset = o;
  }
  if (!direct && rank == 0 && tid == 0) {  // the recount's weight sums, in rank order
    double fk = 0.0, fd = 0.0;
    for (int q = 0; q < CS; ++q) {
      const SelShared* R = cluster.map_shared_rank(&S, q);
      fk += R->fpart[0];
      fd += R->fpart[1];
    }
    sel[row].wh = fk;
    sel[row].wt = fd;
  }
  cluster.sync();  // no CTA reads another's shared memory after this point
  unsigned long long offset = S.offset;
  if (tid == 0 && rank == CS - 1 && offset + run != k_total) atomicOr(status, CTA_DEV_INTERNAL);
  for (int cb = c0; cb < c1; cb += kSelThreads) {
    const int c = cb + tid;
    const unsigned long long v = (c < c1) ? __ldcg(cc + c) : 0ull;
    unsigned long long tot;
    const unsigned long long ex = block_scan_excl(v, &tot, S);
    if (c < c1) cc[c] = (uint32_t)(offset + ex);
    offset += tot;
  }
  __syncthreads();  // this CTA's chunk offsets are written

  // ---- 6. the kept indices of this segment, ascending ------------------------
  // One warp per chunk: a running position from the chunk's offset, 32 keys
  // per ballot, kIdxBatch words of logits in flight (they are still in L2).
  int32_t* dst = idx_out + row * n;
  float dmax = kNegInf;  // the largest dropped logit of this CTA's segment
  for (int c = c0 + warp; c < c1; c += kSelWarps) {
    const int64_t k0 = (int64_t)c * chunk;
    const int nkc = (int)min((int64_t)chunk, n - k0);
    uint32_t pos = __ldcg(cc + c);
    for (int w0 = 0; w0 < nkc; w0 += kWarp * kIdxBatch) {
      float x[kIdxBatch];
#pragma unroll
      for (int b = 0; b < kIdxBatch; ++b) {
        const int i = w0 + b * kWarp + lane;
        x[b] = i < nkc ? __ldcg(ur + k0 + i) : 0.0f;
      }
#pragma unroll
      for (int b = 0; b < kIdxBatch; ++b) {
        const int i = w0 + b * kWarp + lane;
        const bool kept = i < nkc && is_kept(order_key(x[b]), (uint32_t)(k0 + i), kstar, istar);
        if (i < nkc && !kept) dmax = fmaxf(dmax, x[b]);
        const uint32_t m = __ballot_sync(0xffffffffu, kept);
        if (kept) {
          const uint32_t at = pos + __popc(m & ((1u << lane) - 1u));
          if (at < (uint32_t)n) dst[at] = (int32_t)(k0 + i);
        }
        pos += __popc(m);
      }
    }
  }
  dmax = block_max(dmax, S);
  if (tid == 0) gmax[row * kMaxGParts + rank] = dmax;
}

}  // namespace

cudaError_t launch_select(const float* u, const float* cmax, RowSel* sel, int32_t* k_out,
                          float* tv_out, uint32_t* chunk_off, int32_t* idx_out, float* gmax,
                          uint32_t* unit_cnt, const Plan& p, uint32_t* status, cudaStream_t st) {
  const size_t smem = sizeof(SelShared);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.rows * p.sel_cluster), 1, 1);
  cfg.blockDim = dim3(kSelThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)p.sel_cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see the kernel's first lines
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, select_kernel, u, cmax, sel, k_out, tv_out, chunk_off, idx_out, gmax,
                         unit_cnt, p, status);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace cta
