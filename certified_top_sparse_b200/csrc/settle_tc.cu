// Kernel 4 of the tensor-core decode path (bf16 values, d = 128): the exact
// cut, the kept indices and the outputs of every row.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the keys ranked by logit
// (descending; ties by the lower index), k_eps is the least k whose kept mass
// C_k satisfies (Z - C_k) / Z <= eps; the output is Attn_k = mu_head, the
// error tau ||mu_tail - mu_head||_2 with tau = TV = (Z - C_k) / Z, and
// KL(P-hat || P) = log(Z / C_k).
//
// The value pass has already summed the values and exact masses of the keys
// whose side of the cut its bracket decided (kept: level >= lhi; dropped:
// level < llo), marked the kept-for-certain keys in a bit mask and listed the
// keys between (the window) as candidates.  One CTA per (row, segment of
// Plan::settle_group value-pass ranges):
//   1. Inputs: the row's candidate list and the segment's mask words come in
//      by bulk copies (one mbarrier); row totals from the range records: Z,
//      the dropped mass D below the window, the window mass W and the kept
//      count.  The bracket is checked exactly: D / Z <= eps < (D + W) / Z must
//      hold, i.e. the cut lies in the window.  (If it did not - which the
//      bracket's rigorous bounds exclude - the row is recomputed here from the
//      logits alone, with every key treated as a window key, and
//      CTA_DEV_INTERNAL is set.)
//   2. The exact cut.  Usually all the window's keys are in the candidate
//      list (composite keys: logit order, then index).  Every CTA of the row
//      sums their exact 2^-62 masses per sub-level (1/4096 of a halving of the
//      weight, an interval of the ranking), finds the sub-level where the
//      certificate starts to hold, sorts only that sub-level's keys and walks
//      them to the last kept key.  Otherwise (cold paths, out of line: a
//      window wider than the sub-level table, more window keys than the list
//      holds, e.g. many tied logits) a full sort of the list, or a radix
//      select over the 64-bit composite keys of the window, eight bits per
//      pass over the row's logits, with exact 128-bit digit masses.
//   3. The segment: its window keys' value rows (bulk copies, issued before
//      the cut search) added to the kept or dropped side, with the weight sums
//      for KL and the largest dropped logit; its kept indices, ascending, at
//      the offset of the kept keys before it: the mask words OR the kept
//      window keys, compacted in shared memory and written by bulk stores
//      (staging areas taking turns).  Without a usable candidate list the
//      segment's logits are scanned instead (cold path).
//   4. The last CTA of the row (a ticket counter that the logits pass zeroes)
//      adds the range partials in a fixed order and writes out, err, KL, k,
//      TV and the single-gap bound.  The output normalisers are the exact
//      kept and dropped masses; KL comes from the independent weight sums.
// Launched as a programmatic dependent of the value pass; it waits for that
// grid before it reads anything.
#include <climits>

#include "common.cuh"
#include "finalize.cuh"  // single_gap_bound
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kTThreads = 256;
constexpr int kTWarps = kTThreads / kWarp;
constexpr int kTD = 128;                 // head dimension
constexpr int kChunk = 4 * kTThreads;    // keys per chunk: four consecutive keys per thread
constexpr int kBatch = 8;                // chunks whose logits are in flight together
constexpr int kMaxGroup = 32;            // value-pass ranges per CTA
constexpr int kSubMax = 512;             // sub-level bins of the cut search
constexpr int kSubList = 256;            // keys of the cut's sub-level that are sorted
constexpr int kWList = 256;              // per-warp list of window keys awaiting their value rows
constexpr int kMaskBlock = 4 * kTThreads;  // mask words per block of the index writes (4 per thread)
constexpr int kVPre = 128;               // window value rows copied in while the cut is searched
constexpr int kStageWords = 124;         // mask words per staging round (124 x 32 + 3 <= 4096 slots)

static_assert(kCandCap * 2 >= kStageWords * 32 + 3 && kVPre * kTD / 2 >= 2 * kStageWords * 32 + 3 &&
                  kTWarps * kWList * 2 >= kStageWords * 32 + 3,
              "the candidate list, the window rows and the flat list double as the staging areas");

struct SettleShared {
  alignas(16) unsigned long long cand[kCandCap];  // the row's candidates (sorted in place by the fallback)
  union {
    struct {
      unsigned long long lo[kSubMax], hi[kSubMax];  // exact sub-level masses, 128-bit
      uint32_t cnt[kSubMax];
      unsigned long long list[kSubList];            // keys of the cut's sub-level
      unsigned long long sorted[kSubList];
    } sb;
    struct {
      unsigned long long lo[256], hi[256];  // radix digit masses, 128-bit
      uint32_t cnt[256];
    } rx;
    struct {
      uint32_t win[kMaskBlock];   // kept window keys of a block of mask words
      uint32_t word[kMaskBlock];  // kept keys of the block
      uint32_t off[kMaskBlock];   // exclusive offsets of the words' kept keys
    } mk;
  } u;
  alignas(16) uint32_t mask0[kMaskBlock];  // the segment's first block of kept-for-certain words
  alignas(16) uint2 vrow[kVPre][kTD / 4];  // value rows of the segment's first window keys
  unsigned long long bar_in, bar_v;        // bulk copies: candidates and mask words; value rows
  unsigned long long wl_key[kTWarps][kWList];  // window key: logit bits (high 32) | index (low 32)
  unsigned char wl_kept[kTWarps][kWList];
  float accw[2][kTWarps][kTD];           // per-warp window value sums (kept, dropped)
  double wsw[2][kTWarps];                // per-warp window weight sums (for KL)
  float dmw[kTWarps];                    // per-warp largest dropped window logit
  U128 u128buf[kTWarps];
  uint32_t u32buf[kTWarps];
  unsigned long long pk[kTWarps][2];     // packed chunk counts of the block scan
  U128 Z, D, W, C, cum;
  uint32_t NH, NHbefore, NW, ccnt, cabove, nsl, off_win;
  unsigned long long cut;
  long long k;
  uint32_t nlist;
  int found, jstar, last;
};

// Bulk copy shared -> global (async proxy), its commit and waits.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_store(void* dst, const void* src, unsigned bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read2() {
  asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ U128 u128_make(unsigned long long lo, unsigned long long hi) {
  return U128{lo, hi};
}
__device__ __forceinline__ double warp_sum_dbl(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Exclusive scan of one 128-bit and one 32-bit value per thread over the block.
__device__ __noinline__ void block_excl_scan(U128& v, uint32_t& c, SettleShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  U128 x = v;
  uint32_t y = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    U128 t;
    t.lo = __shfl_up_sync(0xffffffffu, x.lo, o);
    t.hi = __shfl_up_sync(0xffffffffu, x.hi, o);
    const uint32_t yc = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) {
      u128_add(x, t);
      y += yc;
    }
  }
  if (lane == 31) {
    S.u128buf[warp] = x;
    S.u32buf[warp] = y;
  }
  __syncthreads();
  U128 before = u128_zero();
  uint32_t cb = 0u;
  for (int w = 0; w < warp; ++w) {
    u128_add(before, S.u128buf[w]);
    cb += S.u32buf[w];
  }
  __syncthreads();
  u128_add(before, u128_sub(x, v));  // exclusive within the warp
  v = before;
  c = cb + y - c;
}

// Exclusive scan of two packed 64-bit words per thread (four 16-bit counts
// each, no field overflows); tot gets the block totals.
__device__ __noinline__ void block_excl_scan_packed(unsigned long long* v, unsigned long long* tot,
                                       SettleShared& S) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x0 = v[0], x1 = v[1];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y0 = __shfl_up_sync(0xffffffffu, x0, o);
    const unsigned long long y1 = __shfl_up_sync(0xffffffffu, x1, o);
    if (lane >= o) {
      x0 += y0;
      x1 += y1;
    }
  }
  if (lane == 31) {
    S.pk[warp][0] = x0;
    S.pk[warp][1] = x1;
  }
  __syncthreads();
  unsigned long long b0 = 0ull, b1 = 0ull, t0 = 0ull, t1 = 0ull;
  for (int w = 0; w < kTWarps; ++w) {
    if (w < warp) {
      b0 += S.pk[w][0];
      b1 += S.pk[w][1];
    }
    t0 += S.pk[w][0];
    t1 += S.pk[w][1];
  }
  __syncthreads();
  v[0] = b0 + x0 - v[0];
  v[1] = b1 + x1 - v[1];
  tot[0] = t0;
  tot[1] = t1;
}

// Descending bitonic sort of a[0, P), P a power of two <= kCandCap.
__device__ void bitonic_sort_desc(unsigned long long* a, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < P / 2; i += kTThreads) {
        const int lo = 2 * i - (i & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const unsigned long long x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      __syncthreads();
    }
  }
}

__device__ __forceinline__ bool in_window(float x, float sc, int llo, int lhi) {
  const int L = key_level(x, sc);
  return L >= llo && L < lhi;
}

// Sub-level of a logit: ceil(4096 x), x = fl(u * scale2); ceil(sub / 64) is
// its level, so the sub-levels of a level are 64 intervals of the ranking.
__device__ __forceinline__ int key_sublevel(float u, float scale2) {
  float x = __fmul_rn(u, scale2);
  x = fminf(fmaxf(x, -1.0e5f), 1.0e5f);
  return __float2int_ru(x * 4096.0f);
}

__device__ __forceinline__ float ck_logit(unsigned long long ck) {
  return key_value((uint32_t)(ck >> 32));
}

// Cold path of the cut search: the whole candidate list sorted (bitonic) and
// walked from the top.  Sets S.cut, S.C, S.k and S.found; returns S.found.
__device__ __noinline__ bool cut_by_sort(SettleShared& S, int m, float M, float sc, uint32_t NH,
                                         U128 Z, U128 base, double eps) {
  const int tid = threadIdx.x;
  // the whole candidate list sorted, then walked from the top
  int P = 1;
  while (P < m) P <<= 1;
  for (int i = m + tid; i < P; i += kTThreads) S.cand[i] = 0ull;  // pad below all keys
  __syncthreads();
  bitonic_sort_desc(S.cand, P);
  constexpr int E = kCandCap / kTThreads;
  unsigned long long Wl[E];
  U128 ls = u128_zero();
#pragma unroll
  for (int j = 0; j < E; ++j) {
    const int i = tid * E + j;
    Wl[j] = (i < m) ? mass62(weight(ck_logit(S.cand[i]), M, sc)) : 0ull;
    u128_add(ls, Wl[j]);
  }
  U128 cum = ls;
  uint32_t dummy = 0u;
  block_excl_scan(cum, dummy, S);
  u128_add(cum, base);
  U128 end = cum;
  u128_add(end, ls);
  if (!certified128(Z, cum, eps) && certified128(Z, end, eps)) {
#pragma unroll
    for (int j = 0; j < E; ++j) {
      const int i = tid * E + j;
      U128 nx = cum;
      u128_add(nx, Wl[j]);
      if (i < m && certified128(Z, nx, eps)) {
        S.C = nx;
        S.cut = S.cand[i];
        S.k = (long long)NH + i + 1;
        S.found = 1;
        break;
      }
      cum = nx;
    }
  }
  __syncthreads();
  return S.found != 0;
}

// Cold path of the cut search (candidate list overflowed or the bracket was
// rejected): radix select over the composite keys of the window's logits,
// eight bits per pass.  Sets S.cut, S.C and S.k.
__device__ __noinline__ void cut_by_radix(SettleShared& S, const float* __restrict__ ur, int64_t n,
                                          float M, float sc, int llo, int lhi, uint32_t NH, U128 Z,
                                          U128 base, double eps, uint32_t* __restrict__ status) {
  const int tid = threadIdx.x;
  // radix select over the window's composite keys, eight bits per pass
  unsigned long long prefix = 0ull;
  U128 bs = base;
  uint32_t above = 0u;
  bool ok = true;
  for (int level = 0; level < 8 && ok; ++level) {
    const int shift = 56 - 8 * level;
    for (int i = tid; i < 256; i += kTThreads) {
      S.u.rx.lo[i] = 0ull;
      S.u.rx.hi[i] = 0ull;
      S.u.rx.cnt[i] = 0u;
    }
    __syncthreads();
    for (int64_t key = tid; key < n; key += kTThreads) {
      const float x = __ldcg(ur + key);
      if (!in_window(x, sc, llo, lhi)) continue;
      const unsigned long long ck = composite(order_key(x), (uint32_t)key);
      if (level > 0 && (ck >> (64 - 8 * level)) != prefix) continue;
      const int dig = (int)((ck >> shift) & 0xffull);
      const unsigned long long w = mass62(weight(x, M, sc));
      const unsigned long long old = atomicAdd(&S.u.rx.lo[dig], w);
      if (old + w < old) atomicAdd(&S.u.rx.hi[dig], 1ull);
      atomicAdd(&S.u.rx.cnt[dig], 1u);
    }
    __syncthreads();
    // digits in descending order: thread t < 256 owns digit 255 - t
    U128 dm = u128_zero();
    uint32_t dc = 0u;
    if (tid < 256) {
      dm = u128_make(S.u.rx.lo[255 - tid], S.u.rx.hi[255 - tid]);
      dc = S.u.rx.cnt[255 - tid];
    }
    U128 mex = dm;
    uint32_t cex = dc;
    block_excl_scan(mex, cex, S);
    U128 before = bs;
    u128_add(before, mex);
    U128 after = before;
    u128_add(after, dm);
    if (tid == 0) S.found = 0;
    __syncthreads();
    if (tid < 256 && dc > 0u && !certified128(Z, before, eps) && certified128(Z, after, eps)) {
      S.jstar = 255 - tid;
      S.cum = before;
      S.cabove = above + cex;  // window keys ranked above this digit
      S.found = 1;
    }
    __syncthreads();
    if (!S.found) {
      ok = false;
      break;
    }
    prefix = (prefix << 8) | (unsigned long long)S.jstar;
    bs = S.cum;
    above = S.cabove;
    __syncthreads();
  }
  if (tid == 0) {
    if (!ok) {
      atomicOr(status, CTA_DEV_NONFINITE);  // only rows with non-finite weights get here
      prefix = 0ull;
    }
    S.cut = prefix;
    U128 c = bs;
    u128_add(c, mass62(weight(ck_logit(prefix), M, sc)));
    S.C = c;
    S.k = (long long)NH + above + 1;
  }
  __syncthreads();
}

// Partial sums of a segment's window keys (kept and dropped), their fp64
// weight sums and largest dropped logit, and the running output position.
struct WinSums {
  float ah[4], at[4];
  double whw, wtw;
  float dmx;
  uint32_t pos_out;
};

// Cold path of a segment (no usable candidate list): the segment's logits are
// scanned chunk by chunk; kept keys' indices are written in order and the
// window keys' value rows gathered through per-warp lists.
template <bool ERR>
__device__ __noinline__ WinSums settle_scan_segment(const float* __restrict__ ur,
                                                    const __nv_bfloat16* __restrict__ Vg,
                                                    int32_t* __restrict__ dst, int64_t n,
                                                    int64_t k_lo, int64_t k_hi, float M, float sc,
                                                    int llo, int lhi, uint32_t cut_key,
                                                    uint32_t cut_idx, uint32_t pos_out,
                                                    SettleShared& S) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float ah[4] = {0.f, 0.f, 0.f, 0.f}, at[4] = {0.f, 0.f, 0.f, 0.f};
  double whw = 0.0, wtw = 0.0;
  float dmx = kNegInf;
  auto gather_list = [&](const unsigned long long* keys, const unsigned char* kept, int first,
                         int end, int stride) {
    for (int e0 = first; e0 < end; e0 += 8 * stride) {
      uint2 v[8];
      float w8[8];
      int kp[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = e0 + q * stride;
        kp[q] = -1;
        w8[q] = 0.0f;
        v[q] = make_uint2(0u, 0u);
        if (e < end) {
          const unsigned long long lk = keys[e];
          const float x = __uint_as_float((uint32_t)(lk >> 32));
          w8[q] = weight(x, M, sc);
          kp[q] = kept[e];
          v[q] = __ldg(reinterpret_cast<const uint2*>(Vg + (int64_t)(uint32_t)lk * kTD) + lane);
          if (!kp[q]) dmx = fmaxf(dmx, x);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (kp[q] < 0) continue;
        const float2 a = bf16x2_to_float2(v[q].x), b = bf16x2_to_float2(v[q].y);
        if (kp[q]) {
          ah[0] = fmaf(w8[q], a.x, ah[0]);
          ah[1] = fmaf(w8[q], a.y, ah[1]);
          ah[2] = fmaf(w8[q], b.x, ah[2]);
          ah[3] = fmaf(w8[q], b.y, ah[3]);
          whw += (double)w8[q];
        } else {
          if constexpr (ERR) {
            at[0] = fmaf(w8[q], a.x, at[0]);
            at[1] = fmaf(w8[q], a.y, at[1]);
            at[2] = fmaf(w8[q], b.x, at[2]);
            at[3] = fmaf(w8[q], b.y, at[3]);
          }
          wtw += (double)w8[q];
        }
      }
    }
    __syncwarp();
  };
  int nl = 0;  // entries in this warp's window list (warp-uniform)
  unsigned long long* wlk = S.wl_key[warp];
  unsigned char* wlf = S.wl_kept[warp];
  auto drain = [&]() {
    gather_list(wlk, wlf, 0, nl, 1);
    nl = 0;
  };
for (int64_t b0 = k_lo; b0 < k_hi; b0 += (int64_t)kBatch * kChunk) {
  float4 xv[kBatch];
#pragma unroll
  for (int c = 0; c < kBatch; ++c) {
    const int64_t key0 = b0 + (int64_t)c * kChunk + 4 * tid;
    // rows of the logits are padded to a multiple of 64 keys: the 16-byte
    // load of four keys starting below k_hi stays inside the row
    xv[c] = key0 < k_hi ? __ldcg(reinterpret_cast<const float4*>(ur + key0))
                        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  uint32_t kbits = 0u, wbits = 0u;  // bit 4c + e: key e of chunk c kept / in the window
  unsigned long long pk[2] = {0ull, 0ull};
#pragma unroll
  for (int c = 0; c < kBatch; ++c) {
    const int64_t key0 = b0 + (int64_t)c * kChunk + 4 * tid;
    const float xs[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool valid = key0 + e < k_hi;
      const uint32_t ok = order_key(xs[e]);
      // kept iff the composite key is >= the cut's (a key outside the
      // window lies on the side of the cut that its bracket side names)
      if (valid && (ok > cut_key || (ok == cut_key && (uint32_t)(key0 + e) <= cut_idx)))
        kbits |= 1u << (4 * c + e);
      const bool win = in_window(xs[e], sc, llo, lhi);
      if (valid && win) wbits |= 1u << (4 * c + e);
    }
    pk[c >> 2] += (unsigned long long)__popc((kbits >> (4 * c)) & 0xfu) << (16 * (c & 3));
  }
  unsigned long long tot[2];
  block_excl_scan_packed(pk, tot, S);
  uint32_t chunk_base = pos_out;
#pragma unroll
  for (int c = 0; c < kBatch; ++c) {
    const int64_t key0 = b0 + (int64_t)c * kChunk + 4 * tid;
    const uint32_t kb = (kbits >> (4 * c)) & 0xfu;
    uint32_t at_ = chunk_base + (uint32_t)((pk[c >> 2] >> (16 * (c & 3))) & 0xffffull);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if ((kb >> e) & 1u) {
        if (at_ < (uint32_t)n) dst[at_] = (int32_t)(key0 + e);
        ++at_;
      }
    }
    chunk_base += (uint32_t)((tot[c >> 2] >> (16 * (c & 3))) & 0xffffull);
    // window keys of the chunk to this warp's list
    const uint32_t wb = (wbits >> (4 * c)) & 0xfu;
    if (__any_sync(0xffffffffu, wb != 0u)) {
      const uint32_t cnt = __popc(wb);
      uint32_t pre = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += y;
      }
      const int total = (int)__shfl_sync(0xffffffffu, pre, 31);
      int slot = nl + (int)(pre - cnt);
      const float xs[4] = {xv[c].x, xv[c].y, xv[c].z, xv[c].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((wb >> e) & 1u) {
          wlk[slot] = ((unsigned long long)__float_as_uint(xs[e]) << 32) | (uint32_t)(key0 + e);
          wlf[slot] = (unsigned char)((kb >> e) & 1u);
          ++slot;
        }
      }
      __syncwarp();
      nl += total;
      if (nl > kWList - 4 * kWarp) drain();  // the next chunk may add 128
    }
  }
  pos_out = chunk_base;
}
  if (nl) drain();
  WinSums r;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    r.ah[i] = ah[i];
    r.at[i] = at[i];
  }
  r.whw = whw;
  r.wtw = wtw;
  r.dmx = dmx;
  r.pos_out = pos_out;
  return r;
}

template <bool ERR>
__global__ void __launch_bounds__(kTThreads, 2)
settle_tc_kernel(const __nv_bfloat16* __restrict__ V, const float* __restrict__ u, TcBufs tb,
                 float* __restrict__ acc, __nv_bfloat16* __restrict__ out,
                 int32_t* __restrict__ k_out, int32_t* __restrict__ idx_out,
                 float* __restrict__ tv_out, float* __restrict__ err_out,
                 float* __restrict__ kl_out, float* __restrict__ gap_out, Plan p,
                 uint32_t* __restrict__ status) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the value pass has completed
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SettleShared& S = *reinterpret_cast<SettleShared*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nr = p.nranges;
  const int G = p.settle_group;
  const int nseg = (nr + G - 1) / G;
  const int64_t row = blockIdx.x / nseg;
  const int seg = (int)(blockIdx.x % nseg);
  const int r_first = seg * G, r_last = min(nr, r_first + G);
  const int64_t n = p.n;
  const float sc = p.scale2;
  const double eps = p.eps;
  const float* ur = u + row * p.ustride;
  const float M = __ldcg(&tb.brk[row].M);
  int llo = __ldcg(&tb.brk[row].llo), lhi = __ldcg(&tb.brk[row].lhi);

  // The candidate list (whole: its length is one of the records) and the
  // segment's first block of kept-for-certain mask words go to shared memory
  // asynchronously, in the same round as the records.
  const int64_t seg_lo = (int64_t)r_first * p.rstages * 128;
  const int64_t seg_hi = min(n, (int64_t)r_last * p.rstages * 128);
  const int64_t mw_lo = seg_lo >> 5, mw_hi = (seg_hi + 31) >> 5;  // 4-word aligned
  // (bulk copies on the barrier bar_in, issued by one thread; a candidate
  // list or mask row starts on a 16-byte boundary and the copied mask words
  // are whole groups of four, inside the row)
  if (tid == 0) {
    mbar_init(&S.bar_in, 1);
    mbar_init(&S.bar_v, 1);
    mbar_fence_init();
    const unsigned long long pol = policy_evict_first();
    const unsigned nb0 = 16u * (unsigned)((min((int64_t)kMaskBlock, mw_hi - mw_lo) + 3) / 4);
    mbar_arrive_expect_tx(&S.bar_in, (unsigned)(kCandCap * 8) + nb0);
    bulk_load(S.cand, tb.cand + row * kCandCap, (unsigned)(kCandCap * 8), &S.bar_in, pol);
    if (nb0) bulk_load(S.mask0, tb.hmask + row * tb.mask_words + mw_lo, nb0, &S.bar_in, pol);
  }
  // ---- 1. row totals (warp 0: one range record per lane) ----------------------
  if (warp == 0) {
    U128 z = u128_zero(), dm = u128_zero(), wm = u128_zero();
    uint32_t nh = 0u, nhb = 0u, nw = 0u;
    for (int r0 = 0; r0 < nr; r0 += 32) {
      const int r = r0 + lane;
      if (r < nr) {
        const uint4* rc = reinterpret_cast<const uint4*>(tb.rrec + row * nr + r);
        const uint4 a = __ldcg(rc), b = __ldcg(rc + 1), c = __ldcg(rc + 2), e = __ldcg(rc + 4);
        const U128 mh = u128_make(((unsigned long long)a.y << 32) | a.x, ((unsigned long long)a.w << 32) | a.z);
        const U128 mt = u128_make(((unsigned long long)b.y << 32) | b.x, ((unsigned long long)b.w << 32) | b.z);
        const U128 mw = u128_make(((unsigned long long)c.y << 32) | c.x, ((unsigned long long)c.w << 32) | c.z);
        u128_add(z, mh);
        u128_add(z, mt);
        u128_add(z, mw);
        u128_add(dm, mt);
        u128_add(wm, mw);
        nh += e.x;  // RangeRec: nh, nw, tmax, pad at bytes 64..79
        if (r < r_first) nhb += e.x;
        nw += e.y;
      }
    }
    z = u128_warp_sum(z);
    dm = u128_warp_sum(dm);
    wm = u128_warp_sum(wm);
    nh = __reduce_add_sync(0xffffffffu, nh);
    nhb = __reduce_add_sync(0xffffffffu, nhb);
    nw = __reduce_add_sync(0xffffffffu, nw);
    if (lane == 0) {
      S.Z = z;
      S.D = dm;
      S.W = wm;
      S.NH = nh;
      S.NHbefore = nhb;
      S.NW = nw;
    }
  } else if (warp == 1 && lane == 0) {
    S.ccnt = __ldcg(tb.cand_cnt + row);
  }
  __syncthreads();
  const U128 Z = S.Z;
  U128 D = S.D, Wm = S.W;
  uint32_t NH = S.NH, NHbefore = S.NHbefore;
  const uint32_t ccnt = S.ccnt;
  const bool valid = certified128(Z, u128_sub(Z, D), eps) &&
                     !certified128(Z, u128_sub(u128_sub(Z, D), Wm), eps);
  const bool ignore = !valid;  // recompute the row from the logits alone
  if (ignore) {
    if (tid == 0 && seg == 0) atomicOr(status, CTA_DEV_INTERNAL);
    llo = INT_MIN;
    lhi = INT_MAX;
    D = u128_zero();
    Wm = Z;
    NH = 0u;
    NHbefore = 0u;
  }
  const U128 base = u128_sub(u128_sub(Z, D), Wm);  // mass of the keys kept for certain
  bool fast = !ignore && ccnt <= (uint32_t)kCandCap;
  if (fast && ccnt != S.NW) {
    if (tid == 0 && seg == 0) atomicOr(status, CTA_DEV_INTERNAL);
    fast = false;
  }
  const int m = fast ? (int)ccnt : 0;
  if (tid == 0) {
    S.found = 0;
    S.nlist = 0u;
  }
  if (!mbar_wait(&S.bar_in, 0u) && tid == 0) atomicOr(status, CTA_DEV_TIMEOUT);
  __syncthreads();
  // fast path: the segment's window keys (the candidates with an index in
  // it) to a flat list, and the value rows of the first kVPre of them copied
  // in while the cut is searched
  unsigned long long* fl_key = &S.wl_key[0][0];  // flat list of kTWarps * kWList entries
  int vcopies = 0;  // value rows in flight on bar_v (waited for on every path)
  if (fast) {
    for (int i = tid; i < m; i += kTThreads) {
      const unsigned long long ck = S.cand[i];
      const uint32_t idx = 0xffffffffu - (uint32_t)(ck & 0xffffffffull);
      if ((int64_t)idx >= seg_lo && (int64_t)idx < seg_hi) {
        const uint32_t slot = atomicAdd(&S.nlist, 1u);
        fl_key[slot] = ck;
      }
    }
    __syncthreads();
    const int npre = min((int)S.nlist, kVPre);
    vcopies = npre;
    if (warp == 0 && npre > 0) {  // one 256-byte bulk copy per row, on bar_v
      const __nv_bfloat16* Vr = V + (row / p.gm) * n * kTD;
      const unsigned long long pol = policy_evict_first();
      if (lane == 0) mbar_arrive_expect_tx(&S.bar_v, (unsigned)npre * (unsigned)(kTD * 2));
      __syncwarp();
      for (int e = lane; e < npre; e += kWarp) {
        const uint32_t idx = 0xffffffffu - (uint32_t)(fl_key[e] & 0xffffffffull);
        bulk_load(&S.vrow[e][0], Vr + (int64_t)idx * kTD, (unsigned)(kTD * 2), &S.bar_v, pol);
      }
    }
  }

  // ---- 2. the exact cut --------------------------------------------------------
  const long long nsub = 64ll * ((long long)lhi - (long long)llo);
  if (fast && nsub <= kSubMax) {
    const long long stop = 64ll * ((long long)lhi - 1);  // sub-level of sub-bin 0 (the top)
    for (int i = tid; i < (int)nsub; i += kTThreads) {
      S.u.sb.lo[i] = 0ull;
      S.u.sb.hi[i] = 0ull;
      S.u.sb.cnt[i] = 0u;
    }
    if (tid == 0) S.nsl = 0u;
    __syncthreads();
    bool huge = false;  // sub-levels are exact for |x| < 1e5 only
    for (int i = tid; i < m; i += kTThreads) {
      const float x = ck_logit(S.cand[i]);
      huge |= !(fabsf(__fmul_rn(x, sc)) < 1.0e5f);
      const int j = (int)min(max(stop - (long long)key_sublevel(x, sc), 0ll), nsub - 1);
      const unsigned long long w = mass62(weight(x, M, sc));
      const unsigned long long old = atomicAdd(&S.u.sb.lo[j], w);
      if (old + w < old) atomicAdd(&S.u.sb.hi[j], 1ull);
      atomicAdd(&S.u.sb.cnt[j], 1u);
    }
    if (__syncthreads_or(huge)) goto full_sort;
    // sub-bins 2t, 2t + 1 per thread, in ranking order from the top
    const int j0 = 2 * tid;
    U128 m0 = u128_zero(), m1 = u128_zero();
    uint32_t c0 = 0u, c1 = 0u;
    if (j0 < nsub) {
      m0 = u128_make(S.u.sb.lo[j0], S.u.sb.hi[j0]);
      c0 = S.u.sb.cnt[j0];
    }
    if (j0 + 1 < nsub) {
      m1 = u128_make(S.u.sb.lo[j0 + 1], S.u.sb.hi[j0 + 1]);
      c1 = S.u.sb.cnt[j0 + 1];
    }
    U128 ex = m0;
    u128_add(ex, m1);
    uint32_t cex = c0 + c1;
    block_excl_scan(ex, cex, S);
    U128 before = base;
    u128_add(before, ex);
    U128 mid = before;
    u128_add(mid, m0);
    U128 after = mid;
    u128_add(after, m1);
    if (c0 > 0u && !certified128(Z, before, eps) && certified128(Z, mid, eps)) {
      S.jstar = j0;
      S.cum = before;
      S.cabove = cex;
      S.found = 1;
    } else if (c1 > 0u && !certified128(Z, mid, eps) && certified128(Z, after, eps)) {
      S.jstar = j0 + 1;
      S.cum = mid;
      S.cabove = cex + c0;
      S.found = 1;
    }
    __syncthreads();
    if (S.found) {
      const int js = S.jstar;
      for (int i = tid; i < m; i += kTThreads) {
        const unsigned long long ck = S.cand[i];
        const int j = (int)min(max(stop - (long long)key_sublevel(ck_logit(ck), sc), 0ll), nsub - 1);
        if (j == js) {
          const uint32_t slot = atomicAdd(&S.nsl, 1u);
          if (slot < (uint32_t)kSubList) S.u.sb.list[slot] = ck;
        }
      }
      __syncthreads();
      const int nsl = (int)S.nsl;
      if (nsl <= kSubList) {
        if (tid < nsl) {  // rank sort (composite keys are distinct)
          const unsigned long long mine = S.u.sb.list[tid];
          int rank = 0;
          for (int q = 0; q < nsl; ++q) rank += S.u.sb.list[q] > mine;
          S.u.sb.sorted[rank] = mine;
        }
        __syncthreads();
        if (tid == 0) {
          U128 cum = S.cum;
          int pos = -1;
          for (int q = 0; q < nsl; ++q) {
            u128_add(cum, mass62(weight(ck_logit(S.u.sb.sorted[q]), M, sc)));
            if (certified128(Z, cum, eps)) {
              pos = q;
              break;
            }
          }
          if (pos >= 0) {
            S.cut = S.u.sb.sorted[pos];
            S.C = cum;
            S.k = (long long)NH + S.cabove + pos + 1;
          } else {
            S.found = 0;
          }
        }
      } else if (tid == 0) {
        S.found = 0;  // too many keys at one sub-level: sort the whole list instead
      }
      __syncthreads();
    }
  }
full_sort:
  if (fast && !S.found) {
    if (!cut_by_sort(S, m, M, sc, NH, Z, base, eps)) {
      if (tid == 0 && seg == 0) atomicOr(status, CTA_DEV_INTERNAL);
      fast = false;
    }
  }
  if (!fast) cut_by_radix(S, ur, n, M, sc, llo, lhi, NH, Z, base, eps, status);
  const unsigned long long cut = S.cut;
  const uint32_t cut_key = (uint32_t)(cut >> 32);
  const uint32_t cut_idx = 0xffffffffu - (uint32_t)(cut & 0xffffffffull);
  const long long k = min((long long)n, S.k);
  const U128 C = S.C;

  // ---- 3. this CTA's keys: ranges r_first .. r_last - 1, one contiguous segment ----
  const int64_t k_lo = (int64_t)r_first * p.rstages * 128;
  const int64_t k_hi = min(n, (int64_t)r_last * p.rstages * 128);
  int32_t* dst = idx_out + row * n;
  const __nv_bfloat16* Vg = V + (row / p.gm) * n * kTD;
  {
    // kept window keys before the segment
    {
      uint32_t c = 0u;
      if (fast) {
        for (int i = tid; i < m; i += kTThreads) {
          const unsigned long long ck = S.cand[i];
          c += (ck >= cut && (int64_t)(0xffffffffu - (uint32_t)(ck & 0xffffffffull)) < k_lo) ? 1u : 0u;
        }
      } else {
        for (int64_t key = tid; key < k_lo; key += kTThreads) {
          const float x = __ldcg(ur + key);
          c += (in_window(x, sc, llo, lhi) && is_kept(order_key(x), (uint32_t)key, cut_key, cut_idx))
                   ? 1u : 0u;
        }
      }
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) S.u32buf[warp] = c;
      __syncthreads();
      if (tid == 0) {
        uint32_t s = 0u;
        for (int w = 0; w < kTWarps; ++w) s += S.u32buf[w];
        S.off_win = s;
      }
      __syncthreads();
    }
    uint32_t pos_out = NHbefore + S.off_win;
    float ah[4] = {0.f, 0.f, 0.f, 0.f}, at[4] = {0.f, 0.f, 0.f, 0.f};
    double whw = 0.0, wtw = 0.0;
    float dmx = kNegInf;
    // value rows of listed window keys: entries first, first + stride, ...
    // below end, eight loads in flight per round (whole warp)
    if (fast) {
      // The window keys of the segment are the candidates with an index in it
      // (the flat list); every other key's side is in the value pass's
      // kept-for-certain mask.  The first kVPre value rows are in shared memory.
      const int nlist = (int)S.nlist;
      if (vcopies > 0 && !mbar_wait(&S.bar_v, 0u) && tid == 0) atomicOr(status, CTA_DEV_TIMEOUT);
      // one entry per warp and step (a short loop body: this code runs once per
      // CTA, so its size rather than its latency decides)
      for (int e = warp; e < nlist; e += kTWarps) {
        const unsigned long long ck = fl_key[e];
        const float x = ck_logit(ck);
        const uint32_t idx = 0xffffffffu - (uint32_t)(ck & 0xffffffffull);
        const float w = weight(x, M, sc);
        const uint2 vv = e < kVPre ? S.vrow[e][lane]
                                   : __ldg(reinterpret_cast<const uint2*>(Vg + (int64_t)idx * kTD) + lane);
        const float2 a = bf16x2_to_float2(vv.x), b = bf16x2_to_float2(vv.y);
        if (ck >= cut) {
          ah[0] = fmaf(w, a.x, ah[0]);
          ah[1] = fmaf(w, a.y, ah[1]);
          ah[2] = fmaf(w, b.x, ah[2]);
          ah[3] = fmaf(w, b.y, ah[3]);
          whw += (double)w;
        } else {
          if constexpr (ERR) {
            at[0] = fmaf(w, a.x, at[0]);
            at[1] = fmaf(w, a.y, at[1]);
            at[2] = fmaf(w, b.x, at[2]);
            at[3] = fmaf(w, b.y, at[3]);
          }
          wtw += (double)w;
          dmx = fmaxf(dmx, x);
        }
      }
      // kept indices: mask words of the segment, in blocks of kMaskBlock words
      const int64_t w_lo = mw_lo, w_hi = mw_hi;
      const uint32_t* hm = tb.hmask + row * tb.mask_words;
      for (int64_t wb0 = w_lo; wb0 < w_hi; wb0 += kMaskBlock) {
        const int nwb = (int)min((int64_t)kMaskBlock, w_hi - wb0);
        uint32_t kw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int wi = 4 * tid + j;
          kw[j] = wi < nwb ? (wb0 == w_lo ? S.mask0[wi] : __ldcg(hm + wb0 + wi)) : 0u;
          S.u.mk.win[wi] = 0u;
        }
        __syncthreads();
        for (int e = tid; e < nlist; e += kTThreads) {  // the block's kept window keys
          const unsigned long long ck = fl_key[e];
          const uint32_t idx = 0xffffffffu - (uint32_t)(ck & 0xffffffffull);
          const int64_t wi = ((int64_t)idx >> 5) - wb0;
          if (ck >= cut && wi >= 0 && wi < nwb) atomicOr(&S.u.mk.win[wi], 1u << (idx & 31u));
        }
        __syncthreads();
        uint32_t c = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          kw[j] |= S.u.mk.win[4 * tid + j];
          c += __popc(kw[j]);
        }
        U128 dummy = u128_zero();
        uint32_t ex = c;
        block_excl_scan(dummy, ex, S);
        uint32_t o = ex;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          S.u.mk.word[4 * tid + j] = kw[j];
          S.u.mk.off[4 * tid + j] = o;
          o += __popc(kw[j]);
        }
        if (tid == kTThreads - 1) S.off_win = o;  // the block's kept keys
        __syncthreads();
        // The block's indices go out through shared memory, kStageWords words
        // at a time: compacted there (the candidate list is no longer read),
        // index i at slot i - g0 + pad so that a 16-byte boundary of idx_out is
        // one of the staging area; the aligned middle goes out as one bulk
        // copy, the (at most three) indices at either end as plain stores.
        // Staging areas take turns: the candidate list (kStageWords words)
        // and the window rows (2 kStageWords), both read by now, and in the
        // segment's last block of mask words also the flat window list
        // (kStageWords), so that a round's compaction overlaps the earlier
        // rounds' bulk copies and a segment of up to 16K keys needs no wait.
        const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(dst) >> 2) & 3u;
        const int nareas = (wb0 + kMaskBlock >= w_hi) ? 3 : 2;
        for (int s0 = 0, rnd = 0; s0 < nwb; ++rnd) {
          const int area = rnd % nareas;
          int* stage = area == 0 ? reinterpret_cast<int*>(S.cand)
                       : area == 1 ? reinterpret_cast<int*>(&S.vrow[0][0])
                                   : reinterpret_cast<int*>(&S.wl_key[0][0]);
          if (rnd >= nareas) {  // this area's copy of nareas rounds ago has read it
            if (tid == 0) {
              if (nareas == 3) bulk_wait_read2();
              else bulk_wait_read1();
            }
            __syncthreads();
          }
          const int s1 = min(nwb, s0 + (area == 1 ? 2 : 1) * kStageWords);
          const uint32_t off0 = S.u.mk.off[s0];
          const uint32_t off1 = s1 < nwb ? S.u.mk.off[s1] : S.off_win;
          // global positions [g0, g1) (never past n, whatever the records say)
          const uint32_t g0 = min(pos_out + off0, (uint32_t)n);
          const uint32_t g1 = min(pos_out + off1, (uint32_t)n);
          const uint32_t pad = (g0 + mis) & 3u;
          for (int w0 = s0 + warp; w0 < s1; w0 += 4 * kTWarps) {
            uint32_t bits[4], off[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int wi = w0 + q * kTWarps;
              bits[q] = wi < s1 ? S.u.mk.word[wi] : 0u;
              off[q] = wi < s1 ? S.u.mk.off[wi] : 0u;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              if ((bits[q] >> lane) & 1u)  // slot < kStageWords * 32 + 3
                stage[pad + off[q] - off0 + __popc(bits[q] & ((1u << lane) - 1u))] =
                    (int)(((wb0 + w0 + q * kTWarps) << 5) + lane);
            }
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // staged indices -> bulk copy
          __syncthreads();
          uint32_t a0 = g0 + ((4u - pad) & 3u);  // first 16-byte boundary
          uint32_t a1 = g1;
          if (a0 >= g1 || g1 - a0 < 4u)
            a0 = g1;  // short: plain stores only
          else
            a1 = g1 - ((g1 + mis) & 3u);  // last 16-byte boundary, >= a0
          for (uint32_t i = g0 + tid; i < a0; i += kTThreads) dst[i] = stage[i - g0 + pad];
          for (uint32_t i = a1 + tid; i < g1; i += kTThreads) dst[i] = stage[i - g0 + pad];
          if (tid == 0) {
            if (a1 > a0) bulk_store(dst + a0, stage + (a0 - g0 + pad), (a1 - a0) * 4u);
            bulk_commit();  // one group per round (possibly empty)
          }
          s0 = s1;
        }
        if (tid == 0) bulk_wait_read();  // both areas may be written again
        __syncthreads();
        pos_out += S.off_win;
        __syncthreads();
      }
    } else {
      const WinSums w = settle_scan_segment<ERR>(ur, Vg, dst, n, k_lo, k_hi, M, sc, llo, lhi,
                                                 cut_key, cut_idx, pos_out, S);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ah[i] += w.ah[i];
        at[i] += w.at[i];
      }
      whw += w.whw;
      wtw += w.wtw;
      dmx = fmaxf(dmx, w.dmx);
      pos_out = w.pos_out;
    }
    // ---- the range's results: value pass partial + window sums -------------------
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      S.accw[0][warp][4 * lane + i] = ah[i];
      S.accw[1][warp][4 * lane + i] = at[i];
    }
    if (lane == 0) {
      S.wsw[0][warp] = whw;
      S.wsw[1][warp] = wtw;
      S.dmw[warp] = dmx;
    }
    __syncthreads();
    {
      // the window sums join the value pass's partial of the segment's first
      // range (the row's last CTA adds the partials of every range)
      const int a = tid / kTD, dim = tid % kTD;  // 256 threads: (kept / dropped, dimension)
      if (ERR || a == 0) {
        double sum = 0.0;
        for (int w = 0; w < kTWarps; ++w) sum += (double)S.accw[a][w][dim];
        float* dstp = acc + ((row * nr + r_first) * 2 + a) * kTD + dim;
        if (!ignore) sum += (double)__ldcg(dstp);
        *dstp = (float)sum;
        if (ignore)  // the value pass's partials of this row do not count
          for (int r = r_first + 1; r < r_last; ++r) acc[((row * nr + r) * 2 + a) * kTD + dim] = 0.0f;
      }
      if (warp == 0) {
        double wh = 0.0, wt = 0.0;
        float tmx = kNegInf;
        if (!ignore) {
          for (int r = r_first + lane; r < r_last; r += 32) {
            const RangeRec* rc = tb.rrec + row * nr + r;
            wh += __ldcg(&rc->wh);
            wt += __ldcg(&rc->wt);
            tmx = fmaxf(tmx, __ldcg(&rc->tmax));
          }
        }
        wh = warp_sum_dbl(wh);
        wt = warp_sum_dbl(wt);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) tmx = fmaxf(tmx, __shfl_xor_sync(0xffffffffu, tmx, o));
        if (lane == 0) {
          for (int w = 0; w < kTWarps; ++w) {
            wh += S.wsw[0][w];
            wt += S.wsw[1][w];
            tmx = fmaxf(tmx, S.dmw[w]);
          }
          SegRec sr;
          sr.wh = wh;
          sr.wt = wt;
          sr.tmax = tmx;
          sr.pad[0] = sr.pad[1] = sr.pad[2] = 0u;
          tb.srec[row * nr + seg] = sr;
        }
      }
    }
  }

  // ---- 4. the row's last CTA forms the outputs ------------------------------------
  if (vcopies > 0) mbar_wait(&S.bar_v, 0u);  // no copy into this CTA is left in flight
  if (tid == 0) bulk_wait_all();             // the bulk index stores are done
  __threadfence();
  __syncthreads();
  if (tid == 0) S.last = atomicAdd(tb.ticket + row, 1u) == (uint32_t)(nseg - 1);
  __syncthreads();
  if (!S.last) return;
  __threadfence();
  double* fin = reinterpret_cast<double*>(&S.accw[0][0][0]);  // [2][kTD] doubles
  {
    const int a = tid / kTD, dim = tid % kTD;
    double s = 0.0;
    if (ERR || a == 0) {
      // the ranges' partials in order, eight loads in flight
      const float* src = acc + (row * nr * 2 + a) * kTD + dim;
      for (int c0 = 0; c0 < nr; c0 += 8) {
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) x[j] = c0 + j < nr ? __ldcg(src + (int64_t)(c0 + j) * 2 * kTD) : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) s += (double)x[j];
      }
    }
    fin[a * kTD + dim] = s;
  }
  if (warp == 0) {  // the row's weight sums (for KL) and largest dropped logit, range order
    double wh = 0.0, wt = 0.0;
    float gm = kNegInf;
    for (int c0 = 0; c0 < nseg; c0 += 32) {
      const int c = c0 + lane;
      double a = 0.0, b = 0.0;
      float t = kNegInf;
      if (c < nseg) {
        a = __ldcg(&tb.srec[row * nr + c].wh);
        b = __ldcg(&tb.srec[row * nr + c].wt);
        t = __ldcg(&tb.srec[row * nr + c].tmax);
      }
      for (int q = 0; q < 32 && c0 + q < nseg; ++q) {
        wh += __shfl_sync(0xffffffffu, a, q);
        wt += __shfl_sync(0xffffffffu, b, q);
        gm = fmaxf(gm, __shfl_sync(0xffffffffu, t, q));
      }
    }
    if (lane == 0) {
      S.wsw[0][0] = wh;
      S.wsw[1][0] = wt;
      S.dmw[0] = gm;
    }
  }
  __syncthreads();
  // output normalisers: the exact kept and dropped masses
  const double hm = ldexp(u128_to_double(C), -kMass62);
  const double tm = ldexp(u128_to_double(u128_sub(Z, C)), -kMass62);
  double* sq = fin + 2 * kTD;  // [kTD] doubles, still inside accw
  if (tid < kTD) {
    const double mu_h = fin[tid] / hm;
    out[row * kTD + tid] = __float2bfloat16_rn((float)mu_h);
    const double diff = (ERR && tm > 0.0) ? fin[kTD + tid] / tm - mu_h : 0.0;
    sq[tid] = diff * diff;
  }
  __syncthreads();
  const double tv = u128_to_double(u128_sub(Z, C)) / u128_to_double(Z);
  if (tid < kWarp) {  // fixed-order tree over the dimensions
    double v = (sq[4 * tid] + sq[4 * tid + 1]) + (sq[4 * tid + 2] + sq[4 * tid + 3]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (tid == 0) {
      const double wh = S.wsw[0][0], wt = S.wsw[1][0];
      if (!(hm > 0.0)) atomicOr(status, CTA_DEV_INTERNAL);
      if (err_out) err_out[row] = (float)(tm > 0.0 ? tv * sqrt(v) : 0.0);
      k_out[row] = (int32_t)k;
      tv_out[row] = (float)tv;
      if (kl_out) kl_out[row] = (float)log1p(wt / wh);
      if (gap_out)
        gap_out[row] = (float)single_gap_bound((double)key_value(cut_key), (double)S.dmw[0], k, n, kTD);
    }
  }
}

template <bool ERR>
cudaError_t launch_e(const void* V, const float* u, const TcBufs& tb, float* acc, void* out,
                     int32_t* k_out, int32_t* idx_out, float* tv_out, float* err_out,
                     float* kl_out, float* gap_out, const Plan& p, uint32_t* status,
                     cudaStream_t st) {
  auto kern = settle_tc_kernel<ERR>;
  constexpr size_t smem = sizeof(SettleShared);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  const int nseg = (p.nranges + p.settle_group - 1) / p.settle_group;
  cfg.gridDim = dim3((unsigned)(p.rows * nseg), 1, 1);
  cfg.blockDim = dim3(kTThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(V), u, tb, acc,
                            static_cast<__nv_bfloat16*>(out), k_out, idx_out, tv_out, err_out,
                            kl_out, gap_out, p, status);
}

}  // namespace

cudaError_t launch_settle_tc(const void* V, const float* u, const TcBufs& tb, float* acc, void* out,
                             int32_t* k_out, int32_t* idx_out, float* tv_out, float* err_out,
                             float* kl_out, float* gap_out, const Plan& p, uint32_t* status,
                             cudaStream_t st) {
  if (p.rstages < 1 || p.d != kTD || p.settle_group < 1 || p.settle_group > kMaxGroup ||
      p.rows * (int64_t)p.nranges > INT32_MAX)
    return cudaErrorInvalidValue;
  return p.want_err ? launch_e<true>(V, u, tb, acc, out, k_out, idx_out, tv_out, err_out, kl_out,
                                     gap_out, p, status, st)
                    : launch_e<false>(V, u, tb, acc, out, k_out, idx_out, tv_out, err_out, kl_out,
                                      gap_out, p, status, st);
}

}  // namespace cta
