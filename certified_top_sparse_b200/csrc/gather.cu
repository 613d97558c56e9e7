// Phases 3 and 4: the head-tail output sums and the final combination.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the exact head-tail
// decomposition Attn = H mu_head + tau mu_tail (H = kept mass, tau = TV), the
// truncated output is Attn_k = mu_head and the error factorises as
// ||Attn - Attn_k||_2 = tau ||mu_tail - mu_head||_2.
//
// Phase 3: persistent CTAs, each owning a contiguous range of key chunks of
// one (KV group, row tile).  Bulk copies (TMA) bring stages of up to 128 V
// rows (32 KB) into shared memory.  Per stage every warp turns the logits of
// the keys it will consume into weights, stored as duplicated fp32 pairs
// (kept, and with the error wanted dropped, zero elsewhere) ready to be
// packed-FMA operands.  Each lane owns 16 bytes of a value row and accumulates
// w v as packed fp32 pairs across the whole range; at the range's end lanes
// and warps combine in a fixed order (fp64 across warps) into one partial per
// row and range.  The weight sums (normalisers), the kept indices and the
// largest dropped logits come from selection.
// Phase 4, in the same kernel: the last CTA to finish a (KV group, row tile)
// adds its rows' range partials in a fixed order and forms mu_head (the
// output), mu_tail, err = tau ||mu_tail - mu_head||, KL = log(sum_all w /
// sum_head w) and the single-gap certificate.
#include <algorithm>

#include "common.cuh"
#include "finalize.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kGWarps = 8;
constexpr int kGatherThreads = kGWarps * kWarp;
constexpr int kGStageMax = 32768;  // bytes per V stage at most (128 keys of 256 B)

template <typename T, int D, int RT>
struct GatherCfg {
  static constexpr int ROWB = D * (int)sizeof(T);   // bytes per value row
  static constexpr int LPK = ROWB / 16;             // lanes per key (16 bytes each)
  static constexpr int KPI = kWarp / LPK;           // keys per warp step
  static constexpr int NP = 16 / (int)sizeof(T) / 2;  // fp32 pairs per lane
  static constexpr int TK = (kGStageMax / ROWB) < 128 ? kGStageMax / ROWB : 128;  // keys per stage
  static constexpr int STAGE = TK * ROWB;           // bytes per stage
  static constexpr int STEPS = TK / (kGWarps * KPI);  // warp steps per stage
  static_assert(LPK >= 1 && LPK <= kWarp && kWarp % LPK == 0, "bad key width");
  static_assert(TK % (kGWarps * KPI) == 0, "a stage must split evenly over the warps");
  static_assert(RT == 1 || RT == 2 || RT == 4, "tile rows");
};

template <typename T> __device__ __forceinline__ void widen16(const uint4& r, unsigned long long* f);
template <> __device__ __forceinline__ void widen16<__nv_bfloat16>(const uint4& r, unsigned long long* f) {
  f[0] = pack2(r.x << 16, r.x & 0xffff0000u);
  f[1] = pack2(r.y << 16, r.y & 0xffff0000u);
  f[2] = pack2(r.z << 16, r.z & 0xffff0000u);
  f[3] = pack2(r.w << 16, r.w & 0xffff0000u);
}
template <> __device__ __forceinline__ void widen16<float>(const uint4& r, unsigned long long* f) {
  f[0] = pack2(r.x, r.y);
  f[1] = pack2(r.z, r.w);
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

// Walks this CTA's (item, chunk, piece) sequence for a copy issuer: pieces of
// PK keys cut each chunk from its start (V tiles: PK = stage keys; logit
// slices: PK = kSlice).
template <int PK>
struct GPieceIter {
  int it, c, c_hi, j, nk, group, tile;
  int64_t key0;
  __device__ void start(int first, int nitems, const Plan& p) {
    it = first;
    begin_item(nitems, p);
  }
  __device__ void begin_item(int nitems, const Plan& p) {
    if (it >= nitems) return;
    const GItem g = gitem_of(it, p);
    group = g.group;
    tile = g.tile;
    c = g.range * p.range_len;
    c_hi = min(p.nchunks, c + p.range_len);
    j = 0;
    load_chunk(p);
  }
  __device__ void load_chunk(const Plan& p) {
    key0 = (int64_t)c * p.chunk;
    nk = (int)min((int64_t)p.chunk, p.n - key0);
  }
  __device__ int keys() const { return min(PK, nk - j * PK); }
  __device__ bool valid(int nitems) const { return it < nitems; }
  __device__ void next(int nitems, const Plan& p) {
    if ((j + 1) * PK < nk) { ++j; return; }
    j = 0;
    if (++c < c_hi) { load_chunk(p); return; }
    it += gridDim.x;
    begin_item(nitems, p);
  }
};

template <typename T, int D, int RT, bool ERR>
struct GatherSmem {
  // dynamic bytes per CTA that let the planned number of CTAs share an SM
  static constexpr size_t kBudget = 110 * 1024;
  using C = GatherCfg<T, D, RT>;
  static constexpr int KW = C::TK / kGWarps;          // keys per warp per stage
  static constexpr int WPK = RT * (ERR ? 2 : 1);      // (w, w) words per key: kept rows, dropped rows
  static constexpr int NPAIR = KW * RT;               // (key, row) pairs per warp per stage
  static constexpr int EPL = (NPAIR + kWarp - 1) / kWarp;  // pairs per lane
  static constexpr size_t kW = sizeof(unsigned long long) * kGWarps * KW * WPK;  // per-warp weights
  // item end (aliases kW): per-warp fp32 partials, then the fp64 range sums
  static constexpr size_t kRedF = sizeof(float) * kGWarps * 2 * D;
  static constexpr size_t kRedD = sizeof(double) * RT * 2 * D;
  static constexpr size_t kRed = kRedF > kRedD ? kRedF : kRedD;
  static constexpr size_t kWR = kW > kRed ? kW : kRed;
  static constexpr int kFit = (int)((kBudget - kWR) / C::STAGE);
  static constexpr int kStages = kFit > 6 ? 6 : kFit;
  static constexpr size_t kBytes = (size_t)kStages * C::STAGE + kWR;
  static_assert(EPL <= 2, "at most two (key, row) pairs per lane");
  static_assert(kStages >= 3, "too few stages");
  static_assert(KW == C::KPI * C::STEPS, "warp keys per stage");
};

// Weight pairs of one key for RT rows (RT u64 words, each (w, w)).
template <int RT>
__device__ __forceinline__ void load_pairs(const unsigned long long* src, unsigned long long* w) {
  if constexpr (RT == 1) {
    w[0] = *src;
  } else {
#pragma unroll
    for (int h = 0; h < RT / 2; ++h) {
      const ulonglong2 x = reinterpret_cast<const ulonglong2*>(src)[h];
      w[2 * h] = x.x;
      w[2 * h + 1] = x.y;
    }
  }
}

// The CTA streams V through a ring of stages; no CTA barrier is taken until
// the end of an item.  Each warp computes, per stage, the weights of exactly
// the keys it will consume (one (key, row) pair per lane, logits prefetched a
// stage ahead) into its own shared-memory slots, multiplies them into its
// accumulators, and releases the stage; the last warp to release a fill
// refills it.  The kernel is issue-bound, so the multiply-adds run without
// branches (a dropped key multiplies a zero kept weight, and vice versa).
// CTAs per SM: two (32 KB stages; measured faster than three CTAs with 16 KB
// stages even without the error term, whose registers would allow three).
constexpr int gather_occupancy(bool) { return 2; }

template <typename T, int D, int RT, bool ERR>
__global__ void __launch_bounds__(kGatherThreads, gather_occupancy(ERR))
gather_kernel(const T* __restrict__ V, const float* __restrict__ u, const RowSel* __restrict__ sel,
              float* __restrict__ acc_out, uint32_t* __restrict__ unit_cnt,
              const float* __restrict__ gmax, T* __restrict__ out, float* __restrict__ err_out,
              float* __restrict__ kl_out, float* __restrict__ gap_out, Plan p,
              uint32_t* __restrict__ status) {
  using C = GatherCfg<T, D, RT>;
  using S = GatherSmem<T, D, RT, ERR>;
  constexpr int NP = C::NP;
  constexpr int NS = S::kStages;
  constexpr int KW = S::KW;
  constexpr int WPK = S::WPK;
  constexpr int EPL = S::EPL;

  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* stage = smem_raw;                                         // [NS][16 KB]
  unsigned long long* wsm = reinterpret_cast<unsigned long long*>(smem_raw + NS * C::STAGE);
  float* red = reinterpret_cast<float*>(wsm);                              // [kGWarps][2][D]
  __shared__ unsigned long long full[NS];
  __shared__ int vcnt[NS];          // warps done with each stage (cumulative)
  __shared__ GPieceIter<C::TK> vprod;  // value-tile issuer state (whoever issues)
  __shared__ int vissued;
  __shared__ int s_last;                 // this CTA finished the last range of its unit
  __shared__ double s_wh[RT], s_wt[RT];  // the tile's rows' kept / dropped weight sums

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nitems = p.tiles_out * p.nranges * p.groups;
  const unsigned long long pol = (p.tiles_out == 1) ? policy_evict_first() : policy_evict_last();
  unsigned long long* ww = wsm + (size_t)warp * KW * WPK;  // this warp's weight slots [KW][WPK]

  auto issue_v = [&]() {
    if (!vprod.valid(nitems)) return;
    const int s = vissued % NS;
    const unsigned bytes = (unsigned)(vprod.keys() * C::ROWB);
    const unsigned char* src = reinterpret_cast<const unsigned char*>(
        V + ((int64_t)vprod.group * p.n + vprod.key0 + (int64_t)vprod.j * C::TK) * D);
    mbar_arrive_expect_tx(&full[s], bytes);
    bulk_load(stage + s * C::STAGE, src, bytes, &full[s], pol);
    ++vissued;
    vprod.next(nitems, p);
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      vcnt[s] = 0;
    }
    mbar_fence_init();
    vissued = 0;
    vprod.start(blockIdx.x, nitems, p);
    for (int s = 0; s < NS; ++s) issue_v();
  }
  __syncthreads();

  const int part = lane % C::LPK;  // 16-byte piece of the value row this lane owns
  const int slot = lane / C::LPK;
  int t = 0;  // value tiles consumed
  unsigned long long ah[RT][NP], at[RT][NP];

  for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
    const GItem g = gitem_of(it, p);
    const int64_t row0 = (int64_t)g.group * p.gm + (int64_t)g.tile * RT;
    const int nrows = min(RT, p.gm - g.tile * RT);
    const int c_lo = g.range * p.range_len;
    const int c_hi = min(p.nchunks, c_lo + p.range_len);
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int e = 0; e < NP; ++e) { ah[r][e] = 0ull; at[r][e] = 0ull; }

    // ---- this lane's (key, row) pairs: pair b = lane + 32 i is row b / KW,
    //      warp key e = b % KW, stage key kk(e) --------------------------------
    auto kk = [&](int e) { return warp * C::KPI + (e / C::KPI) * kGWarps * C::KPI + e % C::KPI; };
    float pM[EPL];
    uint32_t pks[EPL], pis[EPL];
    const float* pu[EPL];  // the pair row's logits
    bool pv[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int b = lane + kWarp * i;
      const int r = b / KW;
      pv[i] = b < S::NPAIR && r < nrows;
      const int rr = pv[i] ? r : 0;
      const RowSel* rs = sel + row0 + rr;
      pM[i] = __ldg(&rs->M);
      pks[i] = __ldg(&rs->kstar);
      pis[i] = (uint32_t)__ldg(&rs->istar);
      pu[i] = u + (row0 + rr) * p.ustride;
    }
    // logits of the first stage
    float px[EPL];
    {
      const int64_t kb = (int64_t)c_lo * p.chunk;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int64_t key = kb + kk((lane + kWarp * i) % KW);
        px[i] = (pv[i] && key < p.n) ? __ldg(pu[i] + key) : 0.0f;
      }
    }

    for (int c = c_lo; c < c_hi; ++c) {
      const int64_t key0 = (int64_t)c * p.chunk;
      const int nk = (int)min((int64_t)p.chunk, p.n - key0);
      for (int j = 0; j * C::TK < nk; ++j, ++t) {
        const int64_t kt = key0 + (int64_t)j * C::TK;
        const int nkt = min(C::TK, nk - j * C::TK);
        // ---- weights of this warp's keys in the stage -------------------------
        __syncwarp();  // the previous stage's weights are consumed
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int b = lane + kWarp * i;
          const int e = b % KW, r = b / KW;
          const int kl = kk(e);
          const bool ok = pv[i] && kl < nkt;
          float w = 0.0f;
          bool kept = false;
          if (ok) {
            w = weight(px[i], pM[i], p.scale2);
            kept = is_kept(order_key(px[i]), (uint32_t)(kt + kl), pks[i], pis[i]);
          }
          if (b < S::NPAIR) {
            const float h = kept ? w : 0.0f;
            ww[e * WPK + r] = pack2(__float_as_uint(h), __float_as_uint(h));
            if constexpr (ERR) {
              const float d = kept ? 0.0f : w;
              ww[e * WPK + RT + r] = pack2(__float_as_uint(d), __float_as_uint(d));
            }
          }
        }
        // ---- prefetch the logits of the next stage of this item -------------
        {
          int64_t kn = kt + C::TK;
          if (j * C::TK + C::TK >= nk) kn = (c + 1 < c_hi) ? key0 + p.chunk : -1;
          if (kn >= 0) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
              const int64_t key = kn + kk((lane + kWarp * i) % KW);
              px[i] = (pv[i] && key < p.n) ? __ldg(pu[i] + key) : 0.0f;
            }
          }
        }
        __syncwarp();
        // ---- value rows of the stage -----------------------------------------
        const int s = t % NS;
        const unsigned ph = (unsigned)(t / NS) & 1u;
        if (!mbar_wait(&full[s], ph)) {
          if (lane == 0) atomicOr(status, CTA_DEV_TIMEOUT);
          return;
        }
        const uint4* stg = reinterpret_cast<const uint4*>(stage + s * C::STAGE);
#pragma unroll
        for (int q = 0; q < C::STEPS; ++q) {
          const int e = q * C::KPI + slot;
          const int key = kk(e);  // < TK
          if (key < nkt) {
            unsigned long long v[NP];
            widen16<T>(stg[key * C::LPK + part], v);
            unsigned long long w[RT];
            load_pairs<RT>(ww + e * WPK, w);
#pragma unroll
            for (int r = 0; r < RT; ++r)
#pragma unroll
              for (int x = 0; x < NP; ++x) ah[r][x] = fma2p(w[r], v[x], ah[r][x]);
            if constexpr (ERR) {
              load_pairs<RT>(ww + e * WPK + RT, w);
#pragma unroll
              for (int r = 0; r < RT; ++r)
#pragma unroll
                for (int x = 0; x < NP; ++x) at[r][x] = fma2p(w[r], v[x], at[r][x]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) {
          // the last of the kGWarps warps to finish with this fill refills it
          __threadfence_block();
          const int done = atomicAdd(&vcnt[s], 1);
          if (done == kGWarps * (t / NS) + kGWarps - 1) {
            __threadfence_block();
            issue_v();
            __threadfence_block();
          }
        }
      }
    }
    __syncthreads();  // every warp is done with its weight slots (reused below)

    // ---- item end: fixed-order reductions into one partial per row ----------
    // lanes of the same piece in other key slots first (xor over the slot
    // bits), then the warps through shared memory, row by row
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
      for (int e = 0; e < NP; ++e)
#pragma unroll
        for (int o = C::LPK; o < kWarp; o <<= 1) {
          float hx, hy, tx, ty;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(hx), "=f"(hy) : "l"(ah[r][e]));
          asm("mov.b64 {%0, %1}, %2;" : "=f"(tx), "=f"(ty) : "l"(at[r][e]));
          hx += __shfl_xor_sync(0xffffffffu, hx, o);
          hy += __shfl_xor_sync(0xffffffffu, hy, o);
          if constexpr (ERR) {
            tx += __shfl_xor_sync(0xffffffffu, tx, o);
            ty += __shfl_xor_sync(0xffffffffu, ty, o);
          }
          ah[r][e] = pack2(__float_as_uint(hx), __float_as_uint(hy));
          at[r][e] = pack2(__float_as_uint(tx), __float_as_uint(ty));
        }
    const int dim0 = part * (16 / (int)sizeof(T));  // first element of this lane's piece
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      if (slot == 0) {
#pragma unroll
        for (int e = 0; e < NP; ++e) {
          float hx, hy, tx, ty;
          asm("mov.b64 {%0, %1}, %2;" : "=f"(hx), "=f"(hy) : "l"(ah[r][e]));
          asm("mov.b64 {%0, %1}, %2;" : "=f"(tx), "=f"(ty) : "l"(at[r][e]));
          red[(warp * 2 + 0) * D + dim0 + 2 * e] = hx;
          red[(warp * 2 + 0) * D + dim0 + 2 * e + 1] = hy;
          red[(warp * 2 + 1) * D + dim0 + 2 * e] = tx;
          red[(warp * 2 + 1) * D + dim0 + 2 * e + 1] = ty;
        }
      }
      __syncthreads();
      if (r < nrows) {
        for (int x = threadIdx.x; x < 2 * D; x += kGatherThreads) {
          const int a = x / D, dim = x % D;
          if (a == 1 && !ERR) continue;
          double acc = 0.0;
          for (int w = 0; w < kGWarps; ++w) acc += (double)red[(w * 2 + a) * D + dim];
          acc_out[(((row0 + r) * p.nranges + g.range) * 2 + a) * D + dim] = (float)acc;
        }
      }
      __syncthreads();
    }

    // ---- the last CTA to finish a (KV group, row tile) finalises its rows ----
    __threadfence();  // this CTA's partials, visible device-wide before the count
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t prev = atomicAdd(&unit_cnt[g.group * p.tiles_out + g.tile], 1u);
      s_last = prev == (uint32_t)(p.nranges - 1);
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      auto sync = []() { __syncthreads(); };
      finalize_rows<T, D, RT, ERR, kGatherThreads>(
          threadIdx.x, sync, reinterpret_cast<double*>(red), s_wh, s_wt, acc_out, sel, gmax, out,
          err_out, kl_out, gap_out, p, row0, nrows, status);
    }
  }
}

struct GatherOut {
  float* acc;
  uint32_t* unit_cnt;
  const float* gmax;
  void* out;
  float* err_out;
  float* kl_out;
  float* gap_out;
};

template <typename T, int D, int RT, bool ERR>
cudaError_t launch_gather_t(const void* V, const float* u, const RowSel* sel, const GatherOut& o,
                            const Plan& p, uint32_t* status, cudaStream_t st) {
  const size_t smem = GatherSmem<T, D, RT, ERR>::kBytes;
  auto kern = gather_kernel<T, D, RT, ERR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGatherThreads, smem);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const long long nitems = (long long)p.tiles_out * p.nranges * p.groups;
  const long long grid = std::min<long long>(nitems, (long long)std::max(per_sm, 1) * sms);
  kern<<<(unsigned)grid, kGatherThreads, smem, st>>>(
      static_cast<const T*>(V), u, sel, o.acc, o.unit_cnt, o.gmax, static_cast<T*>(o.out),
      o.err_out, o.kl_out, o.gap_out, p, status);
  return cudaGetLastError();
}

template <typename T, int D, bool ERR>
cudaError_t launch_gather_e(const void* V, const float* u, const RowSel* sel, const GatherOut& o,
                            const Plan& p, uint32_t* status, cudaStream_t st) {
  switch (p.rt_out) {
    case 1: return launch_gather_t<T, D, 1, ERR>(V, u, sel, o, p, status, st);
    case 2: return launch_gather_t<T, D, 2, ERR>(V, u, sel, o, p, status, st);
    case 4: return launch_gather_t<T, D, 4, ERR>(V, u, sel, o, p, status, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
cudaError_t launch_gather_d(const void* V, const float* u, const RowSel* sel, const GatherOut& o,
                            const Plan& p, uint32_t* status, cudaStream_t st) {
  return p.want_err ? launch_gather_e<T, D, true>(V, u, sel, o, p, status, st)
                    : launch_gather_e<T, D, false>(V, u, sel, o, p, status, st);
}

}  // namespace

int gather_ctas_per_sm(bool want_err) { return gather_occupancy(want_err); }

cudaError_t launch_gather(int dtype, const void* V, const float* u, const RowSel* sel, float* acc,
                          uint32_t* unit_cnt, const float* gmax, void* out, float* err_out,
                          float* kl_out, float* gap_out, const Plan& p, uint32_t* status,
                          cudaStream_t st) {
  const GatherOut o{acc, unit_cnt, gmax, out, err_out, kl_out, gap_out};
  if (dtype == kDtypeF32)
    return p.d == 64 ? launch_gather_d<float, 64>(V, u, sel, o, p, status, st)
                     : launch_gather_d<float, 128>(V, u, sel, o, p, status, st);
  return p.d == 64 ? launch_gather_d<__nv_bfloat16, 64>(V, u, sel, o, p, status, st)
                   : launch_gather_d<__nv_bfloat16, 128>(V, u, sel, o, p, status, st);
}

}  // namespace cta
