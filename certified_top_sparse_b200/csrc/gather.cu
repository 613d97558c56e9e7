// Phases 3 and 4: the head-tail output sums and the final combination.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the exact head-tail
// decomposition Attn = H mu_head + tau mu_tail (H = kept mass, tau = TV), the
// truncated output is Attn_k = mu_head and the error factorises as
// ||Attn - Attn_k||_2 = tau ||mu_tail - mu_head||_2.
//
// Phase 3 (one CTA per row tile x key chunk x KV group): step A turns the
// chunk's logits into signed weights in shared memory (sign bit = dropped key)
// and sums the kept and dropped weights in fp64; step B streams the V rows of
// the chunk with 16-byte coalesced loads, skipping rows that no row of the
// tile keeps unless the error is wanted, and accumulates sum w v for kept
// (and dropped) keys in fp32 over at most chunk / 16 keys per lane.  The
// per-lane partials are combined in fp64 in a fixed order.
// Phase 4 (one CTA per row) adds the chunk partials in fixed order and forms
// mu_head (the output), mu_tail, err = tau ||mu_tail - mu_head|| and
// KL = log(sum_all w / sum_head w).
#include "common.cuh"
#include "kernels.cuh"

namespace cta {

namespace {

constexpr int kGatherThreads = 256;
constexpr int kGatherWarps = kGatherThreads / kWarp;
constexpr int kGUnroll = 4;

template <typename T, int D, int RT, bool ERR>
__global__ void __launch_bounds__(kGatherThreads)
gather_kernel(const T* __restrict__ V, const float* __restrict__ u, const RowSel* __restrict__ sel,
              const uint32_t* __restrict__ chunk_off, int32_t* __restrict__ idx_out,
              float* __restrict__ acc_out, Partial* __restrict__ part_out, Plan p) {
  constexpr int EPL = Elem<T>::EPL;
  constexpr int LPK = D / EPL;
  constexpr int KPI = kWarp / LPK;
  constexpr int SLOTS = kGatherWarps * KPI;     // lane groups per CTA
  constexpr int NACC = ERR ? 2 : 1;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* sw = reinterpret_cast<float*>(smem_raw);                 // [RT][chunk] signed weights
  float* sred = sw + RT * p.chunk;                                 // [SLOTS][NACC][RT][D]
  __shared__ double dred[kGatherWarps][RT][2];

  const int tile = blockIdx.x;
  const int chunk = blockIdx.y;
  const int group = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int part = lane % LPK;
  const int slot = lane / LPK;
  const int gslot = warp * KPI + slot;

  const int64_t row0 = (int64_t)group * p.gm + (int64_t)tile * RT;
  const int nrows = min(RT, p.gm - tile * RT);
  const int64_t key0 = (int64_t)chunk * p.chunk;
  const int nk = (int)min((int64_t)p.chunk, p.n - key0);

  // ---- step A: signed weights and their sums ---------------------------------
  double sh[RT], st[RT];
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    sh[r] = 0.0;
    st[r] = 0.0;
    if (r < nrows) {
      const RowSel rs = sel[row0 + r];
      const float* ur = u + (row0 + r) * p.n + key0;
      for (int i = threadIdx.x; i < nk; i += kGatherThreads) {
        const float x = ur[i];
        const float w = weight(x, rs.M, p.scale2);
        const bool kept = is_kept(order_key(x), (uint32_t)(key0 + i), rs.kstar, (uint32_t)rs.istar);
        sw[r * p.chunk + i] = kept ? w : -w;
        if (kept) sh[r] += (double)w; else st[r] += (double)w;
      }
    } else {
      for (int i = threadIdx.x; i < nk; i += kGatherThreads) sw[r * p.chunk + i] = -0.0f;
    }
  }
#pragma unroll
  for (int r = 0; r < RT; ++r) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      sh[r] += __shfl_xor_sync(0xffffffffu, sh[r], o);
      st[r] += __shfl_xor_sync(0xffffffffu, st[r], o);
    }
    if (lane == 0) { dred[warp][r][0] = sh[r]; dred[warp][r][1] = st[r]; }
  }
  __syncthreads();
  if (threadIdx.x < nrows) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < kGatherWarps; ++w) { a += dred[w][threadIdx.x][0]; b += dred[w][threadIdx.x][1]; }
    Partial pr;
    pr.wh = a;
    pr.wt = b;
    part_out[(row0 + threadIdx.x) * p.nchunks + chunk] = pr;
  }

  // ---- the chunk's kept indices, ascending, at the offset from selection -----
  {
    __shared__ uint32_t wcount[kGatherWarps];
    const int per = ((nk + kGatherThreads - 1) / kGatherThreads) * kWarp;  // keys per warp
    const int k_lo = min(nk, warp * per), k_hi = min(nk, k_lo + per);
    for (int r = 0; r < nrows; ++r) {
      const float* swr = sw + r * p.chunk;
      uint32_t cnt = 0u;
      for (int k0 = k_lo; k0 < k_hi; k0 += kWarp) {
        const int key = k0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, key < k_hi && !signbit(swr[key])));
      }
      if (lane == 0) wcount[warp] = cnt;
      __syncthreads();
      uint32_t off = chunk_off[(row0 + r) * p.nchunks + chunk];
      for (int w = 0; w < warp; ++w) off += wcount[w];
      for (int k0 = k_lo; k0 < k_hi; k0 += kWarp) {
        const int key = k0 + lane;
        const bool kept = key < k_hi && !signbit(swr[key]);
        const uint32_t m = __ballot_sync(0xffffffffu, kept);
        if (kept) {
          const uint32_t at = off + __popc(m & ((1u << lane) - 1u));
          if (at < (uint32_t)p.n) idx_out[(row0 + r) * p.n + at] = (int32_t)(key0 + key);
        }
        off += __popc(m);
      }
      __syncthreads();
    }
  }

  // ---- step B: weighted value sums -------------------------------------------
  float ah[RT][EPL], at[RT][EPL];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) { ah[r][e] = 0.f; at[r][e] = 0.f; }

  const T* Vc = V + ((int64_t)group * p.n + key0) * D;
  const unsigned long long pol = (p.tiles_out == 1) ? policy_evict_first() : policy_evict_last();
  for (int base = gslot; base < nk; base += SLOTS * kGUnroll) {
    uint4 raw[kGUnroll];
    float w[kGUnroll][RT];
#pragma unroll
    for (int j = 0; j < kGUnroll; ++j) {
      const int key = base + j * SLOTS;
      bool need = false;
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        w[j][r] = (key < nk) ? sw[r * p.chunk + key] : -0.0f;
        need |= !signbit(w[j][r]);
      }
      need = (key < nk) && (ERR || need);
      raw[j] = need ? ld_stream_once(Vc + (int64_t)key * D + part * EPL, pol)
                    : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < kGUnroll; ++j) {
      float v[EPL];
      Elem<T>::unpack(raw[j], v);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        const float x = w[j][r];
        const float wh = signbit(x) ? 0.f : x;
#pragma unroll
        for (int e = 0; e < EPL; ++e) ah[r][e] = fmaf(wh, v[e], ah[r][e]);
        if constexpr (ERR) {
          const float wt = signbit(x) ? -x : 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) at[r][e] = fmaf(wt, v[e], at[r][e]);
        }
      }
    }
  }

  // Per-slot partials to shared memory, then a fixed-order fp64 sum over slots.
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      sred[((gslot * NACC + 0) * RT + r) * D + part * EPL + e] = ah[r][e];
      if constexpr (ERR) sred[((gslot * NACC + 1) * RT + r) * D + part * EPL + e] = at[r][e];
    }
  __syncthreads();
  for (int t = threadIdx.x; t < NACC * RT * D; t += kGatherThreads) {
    const int a = t / (RT * D);
    const int r = (t / D) % RT;
    const int dim = t % D;
    if (r >= nrows) continue;
    double s = 0.0;
    for (int g = 0; g < SLOTS; ++g) s += (double)sred[((g * NACC + a) * RT + r) * D + dim];
    acc_out[(((row0 + r) * p.nchunks + chunk) * 2 + a) * D + dim] = (float)s;
  }
}

template <typename T, int D, int RT, bool ERR>
cudaError_t launch_gather_t(const void* V, const float* u, const RowSel* sel,
                            const uint32_t* choff, int32_t* idx, float* acc, Partial* part,
                            const Plan& p, cudaStream_t st) {
  constexpr int EPL = Elem<T>::EPL;
  constexpr int SLOTS = kGatherWarps * (kWarp / (D / EPL));
  const size_t smem = sizeof(float) * ((size_t)RT * p.chunk + (size_t)SLOTS * (ERR ? 2 : 1) * RT * D);
  auto kern = gather_kernel<T, D, RT, ERR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.tiles_out, p.nchunks, p.groups);
  kern<<<grid, kGatherThreads, smem, st>>>(static_cast<const T*>(V), u, sel, choff, idx, acc, part,
                                           p);
  return cudaGetLastError();
}

template <typename T, int D, bool ERR>
cudaError_t launch_gather_e(const void* V, const float* u, const RowSel* sel,
                            const uint32_t* choff, int32_t* idx, float* acc, Partial* part,
                            const Plan& p, cudaStream_t st) {
  switch (p.rt_out) {
    case 1: return launch_gather_t<T, D, 1, ERR>(V, u, sel, choff, idx, acc, part, p, st);
    case 2: return launch_gather_t<T, D, 2, ERR>(V, u, sel, choff, idx, acc, part, p, st);
    case 4: return launch_gather_t<T, D, 4, ERR>(V, u, sel, choff, idx, acc, part, p, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename T, int D>
cudaError_t launch_gather_d(const void* V, const float* u, const RowSel* sel,
                            const uint32_t* choff, int32_t* idx, float* acc, Partial* part,
                            const Plan& p, cudaStream_t st) {
  return p.want_err ? launch_gather_e<T, D, true>(V, u, sel, choff, idx, acc, part, p, st)
                    : launch_gather_e<T, D, false>(V, u, sel, choff, idx, acc, part, p, st);
}

// ---- phase 4 ------------------------------------------------------------------

constexpr int kFinThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kFinThreads)
finalize_kernel(const RowSel* __restrict__ sel, const float* __restrict__ acc,
                const Partial* __restrict__ part, T* __restrict__ out, float* __restrict__ err_out,
                float* __restrict__ kl_out, Plan p, uint32_t* __restrict__ status) {
  constexpr int G = kFinThreads / D;   // thread groups, each over every G-th chunk
  __shared__ double s_ah[G][D], s_at[G][D], s_w[G][2];
  __shared__ double red[D / 32];
  const int64_t row = blockIdx.x;
  const int dim = threadIdx.x % D;
  const int grp = threadIdx.x / D;
  double ah = 0.0, at = 0.0, wh = 0.0, wt = 0.0;
  const float* a = acc + row * p.nchunks * 2 * D + dim;
#pragma unroll 4
  for (int c = grp; c < p.nchunks; c += G) {
    ah += a[(int64_t)c * 2 * D];
    if (p.want_err) at += a[(int64_t)c * 2 * D + D];
    if (dim == 0) {
      const Partial pr = part[row * p.nchunks + c];
      wh += pr.wh;
      wt += pr.wt;
    }
  }
  s_ah[grp][dim] = ah;
  s_at[grp][dim] = at;
  if (dim == 0) { s_w[grp][0] = wh; s_w[grp][1] = wt; }
  __syncthreads();
  if (threadIdx.x >= D) return;
  ah = 0.0; at = 0.0; wh = 0.0; wt = 0.0;
  for (int g = 0; g < G; ++g) {  // fixed order
    ah += s_ah[g][dim];
    at += s_at[g][dim];
    wh += s_w[g][0];
    wt += s_w[g][1];
  }
  const double mu_h = ah / wh;
  Elem<T>::store1(out + row * D + dim, (float)mu_h);
  if (!(wh > 0.0) && dim == 0) atomicOr(status, CTA_DEV_INTERNAL);
  if (err_out) {
    const double diff = (wt > 0.0) ? (at / wt - mu_h) : 0.0;
    double s = diff * diff;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((dim & 31) == 0) red[dim >> 5] = s;
    asm volatile("bar.sync 1, %0;" ::"r"(D));  // the first D threads only
    if (dim == 0) {
      double tot = 0.0;
      for (int w = 0; w < D / 32; ++w) tot += red[w];
      const RowSel rs = sel[row];
      err_out[row] = (float)(rs.C < rs.Z && wt > 0.0 ? rs.tv * sqrt(tot) : 0.0);
    }
  }
  if (kl_out && dim == 0) kl_out[row] = (float)log1p(wt / wh);
}

template <typename T>
cudaError_t launch_finalize_t(const RowSel* sel, const float* acc, const Partial* part, void* out,
                              float* err_out, float* kl_out, const Plan& p, uint32_t* status,
                              cudaStream_t st) {
  if (p.d == 64)
    finalize_kernel<T, 64><<<(unsigned)p.rows, kFinThreads, 0, st>>>(
        sel, acc, part, static_cast<T*>(out), err_out, kl_out, p, status);
  else
    finalize_kernel<T, 128><<<(unsigned)p.rows, kFinThreads, 0, st>>>(
        sel, acc, part, static_cast<T*>(out), err_out, kl_out, p, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather(int dtype, const void* V, const float* u, const RowSel* sel,
                          const uint32_t* choff, int32_t* idx, float* acc, Partial* part,
                          const Plan& p, cudaStream_t st) {
  if (dtype == kDtypeF32)
    return p.d == 64 ? launch_gather_d<float, 64>(V, u, sel, choff, idx, acc, part, p, st)
                     : launch_gather_d<float, 128>(V, u, sel, choff, idx, acc, part, p, st);
  return p.d == 64 ? launch_gather_d<__nv_bfloat16, 64>(V, u, sel, choff, idx, acc, part, p, st)
                   : launch_gather_d<__nv_bfloat16, 128>(V, u, sel, choff, idx, acc, part, p, st);
}

cudaError_t launch_finalize(int dtype, const RowSel* sel, const float* acc, const Partial* part,
                            void* out, float* err_out, float* kl_out, const Plan& p,
                            uint32_t* status, cudaStream_t st) {
  if (dtype == kDtypeF32)
    return launch_finalize_t<float>(sel, acc, part, out, err_out, kl_out, p, status, st);
  return launch_finalize_t<__nv_bfloat16>(sel, acc, part, out, err_out, kl_out, p, status, st);
}

}  // namespace cta
