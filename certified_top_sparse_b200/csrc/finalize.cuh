// Phase 4 of the output passes that split a row's keys into ranges: the last
// CTA to finish a (KV group, row tile) adds its rows' range partials in a fixed
// order and forms the outputs.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the exact head-tail
// decomposition Attn = H mu_head + tau mu_tail (H = kept mass, tau = TV), the
// truncated output is Attn_k = mu_head and ||Attn - Attn_k||_2 =
// tau ||mu_tail - mu_head||_2.  KL(Attn_k || Attn) = log(1 / H) =
// log(1 + W_tail / W_head) in unnormalised weights.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace cta {

// Single-gap certificate: u_k the last kept logit, g the largest dropped one.
__device__ __forceinline__ double single_gap_bound(double u_k, double g, int64_t k, int64_t n,
                                                   int d) {
  if (k >= n || !(g > -INFINITY)) return 0.0;
  const double ratio = (double)k / (double)(n - k);
  return 1.0 / (1.0 + ratio * exp((u_k - g) / sqrt((double)d)));
}

// Range partials: acc_out[row][range][a][D], a = 0 kept (head), 1 dropped
// (tail).  Run by NT threads (thread index tid) that synchronise with sync();
// fin is [RT][2][D] doubles of shared memory, s_wh / s_wt [RT] doubles.
template <typename T, int D, int RT, bool ERR, int NT, typename Sync>
__device__ __forceinline__ void finalize_rows(int tid, Sync sync, double* fin, double* s_wh,
                                              double* s_wt, const float* acc_out,
                                              const RowSel* sel, const float* gmax, T* out,
                                              float* err_out, float* kl_out, float* gap_out,
                                              const Plan& p, int64_t row0, int nrows,
                                              uint32_t* status) {
  if (tid < nrows) {
    s_wh[tid] = sel[row0 + tid].wh;
    s_wt[tid] = sel[row0 + tid].wt;
  }
  // sums over the ranges, fixed order: one thread per (row, head/tail, 4 dims),
  // 16-byte loads, eight in flight; fp64 sums staged in shared memory
  constexpr int NA = ERR ? 2 : 1;
  for (int x = tid; x < nrows * NA * (D / 4); x += NT) {
    const int r = x / (NA * (D / 4)), rem = x % (NA * (D / 4));
    const int a = rem / (D / 4), d4 = rem % (D / 4);
    const float4* src =
        reinterpret_cast<const float4*>(acc_out + (row0 + r) * p.nranges * 2 * D + a * D) + d4;
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll 8
    for (int c = 0; c < p.nranges; ++c) {
      const float4 v = __ldcg(src + (int64_t)c * (2 * D / 4));
      s0 += (double)v.x; s1 += (double)v.y; s2 += (double)v.z; s3 += (double)v.w;
    }
    double* f = fin + (r * 2 + a) * D + 4 * d4;
    f[0] = s0; f[1] = s1; f[2] = s2; f[3] = s3;
  }
  sync();
  // every row of the tile at once: thread x -> (row x / D, dimension x % D)
  for (int x = tid; x < nrows * D; x += NT) {
    const int r = x / D, dim = x % D;
    const double mu_h = fin[(r * 2 + 0) * D + dim] / s_wh[r];
    Elem<T>::store1(out + (row0 + r) * D + dim, (float)mu_h);
    if constexpr (ERR) {
      const double diff = s_wt[r] > 0.0 ? fin[(r * 2 + 1) * D + dim] / s_wt[r] - mu_h : 0.0;
      fin[(r * 2 + 1) * D + dim] = diff * diff;  // each element read and rewritten by one thread
    }
  }
  sync();
  if (tid < nrows) {  // thread r: row r's scalars
    const int r = tid;
    const int64_t row = row0 + r;
    const RowSel rs = sel[row];
    const double wh = rs.wh, wt = rs.wt;
    if (!(wh > 0.0)) atomicOr(status, CTA_DEV_INTERNAL);
    if (err_out) {
      double tot = 0.0;
      for (int dim = 0; dim < D; ++dim) tot += fin[(r * 2 + 1) * D + dim];  // fixed order
      err_out[row] = (float)(rs.C < rs.Z && wt > 0.0 ? rs.tv * sqrt(tot) : 0.0);
    }
    if (kl_out) kl_out[row] = (float)log1p(wt / wh);
    if (gap_out) {
      float gm = kNegInf;
      for (int c = 0; c < p.gparts; ++c) gm = fmaxf(gm, __ldcg(gmax + row * kMaxGParts + c));
      gap_out[row] =
          (float)single_gap_bound((double)key_value(rs.kstar), (double)gm, rs.k, p.n, D);
    }
  }
  sync();
}

}  // namespace cta
