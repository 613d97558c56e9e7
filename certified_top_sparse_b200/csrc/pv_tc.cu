// Phase 3 for the all-query case on the 5th-generation tensor cores:
// O_head = P_head V and O_tail = P_tail V for 128 query rows at a time.
//
// Method ("A Mathematical Theory of Top-k Sparse Attention via Total Variation
// Distance", arXiv 2512.07647, abstract): with the exact head-tail
// decomposition Attn = H mu_head + tau mu_tail, the truncated output is
// mu_head = sum_{head} w_i v_i / sum_{head} w_i, and the error needs mu_tail.
//
// One CTA of 256 threads per (KV group, 128-row tile).  Per 64-key chunk the
// threads turn their row's logits into weights (2 threads per row, 32 keys
// each) and write the kept and the dropped weights as A operands, each split
// into two bf16 parts (hi = bf16(w), lo = bf16(w - hi): |w - hi - lo| <=
// 2^-18 |w|), in the 128-byte-swizzled K-major layout; the chunk's V rows are
// the B operand in the MN-major layout (same swizzled bytes: 8 keys x 64 dims
// per 1024-byte atom).  tcgen05.mma (bf16 x bf16 -> fp32) accumulates
// O_head += (P_head,hi + P_head,lo) V and O_tail likewise in tensor memory;
// A and V are double-buffered so the conversion of chunk j+1 overlaps the MMAs
// of chunk j.  Each thread then finalises its row from tensor memory: out =
// mu_head (fp64 division by selection's kept-weight sum), the error, KL and
// the single-gap certificate.
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "umma.cuh"

namespace cta {

namespace {

constexpr int kPvRows = 128;      // M: query rows per CTA (TMEM lanes)
constexpr int kPvKeys = 64;       // keys per chunk: one 128-byte swizzle atom of bf16
constexpr int kPvThreads = 256;   // two threads per row
constexpr int kATile = kPvRows * kSwRowBytes;  // one A matrix of a chunk: 128 rows x 64 bf16 = 16 KB

// bf16 hi/lo parts of two weights, packed (lower key in the low half).
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 ah = __float2bfloat16_rn(a), bh = __float2bfloat16_rn(b);
  const __nv_bfloat16 al = __float2bfloat16_rn(a - __bfloat162float(ah));
  const __nv_bfloat16 bl = __float2bfloat16_rn(b - __bfloat162float(bh));
  hi = (uint32_t)__bfloat16_as_ushort(ah) | ((uint32_t)__bfloat16_as_ushort(bh) << 16);
  lo = (uint32_t)__bfloat16_as_ushort(al) | ((uint32_t)__bfloat16_as_ushort(bl) << 16);
}

template <int D, bool ERR>
struct PvSmem {
  static constexpr int NA = ERR ? 4 : 2;                  // A matrices per chunk
  static constexpr int kA = NA * kATile;                   // A bytes per buffer
  static constexpr int kV = kPvKeys * D * 2;               // V bytes per buffer
  static constexpr size_t kBytes = 1024 + 2 * (size_t)(kA + kV);
  static constexpr int kCols = ERR ? 2 * D : D;            // TMEM columns (head, tail)
};

template <int D, bool ERR>
__global__ void __launch_bounds__(kPvThreads, ERR ? 1 : 2)
pv_tc_kernel(const __nv_bfloat16* __restrict__ V, const float* __restrict__ u,
             const RowSel* __restrict__ sel, const float* __restrict__ gmax,
             __nv_bfloat16* __restrict__ out, float* __restrict__ err_out,
             float* __restrict__ kl_out, float* __restrict__ gap_out, Plan p,
             uint32_t* __restrict__ status) {
  using S = PvSmem<D, ERR>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char* abuf = base;                  // [2][NA][128 rows][128 B]
  unsigned char* vbuf = base + 2 * S::kA;      // [2][D/64][64 keys][128 B]
  __shared__ unsigned long long done[2];       // MMAs of the chunk in buffer b finished
  __shared__ uint32_t tmem_slot;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = p.gm / kPvRows;
  const int group = blockIdx.x / tiles, tile = blockIdx.x % tiles;
  const int64_t row0 = (int64_t)group * p.gm + (int64_t)tile * kPvRows;
  const int r = threadIdx.x % kPvRows;   // this thread's row (TMEM lane)
  const int half = threadIdx.x / kPvRows;  // which 32 keys of a chunk it converts

  if (warp == 0) tmem_alloc(&tmem_slot, S::kCols);
  if (threadIdx.x == 0) {
    mbar_init(&done[0], 1);
    mbar_init(&done[1], 1);
    mbar_fence_init();
  }
  const RowSel rs = sel[row0 + r];
  const float* ur = u + (row0 + r) * p.ustride;
  const __nv_bfloat16* Vg = V + (int64_t)group * p.n * D;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  constexpr uint32_t idesc = idesc_bf16(kPvRows, D, /*a_mn=*/false, /*b_mn=*/true);
  const int nch = (int)(p.n / kPvKeys);
  bool ok = true;

  // Chunk j + 1's logits and V pieces are loaded into registers while chunk j
  // is converted and multiplied (software pipelining over the chunks).
  constexpr int P = D / 8;                              // 16-byte pieces per V row
  constexpr int VPT = kPvKeys * P / kPvThreads;         // V pieces per thread and chunk
  static_assert(kPvKeys * P % kPvThreads == 0, "V pieces split evenly");
  float x[32];
  uint4 vv[VPT];
  auto load_chunk = [&](int j, float* xs, uint4* vs) {
    const float4* src = reinterpret_cast<const float4*>(ur + j * kPvKeys + half * 32);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float4 f = __ldg(src + e);
      xs[4 * e] = f.x; xs[4 * e + 1] = f.y; xs[4 * e + 2] = f.z; xs[4 * e + 3] = f.w;
    }
    const __nv_bfloat16* vsrc = Vg + (int64_t)j * kPvKeys * D;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int q = threadIdx.x + i * kPvThreads, key = q / P, c = q % P;
      vs[i] = __ldg(reinterpret_cast<const uint4*>(vsrc + (int64_t)key * D) + c);
    }
  };
  if (nch > 0) load_chunk(0, x, vv);

  for (int j = 0; j < nch; ++j) {
    const int b = j & 1;
    // the MMAs that last read buffer b (chunk j - 2) must be done
    if (j >= 2 && !mbar_wait(&done[b], (unsigned)((j - 2) >> 1) & 1u)) ok = false;
    if (__syncthreads_or(ok ? 0 : 1)) break;
    unsigned char* ab = abuf + b * S::kA;
    unsigned char* vb = vbuf + b * S::kV;
    float xn[32];
    uint4 vn[VPT];
    if (j + 1 < nch) load_chunk(j + 1, xn, vn);
    // ---- weights of 32 keys of this row -> A operands (hi, lo; head, tail) --
    {
      const int k0 = j * kPvKeys + half * 32;
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // 16-byte piece c of this thread's 64 bytes
        uint32_t hh[4], hl[4], th[4], tl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float w2[2], kh[2], kd[2];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int kk = 8 * c + 2 * e + t;
            const float xv = x[kk];
            w2[t] = weight(xv, rs.M, p.scale2);
            const bool kept = is_kept(order_key(xv), (uint32_t)(k0 + kk), rs.kstar, (uint32_t)rs.istar);
            kh[t] = kept ? w2[t] : 0.0f;
            kd[t] = kept ? 0.0f : w2[t];
          }
          split2(kh[0], kh[1], hh[e], hl[e]);
          if constexpr (ERR) split2(kd[0], kd[1], th[e], tl[e]);
        }
        const uint32_t off = sw128_offset(r, half * 4 + c, kPvRows);
        *reinterpret_cast<uint4*>(ab + 0 * kATile + off) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
        *reinterpret_cast<uint4*>(ab + 1 * kATile + off) = make_uint4(hl[0], hl[1], hl[2], hl[3]);
        if constexpr (ERR) {
          *reinterpret_cast<uint4*>(ab + 2 * kATile + off) = make_uint4(th[0], th[1], th[2], th[3]);
          *reinterpret_cast<uint4*>(ab + 3 * kATile + off) = make_uint4(tl[0], tl[1], tl[2], tl[3]);
        }
      }
    }
    // ---- the chunk's V rows (B operand, MN-major swizzled) -----------------
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int q = threadIdx.x + i * kPvThreads, key = q / P, c = q % P;
      *reinterpret_cast<uint4*>(vb + sw128_offset(key, c, kPvKeys)) = vv[i];
    }
    fence_proxy_async();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t a0 = smem_u32(ab), v0 = smem_u32(vb);
      constexpr uint32_t lbo = kPvKeys * kSwRowBytes;  // 64-dim blocks of V, 8 KB apart
#pragma unroll
      for (int s = 0; s < kPvKeys / 16; ++s) {
        const unsigned long long bd = desc_mnmajor(v0 + (uint32_t)(s * 2048), lbo);
        const uint32_t acc = (j > 0 || s > 0) ? 1u : 0u;
        tc_mma(tmem, desc_kmajor(a0 + 0 * kATile + s * 32), bd, idesc, acc);
        tc_mma(tmem, desc_kmajor(a0 + 1 * kATile + s * 32), bd, idesc, 1u);
        if constexpr (ERR) {
          tc_mma(tmem + D, desc_kmajor(a0 + 2 * kATile + s * 32), bd, idesc, acc);
          tc_mma(tmem + D, desc_kmajor(a0 + 3 * kATile + s * 32), bd, idesc, 1u);
        }
      }
      tc_commit(&done[b]);
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = xn[e];
#pragma unroll
    for (int i = 0; i < VPT; ++i) vv[i] = vn[i];
  }
  // ---- the last chunks' MMAs, then the sums out of tensor memory -----------
  if (ok && nch >= 1 && !mbar_wait(&done[(nch - 1) & 1], (unsigned)((nch - 1) >> 1) & 1u)) ok = false;
  if (ok && nch >= 2 && !mbar_wait(&done[(nch - 2) & 1], (unsigned)((nch - 2) >> 1) & 1u)) ok = false;
  if (!ok && lane == 0) atomicOr(status, CTA_DEV_TIMEOUT);
  tc_fence_after();
  if (ok && threadIdx.x < kPvRows) {
    // the finalisation of this row: out = mu_head, err = tau ||mu_tail - mu_head||,
    // KL = log(1 + W_tail / W_head), with selection's fp64 weight sums
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const double wh = rs.wh, wt = rs.wt;
    __nv_bfloat16* orow = out + (row0 + r) * D;
    double sq = 0.0;
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      uint32_t h[32];
      tc_ld32(lane_addr + (uint32_t)(cb * 32), h);
      uint32_t packed[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float o0 = (float)((double)__uint_as_float(h[2 * e]) / wh);
        const float o1 = (float)((double)__uint_as_float(h[2 * e + 1]) / wh);
        packed[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o0)) |
                    ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o1)) << 16);
      }
      uint4* o4 = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        o4[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
      if constexpr (ERR) {
        uint32_t t[32];
        tc_ld32(lane_addr + (uint32_t)(D + cb * 32), t);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const double mh = (double)__uint_as_float(h[e]) / wh;
          const double diff = wt > 0.0 ? (double)__uint_as_float(t[e]) / wt - mh : 0.0;
          sq += diff * diff;
        }
      }
    }
    if (!(wh > 0.0)) atomicOr(status, CTA_DEV_INTERNAL);
    if (err_out) err_out[row0 + r] = (float)(rs.C < rs.Z && wt > 0.0 ? rs.tv * sqrt(sq) : 0.0);
    if (kl_out) kl_out[row0 + r] = (float)log1p(wt / wh);
    if (gap_out) {  // single-gap certificate from the last kept and the largest dropped logit
      float g = kNegInf;
      for (int c = 0; c < p.gparts; ++c) g = fmaxf(g, gmax[(row0 + r) * kMaxGParts + c]);
      double b = 0.0;
      if (rs.k < p.n && g > kNegInf) {
        const double ratio = (double)rs.k / (double)(p.n - rs.k);
        b = 1.0 / (1.0 + ratio * exp(((double)key_value(rs.kstar) - (double)g) / sqrt((double)D)));
      }
      gap_out[row0 + r] = (float)b;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, S::kCols);
}

template <int D, bool ERR>
cudaError_t launch_pv_t(const void* V, const float* u, const RowSel* sel, const float* gmax,
                        void* out, float* err_out, float* kl_out, float* gap_out, const Plan& p,
                        uint32_t* status, cudaStream_t st) {
  const size_t smem = PvSmem<D, ERR>::kBytes;
  auto kern = pv_tc_kernel<D, ERR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(p.groups * (p.gm / kPvRows));
  kern<<<grid, kPvThreads, smem, st>>>(static_cast<const __nv_bfloat16*>(V), u, sel, gmax,
                                       static_cast<__nv_bfloat16*>(out), err_out, kl_out, gap_out,
                                       p, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pv_tc(const void* V, const float* u, const RowSel* sel, const float* gmax,
                         void* out, float* err_out, float* kl_out, float* gap_out, const Plan& p,
                         uint32_t* status, cudaStream_t st) {
  if (p.d == 64)
    return p.want_err ? launch_pv_t<64, true>(V, u, sel, gmax, out, err_out, kl_out, gap_out, p,
                                              status, st)
                      : launch_pv_t<64, false>(V, u, sel, gmax, out, err_out, kl_out, gap_out, p,
                                               status, st);
  return p.want_err ? launch_pv_t<128, true>(V, u, sel, gmax, out, err_out, kl_out, gap_out, p,
                                             status, st)
                    : launch_pv_t<128, false>(V, u, sel, gmax, out, err_out, kl_out, gap_out, p,
                                              status, st);
}

}  // namespace cta
