// C ABI of libcta: argument checks, launch planning, workspace layout and the
// four-phase launch sequence of certified Top-k attention.  See include/cta.h
// for the contract of every entry point.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "cta.h"
#include "kernels.cuh"

namespace cta {
namespace {

constexpr int kCtasPerSmTarget = 6;    // score pass: ~6 resident CTAs per SM
constexpr int64_t kMaxN = (int64_t)1 << 28;
constexpr int kMaxChunks = 65535;      // grid.y limit

int next_pow2(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

int ceil_log2(int64_t n) {
  int l = 0;
  while (((int64_t)1 << l) < n) ++l;
  return l;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Layout {
  size_t u, cmax, sel, choff, acc, gmax, unit, status;
  // tensor-core decode path only (zero-sized otherwise)
  size_t hist, rrec, srec, brk, cand, cand_cnt, ticket, brk_ready, hmask;
  size_t total;
};

// Output pass: each CTA owns a contiguous range of chunks of one (group, row
// tile); ranges are cut so that the ranges of all units about fill ctas_per_sm
// CTAs on every one of the device's `sms` SMs.
void set_ranges(Plan* p, int ctas_per_sm, int sms) {
  const int64_t units_out = (int64_t)p->groups * p->tiles_out;
  int64_t nr = ((int64_t)ctas_per_sm * sms + units_out - 1) / units_out;
  if (nr > p->nchunks) nr = p->nchunks;
  if (nr < 1) nr = 1;
  p->range_len = (int)((p->nchunks + nr - 1) / nr);
  p->nranges = (int)((p->nchunks + p->range_len - 1) / p->range_len);
}

int make_plan(int64_t n, int d, int n_heads, int n_kv_heads, int batch, int m, int dtype,
              double eps, int sms, Plan* p) {
  if (d != 64 && d != 128) return CTA_ERR_SHAPE;
  if (n < 1 || n > kMaxN) return CTA_ERR_SHAPE;
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return CTA_ERR_SHAPE;
  if (batch < 1 || m < 1) return CTA_ERR_SHAPE;
  const int64_t g = n_heads / n_kv_heads;
  const int64_t gm = g * m;
  const int64_t rows = (int64_t)batch * n_heads * m;
  const int64_t groups = (int64_t)batch * n_kv_heads;
  if (gm > (1 << 24) || rows > INT32_MAX || groups > 65535) return CTA_ERR_SHAPE;
  memset(p, 0, sizeof(*p));
  p->n = n;
  p->ustride = (n + 63) & ~(int64_t)63;  // 256-byte aligned rows for the bulk copies
  p->rows = rows;
  p->d = d;
  p->gm = (int)gm;
  p->groups = (int)groups;
  // Rows per score tile: 8 for fp32, 4 for bf16 (register budget of 2 CTAs/SM).
  const int rt_max = (dtype == CTA_F32) ? 8 : 4;
  p->rt_score = next_pow2((int)(gm < rt_max ? gm : rt_max));
  p->tiles_score = (int)((gm + p->rt_score - 1) / p->rt_score);
  p->rt_out = next_pow2((int)(gm < 4 ? gm : 4));
  p->tiles_out = (int)((gm + p->rt_out - 1) / p->rt_out);
  // Chunk: enough CTAs to fill the GPU, a multiple of 256 keys, at most 4096
  // keys (the logits of a tile are staged in shared memory).
  const int64_t units = groups * p->tiles_score;
  const int64_t target_ctas = (int64_t)kCtasPerSmTarget * sms;
  const int64_t want = (target_ctas + units - 1) / units;
  int64_t chunk = (n + want - 1) / want;
  chunk = ((chunk + 255) / 256) * 256;
  if (chunk < 256) chunk = 256;
  const int64_t max_chunk = (p->rt_score >= 8) ? 2048 : 4096;
  if (chunk > max_chunk) chunk = max_chunk;
  const int64_t nchunks = (n + chunk - 1) / chunk;
  if (nchunks > kMaxChunks) return CTA_ERR_SHAPE;
  p->chunk = (int)chunk;
  p->nchunks = (int)nchunks;
  p->nmax = (int)nchunks;
  p->scale2 = (float)(1.4426950408889634 / sqrt((double)d));  // log2(e)/sqrt(d)
  int s = 62 - ceil_log2(n);
  if (s > 52) s = 52;
  p->mass_shift = s;
  p->two_s = ldexpf(1.0f, s);
  p->eps = eps;
  // Selection: split rows over a cluster of up to 8 CTAs until ~2 CTAs per SM
  // are busy, keeping at least 4096 keys per CTA.
  int cs = 1;
  while (cs < 8 && rows * cs * 2 <= 2 * (int64_t)sms && n / (cs * 2) >= 4096) cs *= 2;
  p->sel_cluster = cs;
  set_ranges(p, 2, sms);
  p->gparts = (p->n <= (int64_t)kShortMaxN) ? 1 : p->sel_cluster;
  return CTA_OK;
}

// Words per row of the value pass's kept-key mask: four per 128-key stage.
int64_t mask_words(const Plan& p) { return 4 * ((p.n + 127) / 128); }

Layout layout(const Plan& p, bool tc_decode) {
  Layout L;
  size_t off = 0;
  L.u = off;      off = align256(off + sizeof(float) * (size_t)p.rows * (size_t)p.ustride);
  L.cmax = off;   off = align256(off + sizeof(float) * (size_t)p.rows * p.nchunks);
  L.sel = off;    off = align256(off + sizeof(RowSel) * (size_t)p.rows);
  L.choff = off;  off = align256(off + sizeof(uint32_t) * (size_t)p.rows * p.nchunks);
  L.acc = off;    off = align256(off + sizeof(float) * (size_t)p.rows * p.nchunks * 2 * p.d);
  L.gmax = off;   off = align256(off + sizeof(float) * (size_t)p.rows * kMaxGParts);
  L.unit = off;   off = align256(off + sizeof(uint32_t) * (size_t)p.rows);
  L.status = off; off = align256(off + sizeof(uint32_t));
  const size_t rr = tc_decode ? (size_t)p.rows * p.nranges : 0;
  const size_t rw = tc_decode ? (size_t)p.rows : 0;
  L.hist = off;     off = align256(off + sizeof(RangeHist) * rr);
  L.rrec = off;     off = align256(off + sizeof(RangeRec) * rr);
  L.srec = off;     off = align256(off + sizeof(SegRec) * rr);
  L.brk = off;      off = align256(off + sizeof(RowBracket) * rw);
  L.cand = off;     off = align256(off + sizeof(unsigned long long) * kCandCap * rw);
  L.cand_cnt = off; off = align256(off + sizeof(uint32_t) * rw);
  L.ticket = off;   off = align256(off + sizeof(uint32_t) * rw);
  L.brk_ready = off; off = align256(off + sizeof(uint32_t) * rw);
  L.hmask = off;    off = align256(off + sizeof(uint32_t) * rw * (size_t)mask_words(p));
  L.total = off;
  return L;
}

// The complete launch plan of one call: shapes, chunking, which kernels run
// (all-query tensor-core tiles, the tensor-core decode path, or the CUDA-core
// kernels) and their ranges.  Used by cta_workspace_size and the call itself.
struct CallPlan {
  Plan p;
  bool tc;   // all-query tensor-core tiles
  bool gtc;  // tensor-core decode path
};

int plan_call(int64_t n, int d, int n_heads, int n_kv_heads, int batch, int m, int dtype,
              double eps, bool want_err, CallPlan* cp) {
  const int sms = sm_count();
  const int rc = make_plan(n, d, n_heads, n_kv_heads, batch, m, dtype, eps, sms, &cp->p);
  if (rc != CTA_OK) return rc;
  Plan& p = cp->p;
  p.want_err = want_err ? 1 : 0;
  set_ranges(&p, gather_ctas_per_sm(want_err), sms);
  cp->tc = score_tc_applies(p, dtype);
  cp->gtc = !cp->tc && gather_tc_applies(p, dtype);
  if (cp->gtc) {
    set_ranges_tc(&p, sms);
    p.nmax = p.nranges;  // the tensor-core logits pass writes one maximum per range
    // the last kernel: the fewest value-pass ranges per CTA that let every CTA
    // be resident at once (two per SM)
    int g = 1;
    while (g < 32 && (int64_t)p.rows * ((p.nranges + g - 1) / g) > 2 * (int64_t)sms) ++g;
    p.settle_group = g;
  }
  return CTA_OK;
}

bool aligned16(const void* x) { return ((uintptr_t)x & 15u) == 0; }

int record(void** ev, int i, cudaStream_t st) {
  if (!ev) return CTA_OK;
  return cudaEventRecord((cudaEvent_t)ev[i], st) == cudaSuccess ? CTA_OK : CTA_ERR_CUDA;
}

}  // namespace
int g_sm_count[64];  // per device, filled on first use (every thread writes the same value)

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (g_sm_count[dev] == 0) {
    int c = 0;
    if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || c <= 0) c = 148;
    g_sm_count[dev] = c;
  }
  return g_sm_count[dev];
}

}  // namespace cta

using namespace cta;

extern "C" {

void cta_opts_init(cta_opts* o) {
  if (!o) return;
  memset(o, 0, sizeof(*o));
  o->batch = 1;
  o->m = 1;
  o->dtype = CTA_BF16;
}

size_t cta_workspace_size(int64_t n, int d, int n_heads, int n_kv_heads, const cta_opts* o) {
  cta_opts def;
  cta_opts_init(&def);
  if (!o) o = &def;
  CallPlan cp;
  if (plan_call(n, d, n_heads, n_kv_heads, o->batch, o->m, o->dtype, 0.5, true, &cp) != CTA_OK)
    return 0;
  return layout(cp.p, cp.gtc).total;
}

int cta_certified_topk_attn(const void* q, const void* K, const void* V, int64_t n, int d,
                            int n_heads, int n_kv_heads, double eps, void* out, int32_t* k_out,
                            int32_t* idx_out, float* tv_out, const cta_opts* opts) {
  if (!q || !K || !V || !out || !k_out || !idx_out || !tv_out) return CTA_ERR_ARG;
  if (!(eps > 0.0 && eps < 1.0)) return CTA_ERR_ARG;
  if (!opts) return CTA_ERR_WORKSPACE;  // the workspace is mandatory
  if (opts->dtype != CTA_F32 && opts->dtype != CTA_BF16) return CTA_ERR_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return CTA_ERR_ARG;
  CallPlan cp;
  const int rc = plan_call(n, d, n_heads, n_kv_heads, opts->batch, opts->m, opts->dtype, eps,
                           opts->err_out != nullptr, &cp);
  if (rc != CTA_OK) return rc;
  const Plan& p = cp.p;
  const bool tc = cp.tc, gtc = cp.gtc;
  const Layout L = layout(p, gtc);
  if (!opts->workspace || ((uintptr_t)opts->workspace & 255u) != 0 || opts->workspace_bytes < L.total)
    return CTA_ERR_WORKSPACE;

  char* ws = static_cast<char*>(opts->workspace);
  float* u = reinterpret_cast<float*>(ws + L.u);
  float* cmax = reinterpret_cast<float*>(ws + L.cmax);
  RowSel* sel = reinterpret_cast<RowSel*>(ws + L.sel);
  uint32_t* choff = reinterpret_cast<uint32_t*>(ws + L.choff);
  float* acc = reinterpret_cast<float*>(ws + L.acc);
  float* gmax = reinterpret_cast<float*>(ws + L.gmax);
  uint32_t* unit_cnt = reinterpret_cast<uint32_t*>(ws + L.unit);
  uint32_t* status = opts->status_dev ? opts->status_dev : reinterpret_cast<uint32_t*>(ws + L.status);
  cudaStream_t st = static_cast<cudaStream_t>(opts->stream);
  void** ev = opts->phase_events;

  if (record(ev, 0, st) != CTA_OK) return CTA_ERR_CUDA;
  if (gtc) {
    // tensor-core decode path: logits (+ level histograms), the row brackets,
    // the bracketed value pass (+ exact masses), then the exact cut, indices
    // and outputs; the events fall between the four kernels
    TcBufs tb;
    tb.hist = reinterpret_cast<RangeHist*>(ws + L.hist);
    tb.rrec = reinterpret_cast<RangeRec*>(ws + L.rrec);
    tb.srec = reinterpret_cast<SegRec*>(ws + L.srec);
    tb.brk = reinterpret_cast<RowBracket*>(ws + L.brk);
    tb.cand = reinterpret_cast<unsigned long long*>(ws + L.cand);
    tb.cand_cnt = reinterpret_cast<uint32_t*>(ws + L.cand_cnt);
    tb.ticket = reinterpret_cast<uint32_t*>(ws + L.ticket);
    tb.brk_ready = reinterpret_cast<uint32_t*>(ws + L.brk_ready);
    tb.hmask = reinterpret_cast<uint32_t*>(ws + L.hmask);
    tb.mask_words = mask_words(p);
    if (launch_score_kv_tc(q, K, u, cmax, tb, p, status, st) != cudaSuccess) return CTA_ERR_CUDA;
    if (record(ev, 1, st) != CTA_OK) return CTA_ERR_CUDA;
    if (launch_bracket_tc(cmax, tb, p, st) != cudaSuccess) return CTA_ERR_CUDA;
    if (record(ev, 2, st) != CTA_OK) return CTA_ERR_CUDA;
    if (launch_gather_tc(V, u, tb, acc, p, status, st) != cudaSuccess) return CTA_ERR_CUDA;
    if (record(ev, 3, st) != CTA_OK) return CTA_ERR_CUDA;
    if (launch_settle_tc(V, u, tb, acc, out, k_out, idx_out, tv_out, opts->err_out, opts->kl_out,
                         opts->gap_out, p, status, st) != cudaSuccess)
      return CTA_ERR_CUDA;
    if (record(ev, 4, st) != CTA_OK) return CTA_ERR_CUDA;
    return CTA_OK;
  }
  if ((tc ? launch_score_tc(q, K, u, p, status, st)
          : launch_score(opts->dtype, q, K, u, cmax, p, status, st)) != cudaSuccess)
    return CTA_ERR_CUDA;
  if (record(ev, 1, st) != CTA_OK) return CTA_ERR_CUDA;
  if ((select_short_applies(p)
           ? launch_select_short(u, sel, k_out, tv_out, idx_out, gmax, unit_cnt, p, status, st)
           : launch_select(u, cmax, sel, k_out, tv_out, choff, idx_out, gmax, unit_cnt, p, status,
                           st)) !=
      cudaSuccess)
    return CTA_ERR_CUDA;
  if (record(ev, 2, st) != CTA_OK) return CTA_ERR_CUDA;
  if (tc) {  // value sums and finalisation in one tensor-core pass
    if (launch_pv_tc(V, u, sel, gmax, out, opts->err_out, opts->kl_out, opts->gap_out, p, status,
                     st) != cudaSuccess)
      return CTA_ERR_CUDA;
    if (record(ev, 3, st) != CTA_OK) return CTA_ERR_CUDA;
  } else {  // value sums, then the last CTA of each row tile finalises it
    if (launch_gather(opts->dtype, V, u, sel, acc, unit_cnt, gmax, out, opts->err_out,
                      opts->kl_out, opts->gap_out, p, status, st) != cudaSuccess)
      return CTA_ERR_CUDA;
    if (record(ev, 3, st) != CTA_OK) return CTA_ERR_CUDA;
  }
  if (record(ev, 4, st) != CTA_OK) return CTA_ERR_CUDA;
  return CTA_OK;
}

int cta_dense_attn(const void* q, const void* K, const void* V, int64_t n, int d, int n_heads,
                   int n_kv_heads, void* out, const cta_opts* opts) {
  cta_opts def;
  cta_opts_init(&def);
  if (!opts) opts = &def;
  if (!q || !K || !V || !out) return CTA_ERR_ARG;
  if (opts->dtype != CTA_F32 && opts->dtype != CTA_BF16) return CTA_ERR_ARG;
  if (!aligned16(q) || !aligned16(K) || !aligned16(V)) return CTA_ERR_ARG;
  Plan p;
  const int rc =
      make_plan(n, d, n_heads, n_kv_heads, opts->batch, opts->m, opts->dtype, 0.5, sm_count(), &p);
  if (rc != CTA_OK) return rc;
  if (launch_dense(opts->dtype, q, K, V, out, n, d, p.rows, p.gm,
                   static_cast<cudaStream_t>(opts->stream)) != cudaSuccess)
    return CTA_ERR_CUDA;
  return CTA_OK;
}

const char* cta_status_string(int status) {
  switch (status) {
    case CTA_OK: return "ok";
    case CTA_ERR_ARG: return "invalid argument (NULL pointer, misaligned tensor, eps outside (0,1) or bad dtype)";
    case CTA_ERR_SHAPE: return "unsupported shape (d not 64/128, n outside [1, 2^28], n_heads % n_kv_heads != 0)";
    case CTA_ERR_WORKSPACE: return "workspace missing, not 256-byte aligned or smaller than cta_workspace_size()";
    case CTA_ERR_CUDA: return "a CUDA launch or runtime call failed";
    case CTA_ERR_NONFINITE: return "non-finite logit";
    case CTA_ERR_TIMEOUT: return "timeout";
    case CTA_ERR_TOO_LARGE: return "problem needs more scratch than the no-allocation entry point holds (CTA_NOALLOC_SCRATCH_BYTES = 32 MiB)";
    default: return "unknown status";
  }
}

int cta_version(void) { return 100; }

}  // extern "C"
