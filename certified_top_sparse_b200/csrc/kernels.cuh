// Host-side launchers of the libcta kernels (internal to the library).
#pragma once

#include <cuda.h>  // CUtensorMap
#include <cuda_runtime.h>
#include <stdint.h>

#include "cta.h"
#include "common.cuh"

namespace cta {

constexpr int kDtypeF32 = CTA_F32;
constexpr int kDtypeBF16 = CTA_BF16;

// SMs of the current device (cached per device; 148 if the query fails).
int sm_count();

// Phase 1: logits u [rows, n] and per-(row, chunk) maxima cmax [rows, nchunks].
cudaError_t launch_score(int dtype, const void* q, const void* K, float* u, float* cmax,
                         const Plan& p, uint32_t* status, cudaStream_t st);

// Phase 2: per-row certified selection; writes sel, k_out, tv_out, the kept
// indices (idx_out) and per CTA the largest dropped logit (gmax[row][rank],
// p.gparts per row), using chunk_off as its per-chunk offset scratch.
constexpr int kMaxGParts = 8;
cudaError_t launch_select(const float* u, const float* cmax, RowSel* sel, int32_t* k_out,
                          float* tv_out, uint32_t* chunk_off, int32_t* idx_out, float* gmax,
                          uint32_t* unit_cnt, const Plan& p, uint32_t* status, cudaStream_t st);

// Phase 1 on tcgen05 for the all-query case (bf16, d in {64, 128}, rows of a
// KV group a multiple of 128, n a multiple of 256 and <= kShortMaxN): writes
// the logits only (the short-row selection takes the row maxima itself).
bool score_tc_applies(const Plan& p, int dtype);
cudaError_t launch_score_tc(const void* q, const void* K, float* u, const Plan& p,
                            uint32_t* status, cudaStream_t st);

// Phases 3 and 4 on tcgen05 for the same all-query case (score_tc_applies):
// value sums and the finalisation (out, err, KL) of 128-row tiles.
cudaError_t launch_pv_tc(const void* V, const float* u, const RowSel* sel, const float* gmax,
                         void* out, float* err_out, float* kl_out, float* gap_out, const Plan& p,
                         uint32_t* status, cudaStream_t st);

// Phase 2 for short rows (n <= kShortMaxN): one warp per row; same outputs as
// launch_select (chunk_off unused).
constexpr int kShortMaxN = 1024;
bool select_short_applies(const Plan& p);
cudaError_t launch_select_short(const float* u, RowSel* sel, int32_t* k_out, float* tv_out,
                                int32_t* idx_out, float* gmax, uint32_t* unit_cnt, const Plan& p,
                                uint32_t* status, cudaStream_t st);

// Phases 3 and 4: per-(row, chunk range) weighted value sums of kept (and
// dropped) keys, then (the last CTA of each (KV group, row tile), counted in
// unit_cnt, which selection zeroes) out, err, KL and the single-gap bound.
// gather_ctas_per_sm: the CTAs per SM its launch is planned for.
// The tensor-core decode path (bf16 q, K, V with d = 128), four kernels:
//   launch_score_kv_tc: logits (TMA-fed K stages, the row tile's queries as the
//     B operand), one partial maximum per row and range (Plan::nmax) and the
//     per-range level histograms; zeroes tb.cand_cnt and tb.ticket;
//   launch_bracket_tc: every row's bracket of the cut (tb.brk) from the
//     histograms and maxima, one CTA per row;
//   launch_gather_tc: the value pass after set_ranges_tc: value sums of the
//     keys on either side of the bracket (range partials in acc), exact masses
//     (tb.rrec), window candidates (tb.cand) and the kept-for-certain mask;
//   launch_settle_tc: the exact cut, the kept indices and the outputs.
bool gather_tc_applies(const Plan& p, int dtype);
cudaError_t launch_score_kv_tc(const void* q, const void* K, float* u, float* cmax,
                               const TcBufs& tb, const Plan& p, uint32_t* status,
                               cudaStream_t st);
// Tensor map of a bf16 [groups][n][128] K or V cache: 128-byte-swizzled boxes
// of 64 dimensions x 128 keys (the stages of the streaming tensor-core kernels).
bool encode_kv_map(CUtensorMap* map, const void* base, const Plan& p);
void set_ranges_tc(Plan* p, int sms);
cudaError_t launch_bracket_tc(const float* cmax, const TcBufs& tb, const Plan& p, cudaStream_t st);
cudaError_t launch_gather_tc(const void* V, const float* u, const TcBufs& tb, float* acc,
                             const Plan& p, uint32_t* status, cudaStream_t st);
cudaError_t launch_settle_tc(const void* V, const float* u, const TcBufs& tb, float* acc, void* out,
                             int32_t* k_out, int32_t* idx_out, float* tv_out, float* err_out,
                             float* kl_out, float* gap_out, const Plan& p, uint32_t* status,
                             cudaStream_t st);
int gather_ctas_per_sm(bool want_err);
cudaError_t launch_gather(int dtype, const void* V, const float* u, const RowSel* sel, float* acc,
                          uint32_t* unit_cnt, const float* gmax, void* out, float* err_out,
                          float* kl_out, float* gap_out, const Plan& p, uint32_t* status,
                          cudaStream_t st);


// Dense reference attention (all keys, fp32 online softmax).
cudaError_t launch_dense(int dtype, const void* q, const void* K, const void* V, void* out,
                         int64_t n, int d, int64_t rows, int gm, cudaStream_t st);

}  // namespace cta
