// route.cuh -- the per-token router of GQE and the token compaction.
//
// Method: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
// gist.science technical summary, section "Architecture and routing"
// (conditional activation: per token, k query-head experts of every GQA group;
// renormalised weighted sum over the selected experts using router
// probabilities); animattoys.com article, section 4 (a light router scores the
// experts of each group and activates the k best).
//
// Three steps, no host synchronisation between them:
//   router logits + decisions: x Wr on the tensor cores as 256-row tiles of
//                         the CTA-pair GEMM (gemm2sm.cuh; alone, or next to the
//                         K/V projection tiles over the same x). Each CTA's
//                         epilogue holds one chunk of 128 tokens of one
//                         sequence: logits + br (fp32), in-group top-k,
//                         renormalised weights, margins, every token's rank in
//                         its experts' lists within the chunk (kept in sel's
//                         upper bits until the last step), per-chunk counts
//   route_scan_kernel   : exclusive scans of the counts -> segment offsets and
//                         per-chunk bases inside each segment
//   route_finalize_kernel: segment offset + chunk base + rank -> the compacted
//                         token list of every segment and row_map
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kRouteChunk = 128;  // tokens per chunk (= the rows of one CTA of a routing pair tile)

struct RouteParams {
  int32_t* sel;
  int32_t* counts;      // [B][nch][G*M]
  int32_t* chunk_base;  // [B][nch][G*M]
  int32_t* seg_off;     // [B*G*M + 1]
  int32_t* seg_tok;
  int32_t* row_map;
  int B, T, G, M, k, nch;
};

// Decision of one group for one token from its RM logits (br included): top-k
// by logit, exact ties to the lower expert; weights = softmax over the
// selected logits only (the in-group softmax renormalised over the selected
// set); margin = k-th largest minus (k+1)-th largest logit (+inf when k == M).
// Returns the selected experts as a bit mask; when `out` is true writes
// sel[.., j] (ascending expert order), w[.., j], the margin and, when `pr` is
// PR is set, pr[.., j] = the selected expert's in-group softmax probability
// over all M experts (not renormalised; the weighted-concatenation variant).
template <int RM, bool PR = false>
__device__ __forceinline__ uint32_t route_decide(const float (&l)[RM], int k, bool out, int32_t* sel, float* w,
                                                 float* margin, float* pr = nullptr) {
  uint32_t chosen = 0;
  float kth = 0.f;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    float bv = 0.f;
#pragma unroll
    for (int e = 0; e < RM; ++e) {
      const bool free_e = !(chosen & (1u << e));
      if (free_e && (best < 0 || l[e] > bv)) {
        best = e;
        bv = l[e];
      }
    }
    chosen |= 1u << best;
    kth = bv;
  }
  float mg = __int_as_float(0x7f800000);  // +inf when k == M
  if (k < RM) {
    int best = -1;
    float bv = 0.f;
#pragma unroll
    for (int e = 0; e < RM; ++e) {
      const bool free_e = !(chosen & (1u << e));
      if (free_e && (best < 0 || l[e] > bv)) {
        best = e;
        bv = l[e];
      }
    }
    mg = kth - bv;
  }
  if (out) {
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < RM; ++e)
      if (chosen & (1u << e)) mx = fmaxf(mx, l[e]);
    float ex[RM];
    float den = 0.f;
#pragma unroll
    for (int e = 0; e < RM; ++e) {
      ex[e] = (chosen & (1u << e)) ? expf(l[e] - mx) : 0.f;
      den += ex[e];
    }
    const float inv = 1.f / den;
    // all M experts for the full in-group softmax (mx is also the largest
    // logit overall: the best expert is always selected)
    float inv_all = 0.f;
    if constexpr (PR) {
      float den_all = 0.f;
#pragma unroll
      for (int e = 0; e < RM; ++e) den_all += (chosen & (1u << e)) ? ex[e] : expf(l[e] - mx);
      inv_all = 1.f / den_all;
    }
    int j = 0;
#pragma unroll
    for (int e = 0; e < RM; ++e) {
      if (!(chosen & (1u << e))) continue;
      sel[j] = e;
      w[j] = ex[e] * inv;
      if constexpr (PR) pr[j] = ex[e] * inv_all;
      ++j;
    }
    if (margin) *margin = mg;
  }
  return chosen;
}

// One CTA. Segment s = b*GM + g*M + e (= (b*G + g)*M + e).
__global__ void __launch_bounds__(1024) route_scan_kernel(const RouteParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int s_tot[];  // [nseg]
  const int GM = p.G * p.M;
  const int nseg = p.B * GM;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int s = warp; s < nseg; s += nwarps) {
    const int b = s / GM, ge = s % GM;
    int running = 0;
    for (int c0 = 0; c0 < p.nch; c0 += 32) {
      const int c = c0 + lane;
      const size_t idx = ((size_t)b * p.nch + c) * GM + ge;
      const int v = c < p.nch ? p.counts[idx] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (c < p.nch) p.chunk_base[idx] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_tot[s] = running;
  }
  __syncthreads();
  if (warp == 0) {
    int running = 0;
    for (int s0 = 0; s0 < nseg; s0 += 32) {
      const int s = s0 + lane;
      const int v = s < nseg ? s_tot[s] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (s < nseg) p.seg_off[s] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) p.seg_off[nseg] = running;
  }
}

// One thread per (token, group, selection). The routing epilogue leaves
// sel = e | rank << 8, rank being the token's place in expert e's list within
// its chunk; here it becomes the row of the compacted list and sel goes back
// to the expert index.
__global__ void __launch_bounds__(256) route_finalize_kernel(const RouteParams p) {
  pdl_wait();
  pdl_trigger();
  const int GM = p.G * p.M, Gk = p.G * p.k;
  const long long total = (long long)p.B * p.T * Gk;
  const long long rows = total;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const long long n = i / Gk;
    const int g = (int)(i % Gk) / p.k;
    const int b = (int)(n / p.T), c = (int)(n % p.T) / kRouteChunk;
    const int packed = p.sel[i];
    const int e = packed & 0xFF, rank = packed >> 8;
    p.sel[i] = e;
    if (e >= p.M || rank < 0 || rank >= kRouteChunk) {
      flag_bounds_error();
      continue;
    }
    const int ge = g * p.M + e;
    const long long dst = (long long)p.seg_off[b * GM + ge] + p.chunk_base[((size_t)b * p.nch + c) * GM + ge] + rank;
    if (dst < 0 || dst >= rows) {
      flag_bounds_error();
      continue;
    }
    p.seg_tok[dst] = static_cast<int32_t>(n);
    if (p.row_map) p.row_map[i] = static_cast<int32_t>(dst);
  }
}

// Scan and compaction in one launch, for problems whose per-chunk counts fit
// in shared memory (B * nch * G*M <= kRouteFusedMax). Every block rebuilds,
// from the counts, the exclusive prefixes it needs (segment offsets over all
// segments, chunk bases within each segment) in its own shared memory, then
// places its (token, group, selection) items as route_finalize_kernel does;
// block 0 also writes seg_off. The counts are a few KB, so the redundant
// per-block scan costs less than a second launch.
constexpr int kRouteFusedMax = 4096;

__global__ void __launch_bounds__(1024) route_scan_finalize_kernel(const RouteParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int sh[];
  const int GM = p.G * p.M, Gk = p.G * p.k;
  const int nseg = p.B * GM;
  const int ncnt = nseg * p.nch;
  int* s_base = sh;            // [B][nch][GM]: chunk base within its segment
  int* s_off = sh + ncnt;      // [nseg + 1]: segment offsets
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < ncnt; i += blockDim.x) s_base[i] = p.counts[i];
  __syncthreads();
  // per segment (one warp each): exclusive scan over its chunks, in place
  for (int sgi = warp; sgi < nseg; sgi += blockDim.x >> 5) {
    const int b = sgi / GM, ge = sgi % GM;
    int running = 0;
    for (int c0 = 0; c0 < p.nch; c0 += 32) {
      const int c = c0 + lane;
      const int idx = (b * p.nch + c) * GM + ge;
      const int v = c < p.nch ? s_base[idx] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (c < p.nch) s_base[idx] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[sgi] = running;  // the segment's total, scanned below
  }
  __syncthreads();
  if (warp == 0) {
    int running = 0;
    for (int s0 = 0; s0 < nseg; s0 += 32) {
      const int sgi = s0 + lane;
      const int v = sgi < nseg ? s_off[sgi] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (sgi < nseg) s_off[sgi] = running + incl - v;
      running += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[nseg] = running;
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int i = tid; i <= nseg; i += blockDim.x) p.seg_off[i] = s_off[i];
  const long long total = (long long)p.B * p.T * Gk;
  for (long long i = blockIdx.x * (long long)blockDim.x + tid; i < total; i += (long long)gridDim.x * blockDim.x) {
    const long long n = i / Gk;
    const int g = (int)(i % Gk) / p.k;
    const int b = (int)(n / p.T), c = (int)(n % p.T) / kRouteChunk;
    const int packed = p.sel[i];
    const int e = packed & 0xFF, rank = packed >> 8;
    p.sel[i] = e;
    if (e >= p.M || rank < 0 || rank >= kRouteChunk) {
      flag_bounds_error();
      continue;
    }
    const int ge = g * p.M + e;
    const long long dst = (long long)s_off[b * GM + ge] + s_base[(b * p.nch + c) * GM + ge] + rank;
    if (dst < 0 || dst >= total) {
      flag_bounds_error();
      continue;
    }
    p.seg_tok[dst] = static_cast<int32_t>(n);
    if (p.row_map) p.row_map[i] = static_cast<int32_t>(dst);
  }
}

}  // namespace gqe
