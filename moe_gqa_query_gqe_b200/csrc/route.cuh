// route.cuh -- the per-token router of GQE and the token compaction.
//
// Method: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
// gist.science technical summary, section "Architecture and routing"
// (conditional activation: per token, k query-head experts of every GQA group;
// renormalised weighted sum over the selected experts using router
// probabilities); animattoys.com article, section 4 (a light router scores the
// experts of each group and activates the k best).
//
// Three launches, no host synchronisation between them:
//   router logits + decisions: x Wr on the tensor cores (gemm2.cuh, routing
//                         epilogue): logits + br (fp32), in-group top-k,
//                         renormalised weights, margins, per-chunk counts of
//                         every (group, expert)
//   route_scan_kernel   : exclusive scans of the counts -> segment offsets and
//                         per-chunk bases inside each segment
//   route_scatter_kernel: block-scan of packed per-expert flags -> the
//                         compacted token list of every segment and row_map
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kRouteChunk = 128;      // tokens per chunk (= one routing GEMM tile, one scatter CTA)

struct RouteParams {
  int32_t* sel;
  int32_t* counts;      // [B][nch][G*M]
  int32_t* chunk_base;  // [B][nch][G*M]
  int32_t* seg_off;     // [B*G*M + 1]
  int32_t* seg_tok;
  int32_t* row_map;
  int B, T, G, M, k, nch;
};

// One CTA. Segment s = b*GM + g*M + e (= (b*G + g)*M + e).
__global__ void __launch_bounds__(1024) route_scan_kernel(const RouteParams p) {
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

// One CTA per chunk of kRouteChunk tokens, one thread per token. For every
// group, each thread packs one 8-bit count per expert (M <= 8, counts <= 128)
// into a 64-bit word; a block-wide exclusive scan of the words gives every
// token its rank inside each expert's list for this chunk.
__global__ void __launch_bounds__(kRouteChunk) route_scatter_kernel(const RouteParams p) {
  __shared__ unsigned long long s_warp[kRouteChunk / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x / p.nch, c = blockIdx.x % p.nch;
  const int t = c * kRouteChunk + tid;
  const bool valid = t < p.T;
  const size_t n = (size_t)b * p.T + (valid ? t : 0);
  const int GM = p.G * p.M;
  for (int g = 0; g < p.G; ++g) {
    int es[8];
    unsigned long long mine = 0;
    for (int j = 0; j < p.k; ++j) {
      es[j] = valid ? p.sel[(n * p.G + g) * p.k + j] : 0;
      if (valid) mine += 1ull << (8 * es[j]);
    }
    unsigned long long incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    unsigned long long base = 0;
    for (int w2 = 0; w2 < warp; ++w2) base += s_warp[w2];
    const unsigned long long excl = base + incl - mine;
    if (valid) {
      for (int j = 0; j < p.k; ++j) {
        const int e = es[j];
        const int rank = static_cast<int>((excl >> (8 * e)) & 0xFFull);
        const int ge = g * p.M + e;
        const long long dst = (long long)p.seg_off[b * GM + ge] + p.chunk_base[((size_t)b * p.nch + c) * GM + ge] + rank;
        if (dst < 0 || dst >= (long long)p.B * p.T * p.G * p.k) { flag_bounds_error(); continue; }
        p.seg_tok[dst] = static_cast<int32_t>(n);
        if (p.row_map) p.row_map[(n * p.G + g) * p.k + j] = static_cast<int32_t>(dst);
      }
    }
    __syncthreads();
  }
}

}  // namespace gqe
