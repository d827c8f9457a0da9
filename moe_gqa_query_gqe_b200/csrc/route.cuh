// route.cuh -- the per-token router of GQE and the token compaction.
//
// Method: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
// gist.science technical summary, section "Architecture and routing"
// (conditional activation: per token, k query-head experts of every GQA group;
// renormalised weighted sum over the selected experts using router
// probabilities); animattoys.com article, section 4 (a light router scores the
// experts of each group and activates the k best).
//
// Three kernels, no host synchronisation between them:
//   route_select_kernel : logits = x Wr + br (fp32), in-group softmax, top-k,
//                         renormalised weights, margins; per-chunk counts of
//                         every (group, expert)
//   route_scan_kernel   : exclusive scans of the counts -> segment offsets and
//                         per-chunk bases inside each segment
//   route_scatter_kernel: block-scan of packed per-expert flags -> the
//                         compacted token list of every segment and row_map
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kRouteChunk = 128;      // tokens per chunk (select and scatter CTAs)
constexpr int kRouteWarps = 8;        // warps of a select CTA
constexpr int kRouteMaxWrBytes = 128 * 1024;

struct RouteParams {
  const __nv_bfloat16* x;
  const __nv_bfloat16* Wr;
  const float* br;
  int32_t* sel;
  float* w;
  float* margin;
  int32_t* counts;      // [B][nch][G*M]
  int32_t* chunk_base;  // [B][nch][G*M]
  int32_t* seg_off;     // [B*G*M + 1]
  int32_t* seg_tok;
  int32_t* row_map;
  int B, T, D, G, M, k, nch;
};

// Recursive-halving reduce-scatter over the 32 lanes: on entry every lane
// holds V partial sums; on exit lane l holds the complete sums of entries
// [l*V/32, (l+1)*V/32) in v[0 .. V/32-1]. V is a power of two >= 32.
template <int V>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[V], int lane) {
#pragma unroll
  for (int step = 16, len = V; step >= 1; step >>= 1, len >>= 1) {
    const bool upper = (lane & step) != 0;
    const int half = len / 2;
#pragma unroll
    for (int i = 0; i < V / 2; ++i) {
      if (i < half) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, step);
      }
    }
  }
}

// GM = G*M (power of two, 2..64). TPW tokens per warp pass, V = TPW*GM sums.
template <int GM>
__global__ void __launch_bounds__(kRouteWarps * 32) route_select_kernel(const RouteParams p) {
  constexpr int TPW = (64 / GM) < 1 ? 1 : ((64 / GM) > 16 ? 16 : (64 / GM));
  constexpr int V = TPW * GM;
  static_assert(V >= 32 && (V & (V - 1)) == 0, "V must be a power of two >= 32");
  constexpr int PIECES = GM;  // 16-byte pieces in a row-block of 8 d's (8*GM bf16)

  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* s_wr = smem;                                                      // D*GM bf16, swizzled
  float* s_red = reinterpret_cast<float*>(smem + (size_t)p.D * GM * 2);      // [warps][V]
  int* s_cnt = reinterpret_cast<int*>(s_red + kRouteWarps * V);              // [GM]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.x / p.nch, c = blockIdx.x % p.nch;
  const int t_begin = c * kRouteChunk;

  // Stage Wr: row-block rb = d/8 (8 rows x GM columns, 16*GM bytes); 16-byte
  // piece q of row-block rb is stored at piece (q ^ (rb % PIECES)), so that
  // lanes reading consecutive row-blocks hit distinct banks.
  {
    const int nblk = p.D / 8;
    const uint4* src = reinterpret_cast<const uint4*>(p.Wr);
    for (int i = tid; i < nblk * PIECES; i += blockDim.x) {
      const int rb = i / PIECES, q = i % PIECES;
      const int phys = rb * PIECES + (q ^ (rb & (PIECES - 1)));
      reinterpret_cast<uint4*>(s_wr)[phys] = src[i];
    }
    for (int i = tid; i < GM; i += blockDim.x) s_cnt[i] = 0;
  }
  __syncthreads();

  const int tokens_per_warp = kRouteChunk / kRouteWarps;
  for (int tw = 0; tw < tokens_per_warp; tw += TPW) {
    const int tl0 = warp * tokens_per_warp + tw;  // first token (chunk-local) of this pass
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.f;

    for (int rb = lane; rb < p.D / 8; rb += 32) {
      uint4 xv[TPW];
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        const int tt = t_begin + tl0 + t;
        if (tt < p.T)
          xv[t] = __ldg(reinterpret_cast<const uint4*>(p.x + ((size_t)b * p.T + tt) * p.D) + rb);
        else
          xv[t] = make_uint4(0, 0, 0, 0);
      }
      const uint4* wr = reinterpret_cast<const uint4*>(s_wr) + (size_t)rb * PIECES;
#pragma unroll
      for (int q = 0; q < PIECES; ++q) {
        const uint4 wq = wr[q ^ (rb & (PIECES - 1))];
        const uint32_t wu[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const int el = q * 8 + h;  // element of the row-block: row r = el / GM, expert col = el % GM
          const int r = el / GM, col = el % GM;
          const float wv = (h & 1) ? bf16hi_to_f32(wu[h >> 1]) : bf16lo_to_f32(wu[h >> 1]);
#pragma unroll
          for (int t = 0; t < TPW; ++t) {
            const uint32_t xu = (r >> 1) == 0 ? xv[t].x : (r >> 1) == 1 ? xv[t].y : (r >> 1) == 2 ? xv[t].z : xv[t].w;
            const float xf = (r & 1) ? bf16hi_to_f32(xu) : bf16lo_to_f32(xu);
            acc[t * GM + col] = fmaf(xf, wv, acc[t * GM + col]);
          }
        }
      }
    }

    warp_reduce_scatter<V>(acc, lane);
    float* red = s_red + warp * V;
#pragma unroll
    for (int i = 0; i < V / 32; ++i) red[lane * (V / 32) + i] = acc[i];
    __syncwarp();

    // one lane per (token, group): softmax, top-k, renormalised weights
    for (int pr = lane; pr < TPW * p.G; pr += 32) {
      const int tk = pr / p.G, g = pr % p.G;
      const int tt = t_begin + tl0 + tk;
      if (tt >= p.T) continue;
      const size_t n = (size_t)b * p.T + tt;
      float lg[8];
      for (int e = 0; e < p.M; ++e) {
        float v = red[tk * GM + g * p.M + e];
        if (p.br) v += p.br[g * p.M + e];
        lg[e] = v;
      }
      // pick k times the largest remaining logit, ties -> lower expert index
      uint32_t chosen = 0;
      float kth = 0.f;
      for (int j = 0; j < p.k; ++j) {
        int best = -1;
        float bv = 0.f;
        for (int e = 0; e < p.M; ++e) {
          if (chosen & (1u << e)) continue;
          if (best < 0 || lg[e] > bv) { best = e; bv = lg[e]; }
        }
        chosen |= 1u << best;
        kth = bv;
      }
      float mg = __int_as_float(0x7f800000);  // +inf when k == M
      if (p.k < p.M) {
        int best = -1;
        float bv = 0.f;
        for (int e = 0; e < p.M; ++e) {
          if (chosen & (1u << e)) continue;
          if (best < 0 || lg[e] > bv) { best = e; bv = lg[e]; }
        }
        mg = kth - bv;
      }
      float mx = -INFINITY;
      for (int e = 0; e < p.M; ++e)
        if (chosen & (1u << e)) mx = fmaxf(mx, lg[e]);
      float den = 0.f;
      for (int e = 0; e < p.M; ++e)
        if (chosen & (1u << e)) den += expf(lg[e] - mx);
      const float inv = 1.f / den;
      int j = 0;
      for (int e = 0; e < p.M; ++e) {
        if (!(chosen & (1u << e))) continue;
        const size_t o = (n * p.G + g) * p.k + j;
        p.sel[o] = e;
        p.w[o] = expf(lg[e] - mx) * inv;
        atomicAdd(&s_cnt[g * p.M + e], 1);
        ++j;
      }
      if (p.margin) p.margin[n * p.G + g] = mg;
    }
    __syncwarp();
  }
  __syncthreads();
  for (int i = tid; i < GM; i += blockDim.x) p.counts[((size_t)b * p.nch + c) * GM + i] = s_cnt[i];
}

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
