// decode_proj.cuh -- the token-side work of one decode step for up to
// kSkinnyMaxTokens new tokens: routing, the K/V and query projections and the
// output construction with its projection, as skinny products, each 64-column
// weight slice split over the rows of a cluster.
//
// Method: the layer of the gist.science summary ("Architecture and routing":
// conditional activation, renormalised weighted sum, dense K/V, output
// construction) and the animattoys.com article (section 4), applied to the
// new token of every sequence; the aiboss88.com wiki on grouped-query
// attention, inference section (the new token's key/value rows are appended
// to the cache).
//
// With a few dozen rows a projection is a read of its weights: B x K times
// K x 64 per 64-column slice. The tensor-core tiles of the prefill path would
// pad the B rows to 256 and stream each weight through a few SMs; here every
// slice is read by its own cluster of kSkCluster CTAs. CTA rank q loads rows
// [q RR, q RR + RR) of the slice by TMA (RR: the slice's rows / kSkCluster,
// rounded up to whole kSkBoxRows boxes) and multiplies them with the same
// rows of all the tokens' inputs (staged once, up to kSkinnyMaxTokens); the
// eight partial sums meet in distributed shared memory, where rank q adds up
// tokens [8q, 8q + 8) (ranks in order, so the sum is the same on every run).
// A launch takes two cluster barriers whatever the token count.
//   decode_proj_kernel : 2G + 1 + G*M clusters: K and V of group g (written
//                        into the caches at cache_len[b]), the shared head's
//                        query, and routed head h = g*M + e: its query and
//                        group g's router logits x Wr + br for every token;
//                        rank q decides its tokens for group g and keeps a
//                        token's query row if it selected e (the e = 0
//                        cluster writes sel, w, margin)
//   decode_out_kernel  : D / 64 clusters: y = A Wo, A = [concat | per-group
//                        slot sum_j w_j O_j | shared] built for the CTA's rows
//                        (A's columns) from O and w (the slot rounded to
//                        bf16, as the combine kernel does)
// A CTA's product is mma.sync m16n8k16 (bf16 in, fp32 accumulate): warp w
// takes the slice's columns [8w, 8w + 8) for every 16-token tile, A (the
// tokens' rows) by matrix loads from a padded buffer, B (the weight rows,
// [k][n] in the TMA's 128-byte swizzle) by transposing matrix loads. Every
// launch issues its weight loads before its dependency wait (weights depend
// on no launch).
#pragma once

#include "decode.cuh"
#include "route.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kSkinnyMaxTokens = 64;
constexpr int kSkCluster = 8;
constexpr int kSkinnyThreads = 256;  // 8 warps: one 8-column tile of the slice each
constexpr int kSkPerRank = kSkinnyMaxTokens / kSkCluster;  // tokens a rank adds up
constexpr int kSkBoxRows = 32; // TMA box: 64 columns x 32 rows, 4 KB
static_assert(kSkPerRank <= 8 && kSkinnyMaxTokens % 16 == 0, "decision area and 16-token tiles");

struct DecodeProjParams {
  // weights as TMA tensor maps: box 64 columns x kSkBoxRows rows, 128-byte swizzle
  CUtensorMap tmWq, tmWk, tmWv, tmWr, tmWo;
  const __nv_bfloat16* x;   // [B, D] new tokens
  const float* br;          // [G*M] or null
  const int32_t* cache_len; // [B]
  __nv_bfloat16* Kc;        // [B, T, G, 64]
  __nv_bfloat16* Vc;
  __nv_bfloat16* Q;         // [B, G*k + 1, 64]
  int32_t* sel;             // [B, G, k]
  float* w;                 // [B, G, k]
  float* margin;            // [B, G] or null
  const __nv_bfloat16* O;   // [B, G*k + 1, 64]
  __nv_bfloat16* y;         // [B, D]
  int B, T, D, G, M, k;
};

// Rows of a K-row slice per CTA.
__host__ __device__ inline int sk_rows(int K) {
  const int r = (K + kSkCluster - 1) / kSkCluster;
  return (r + kSkBoxRows - 1) / kSkBoxRows * kSkBoxRows;
}
// Shared memory (from a 1024-aligned base): the CTA's weight rows wbuf
// [RR][128 B] and, with `router`, the router rows wbuf_r [RR][128 B]; their
// barriers and the abort flag (64 B); all tokens' input rows xs [cap][RR + 8]
// (bf16; the 16-byte pad makes the rows of a matrix load fall in different
// banks); the CTA's partials part (and, with `router`, part_r) [cap][64] (read
// by the cluster); the decision area: logits [8][8] and slots [8]. cap is B
// rounded up to a 16-token tile, so a small step leaves room on the SM for
// the attention launch's CTAs.
__host__ __device__ inline int sk_cap(int B) { return (B + 15) / 16 * 16; }
__host__ __device__ inline int sk_smem(int K, bool router, int B) {
  const int RR = sk_rows(K), cap = sk_cap(B);
  return 1024 + (router ? 2 : 1) * RR * 128 + 64 + cap * (RR + 8) * 2 + (router ? 2 : 1) * cap * 64 * 4 + 64 * 4 +
         8 * 4;
}

struct SkCta {
  uint8_t* wbuf;
  uint8_t* wbuf_r;
  uint64_t* bar;
  uint64_t* bar_r;
  volatile int* abort_flag;
  __nv_bfloat16* xs;  // [cap][RR + 8]
  float* part;
  float* part_r;
  float* logits;  // [8 tokens][8]
  int* slot;      // [8 tokens]
  int RR, row0, rank, cap;
};

__device__ __forceinline__ SkCta sk_init(uint8_t* raw, int K, bool router, int B) {
  SkCta s;
  uint8_t* b = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
  s.RR = sk_rows(K);
  s.cap = sk_cap(B);
  s.rank = (int)cluster_ctarank();
  s.row0 = s.rank * s.RR;
  s.wbuf = b;
  s.wbuf_r = b + s.RR * 128;
  uint8_t* h = b + (router ? 2 : 1) * s.RR * 128;
  s.bar = reinterpret_cast<uint64_t*>(h);
  s.bar_r = s.bar + 1;
  s.abort_flag = reinterpret_cast<volatile int*>(h + 16);
  s.xs = reinterpret_cast<__nv_bfloat16*>(h + 64);
  s.part = reinterpret_cast<float*>(h + 64 + s.cap * (s.RR + 8) * 2);
  s.part_r = s.part + s.cap * 64;  // (router only)
  s.logits = s.part + (router ? 2 : 1) * s.cap * 64;
  s.slot = reinterpret_cast<int*>(s.logits + 64);
  if (threadIdx.x == 0) {
    mbar_init(s.bar, 1);
    mbar_init(s.bar_r, 1);
    *s.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  return s;
}

// Thread 0: TMA loads of this CTA's rows of the slice starting at column
// col0 into wbuf (all boxes on barrier bar; rows past the weight read as zero).
__device__ __forceinline__ void sk_load(const SkCta& s, uint8_t* wbuf, uint64_t* bar, const CUtensorMap* tm,
                                        int col0) {
  if (threadIdx.x == 0) {
    const int nbox = s.RR / kSkBoxRows;
    mbar_arrive_expect_tx(bar, nbox * kSkBoxRows * 128);
    for (int i = 0; i < nbox; ++i)
      tma_load_2d(wbuf + i * kSkBoxRows * 128, tm, bar, col0, s.row0 + i * kSkBoxRows);
  }
}

// part[n][c] = sum over this CTA's rows r of xs[n][r] * W[row0 + r][col0 + c]
// for tokens n < ntok (rounded up to 16, the rest zero) and the slice in wbuf
// (columns at or past ncols are zeros). Warp w computes columns [8w, 8w + 8)
// for every 16-token tile on mma.sync m16n8k16. Waits for the weights first.
// Returns false if that wait ran out (part is then zero).
__device__ __forceinline__ bool sk_product(const SkCta& s, const uint8_t* wbuf, uint64_t* bar, int ncols, int ntok,
                                           float* part) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool ok = __syncthreads_and(mbar_wait(bar, 0, s.abort_flag));
  const int RRp = s.RR + 8;
  const int nmt = (ntok + 15) / 16;  // 16-token tiles
  const int col = warp * 8;
  float acc[kSkinnyMaxTokens / 16][4];
#pragma unroll
  for (int mt = 0; mt < kSkinnyMaxTokens / 16; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
  if (ok && col < ncols) {
    const uint32_t wb = smem_u32(wbuf), xb = smem_u32(s.xs);
    const int mi = lane >> 3, mr = lane & 7;
    for (int ks = 0; ks < s.RR / 16; ++ks) {
      // B: weight rows k = 16 ks .. 16 ks + 15 (lanes 0-15 address them),
      // this warp's 16-byte column chunk, transposed into the (k, n) fragment
      const int kb = ks * 16 + (lane & 15);
      uint32_t b0, b1;
      ldsm_x2_t(wb + kb * 128 + (((col >> 3) ^ (kb & 7)) << 4), b0, b1);
#pragma unroll
      for (int mt = 0; mt < kSkinnyMaxTokens / 16; ++mt) {
        if (mt >= nmt) break;
        // A: tokens 16 mt .. 16 mt + 15 x k 16 ks .. 16 ks + 15
        const int row = mt * 16 + (mi & 1) * 8 + mr, kc = ks * 16 + (mi >> 1) * 8;
        uint32_t a[4];
        ldsm_x4(xb + (row * RRp + kc) * 2, a[0], a[1], a[2], a[3]);
        mma_bf16_16816(acc[mt], a, b0, b1);
      }
    }
  }
  // accumulator fragment: tokens 16 mt + lane / 4 (+ 8), columns col + 2 (lane % 4) (+ 1)
  const int tr = lane >> 2, tc = col + 2 * (lane & 3);
#pragma unroll
  for (int mt = 0; mt < kSkinnyMaxTokens / 16; ++mt) {
    if (mt >= nmt) break;
    *reinterpret_cast<float2*>(part + (mt * 16 + tr) * 64 + tc) = make_float2(acc[mt][0], acc[mt][1]);
    *reinterpret_cast<float2*>(part + (mt * 16 + tr + 8) * 64 + tc) = make_float2(acc[mt][2], acc[mt][3]);
  }
  __syncthreads();
  return ok;
}

// After a cluster barrier: the sum over the cluster's ranks (in rank order)
// of part[i] (part: this CTA's s.part or s.part_r; i = token * 64 + column).
__device__ __forceinline__ float sk_cluster_sum(const float* part, int i) {
  const uint32_t a = smem_u32(part + i);
  float v = 0.f;
#pragma unroll
  for (int r = 0; r < kSkCluster; ++r) v += ld_dsmem_f32(mapa_shared(a, (uint32_t)r));
  return v;
}

// Stage rows [row0, row0 + RR) of x for tokens 0..B-1 into xs (zeros past B
// or past D); 16-byte pieces, four loaded before any is stored.
__device__ __forceinline__ void sk_stage_x(const SkCta& s, const DecodeProjParams& p) {
  const int per = s.RR / 8;  // 16-byte pieces of a row
  const int total = s.cap * per;
  for (int i0 = threadIdx.x; i0 < total; i0 += 4 * kSkinnyThreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kSkinnyThreads;
      const int n = i / per, col = s.row0 + (i % per) * 8;
      v[u] = (i < total && n < p.B && col < p.D) ? *reinterpret_cast<const uint4*>(p.x + (size_t)n * p.D + col)
                                                 : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kSkinnyThreads;
      if (i < total) reinterpret_cast<uint4*>(s.xs)[(i / per) * (per + 1) + i % per] = v[u];
    }
  }
  __syncthreads();
}

// Thread i < kSkPerRank of rank q: the decision of group g for token n = n0 + i from
// the logits in s.logits[i][.]; the slot of expert e among the selections
// (-1: not selected) into s.slot[i]; the e = 0 cluster writes sel, w, margin.
template <int RM>
__device__ __forceinline__ void sk_decide(const SkCta& s, const DecodeProjParams& p, int g, int e, int i, int n) {
  float l[RM];
#pragma unroll
  for (int x = 0; x < RM; ++x) l[x] = s.logits[i * 8 + x];
  int32_t sl[8];
  float wl[8];
  float mg;
  route_decide<RM, false>(l, p.k, true, sl, wl, &mg);
  int slot = -1;
  for (int j = 0; j < p.k; ++j)
    if (sl[j] == e) slot = j;
  s.slot[i] = slot;
  if (e == 0) {
    for (int j = 0; j < p.k; ++j) {
      p.sel[((size_t)n * p.G + g) * p.k + j] = sl[j];
      p.w[((size_t)n * p.G + g) * p.k + j] = wl[j];
    }
    if (p.margin) p.margin[(size_t)n * p.G + g] = mg;
  }
}

// Cluster h: the projection of one 64-column weight slice (see the file
// comment); a routed head's cluster also multiplies the 64-column slice of
// Wr that holds its group's logits and decides.
__global__ void __cluster_dims__(kSkCluster, 1, 1) __launch_bounds__(kSkinnyThreads)
    decode_proj_kernel(const __grid_constant__ DecodeProjParams p) {
  extern __shared__ uint8_t sk_raw[];
  const int GM = p.G * p.M;
  const int blk = blockIdx.x / kSkCluster;
  const int Ha = p.G * p.k + 1;
  const bool routed = blk > 2 * p.G;
  SkCta s = sk_init(sk_raw, p.D, routed, p.B);
  const CUtensorMap* W;
  int col0, g = 0, e = 0;
  if (blk < 2 * p.G) {
    g = blk % p.G;
    W = blk < p.G ? &p.tmWk : &p.tmWv;
    col0 = g * 64;
  } else {
    W = &p.tmWq;
    if (!routed) {
      col0 = GM * 64;
    } else {
      const int h = blk - 2 * p.G - 1;
      g = h / p.M;
      e = h % p.M;
      col0 = h * 64;
    }
  }
  const int rcol = (g * p.M / 64) * 64;  // Wr slice holding group g's logits
  const int roff = g * p.M - rcol;
  // weights depend on no launch; x, and the buffers the previous step's
  // launches read (caches, Q, sel, w), only after the wait
  sk_load(s, s.wbuf, s.bar, W, col0);
  if (routed) sk_load(s, s.wbuf_r, s.bar_r, &p.tmWr, rcol);
  pdl_wait();
  pdl_trigger();
  sk_stage_x(s, p);
  bool ok = sk_product(s, s.wbuf, s.bar, 64, p.B, s.part);
  if (routed) ok = sk_product(s, s.wbuf_r, s.bar_r, roff + p.M, p.B, s.part_r) && ok;
  cluster_sync();  // every rank's partials are ready
  const int n0 = s.rank * kSkPerRank;  // this rank's tokens [n0, n0 + kSkPerRank)
  const int nr = max(0, min(kSkPerRank, p.B - n0));
  if (routed) {
    for (int i = threadIdx.x; i < nr * p.M; i += kSkinnyThreads) {
      const int ti = i / p.M, x = i % p.M;
      s.logits[ti * 8 + x] =
          sk_cluster_sum(s.part_r, (n0 + ti) * 64 + roff + x) + (p.br ? p.br[g * p.M + x] : 0.f);
    }
    __syncthreads();
    if ((int)threadIdx.x < nr && ok) {
      const int i = threadIdx.x;
      switch (p.M) {
        case 1: sk_decide<1>(s, p, g, e, i, n0 + i); break;
        case 2: sk_decide<2>(s, p, g, e, i, n0 + i); break;
        case 4: sk_decide<4>(s, p, g, e, i, n0 + i); break;
        default: sk_decide<8>(s, p, g, e, i, n0 + i); break;
      }
    }
    __syncthreads();
  }
  for (int i = threadIdx.x; ok && i < nr * 64; i += kSkinnyThreads) {
    const int ti = i / 64, c = i % 64, n = n0 + ti;
    const int slot = routed ? s.slot[ti] : 0;
    if (slot < 0) continue;
    const __nv_bfloat16 v = __float2bfloat16_rn(sk_cluster_sum(s.part, n * 64 + c));
    if (blk < 2 * p.G) {
      const int L = p.cache_len[n];
      if (L < 0 || L >= p.T) {
        if (c == 0) flag_bounds_error();
      } else {
        (blk < p.G ? p.Kc : p.Vc)[(((size_t)n * p.T + L) * p.G + g) * 64 + c] = v;
      }
    } else if (!routed) {
      p.Q[((size_t)n * Ha + p.G * p.k) * 64 + c] = v;
    } else {
      p.Q[((size_t)n * Ha + g * p.k + slot) * 64 + c] = v;
    }
  }
  cluster_sync();  // the ranks are done reading the partials
  if (!ok) {  // a wait ran out: let copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

// Cluster j: columns [64 j, 64 j + 64) of y = A Wo for the new tokens; this
// CTA's rows of Wo are A's columns [row0, row0 + RR).
__global__ void __cluster_dims__(kSkCluster, 1, 1) __launch_bounds__(kSkinnyThreads)
    decode_out_kernel(const __grid_constant__ DecodeProjParams p) {
  pdl_trigger();
  extern __shared__ uint8_t sk_raw[];
  const int Gk = p.G * p.k, Ha = Gk + 1;
  const int Ka = (Gk + p.G + 1) * 64;
  SkCta s = sk_init(sk_raw, Ka, false, p.B);
  const int col0 = (blockIdx.x / kSkCluster) * 64;
  sk_load(s, s.wbuf, s.bar, &p.tmWo, col0);  // Wo depends on no launch
  pdl_wait();
  // A's columns of this CTA for every token: 64-wide blocks [concat (G*k) |
  // slot (G) | shared], in 16-byte pieces of 8 columns; a thread loads all of
  // a piece's inputs before storing it
  const int per = s.RR / 8;
  for (int i = threadIdx.x; i < s.cap * per; i += kSkinnyThreads) {
    const int n = i / per, col = s.row0 + (i % per) * 8, blkc = col / 64, d = col % 64;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < p.B && col < Ka) {
      const size_t orow = (size_t)n * Ha;
      if (blkc < Gk || blkc >= Gk + p.G) {
        const int src = blkc < Gk ? blkc : Gk;  // concatenation, or the shared head
        v = *reinterpret_cast<const uint4*>(p.O + (orow + src) * 64 + d);
      } else {
        const int g = blkc - Gk;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < p.k; ++j) {
          const float wj = p.w[((size_t)n * p.G + g) * p.k + j];
          const uint4 o = *reinterpret_cast<const uint4*>(p.O + (orow + g * p.k + j) * 64 + d);
          const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            acc[2 * q] = fmaf(wj, bf16lo_to_f32(ou[q]), acc[2 * q]);
            acc[2 * q + 1] = fmaf(wj, bf16hi_to_f32(ou[q]), acc[2 * q + 1]);
          }
        }
        v = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
      }
    }
    reinterpret_cast<uint4*>(s.xs)[n * (per + 1) + i % per] = v;
  }
  __syncthreads();
  const bool ok = sk_product(s, s.wbuf, s.bar, 64, p.B, s.part);
  cluster_sync();  // every rank's part is ready
  const int n0 = s.rank * kSkPerRank;
  const int nr = max(0, min(kSkPerRank, p.B - n0));
  for (int i = threadIdx.x; ok && i < nr * 64; i += kSkinnyThreads) {
    const int n = n0 + i / 64, c = i % 64;
    p.y[(size_t)n * p.D + col0 + c] = __float2bfloat16_rn(sk_cluster_sum(s.part, n * 64 + c));
  }
  cluster_sync();  // the ranks are done reading part
  if (!ok) {  // a wait ran out: let copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

}  // namespace gqe
