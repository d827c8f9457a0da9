// decode_proj.cuh -- the token-side work of one decode step for a few new
// tokens (B <= kSkinnyMaxTokens): routing, the K/V and query projections and
// the output construction with its projection, as skinny products on CUDA
// cores.
//
// Method: the layer of the gist.science summary ("Architecture and routing":
// conditional activation, renormalised weighted sum, dense K/V, output
// construction) and the animattoys.com article (section 4), applied to the
// new token of every sequence; the aiboss88.com wiki on grouped-query
// attention, inference section (the new token's key/value rows are appended
// to the cache).
//
// With a handful of rows a projection is a read of its weights: B x D times
// D x 64 per 64-column block. The tensor-core tiles of the prefill path would
// pad the B rows to 256 and stream each weight through a few SMs; here every
// 64-column weight slice is read by its own CTA, so all slices stream at once.
//   decode_route_kernel: one block: router logits x Wr + br of the B tokens,
//                        their decisions -> sel, w, margin
//   decode_proj_kernel : block 0..G-1   K of group g -> cache row cache_len[b]
//                        block G..2G-1  V of group g -> cache row cache_len[b]
//                        block 2G       the shared head's query
//                        block 2G+1+h   routed head h = g*M + e: the query of
//                                       the tokens that selected it (only)
//                        Its weight slices load while the routing launch runs
//                        (programmatic dependent launch: the wait for it comes
//                        after the loads are issued).
//   decode_out_kernel  : block j: columns [64j, 64j + 64) of y = A Wo, with
//                        A = [concat | per-group slot sum_j w_j O_j | shared]
//                        built from O and w in shared memory (the slot rounded
//                        to bf16, as the combine kernel does).
// Thread t of a 256-thread block owns 8 consecutive columns (t % 8) and the
// rows k = t / 8 (mod 32) of the reduction; the 32 row-partial sums are added
// by shuffles within a warp and through shared memory across warps.
#pragma once

#include "decode.cuh"
#include "route.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kSkinnyMaxTokens = 16;
constexpr int kSkinnyThreads = 256;
constexpr int kSkinnyTB = 8;     // tokens per pass
constexpr int kSkChunk = 256;    // weight rows per TMA chunk (32 KB of a 64-column slice)
constexpr int kSkBufs = 4;       // chunks in flight (a whole 1024-row slice)

struct DecodeProjParams {
  // weights as TMA tensor maps: box 64 columns x kSkChunk rows, 128-byte swizzle
  CUtensorMap tmWq, tmWk, tmWv, tmWr, tmWo;
  const __nv_bfloat16* x;   // [B, D] new tokens
  const __nv_bfloat16* Wq;  // [D, (G*M + 1)*64]
  const __nv_bfloat16* Wk;  // [D, G*64]
  const __nv_bfloat16* Wv;
  const __nv_bfloat16* Wr;  // [D, G*M]
  const float* br;          // [G*M] or null
  const int32_t* cache_len; // [B]
  __nv_bfloat16* Kc;        // [B, T, G, 64]
  __nv_bfloat16* Vc;
  __nv_bfloat16* Q;         // [B, G*k + 1, 64]
  int32_t* sel;             // [B, G, k]
  float* w;                 // [B, G, k]
  float* margin;            // [B, G] or null
  // output side
  const __nv_bfloat16* O;   // [B, G*k + 1, 64]
  const __nv_bfloat16* Wo;  // [(G*k + G + 1)*64, D]
  __nv_bfloat16* y;         // [B, D]
  int B, T, D, G, M, k;
};

// Shared memory (from a 1024-aligned base): kSkBufs weight chunk buffers
// [kSkBufs][kSkChunk][128 B], their mbarriers and the abort flag (1 KB), then the
// tokens' rows xs [TB][K] (bf16), per-warp partials red [8][TB][64] (float),
// and for decode_route_kernel the logits [B][G*M] (float), for
// decode_proj_kernel the token list of a routed head [kSkinnyMaxTokens + 1]
// (int; the last entry holds its length).
constexpr int kSkWbuf = kSkBufs * kSkChunk * 128;
constexpr int kSkHead = kSkWbuf + 1024;
__host__ __device__ inline int skinny_route_smem(int B, int D, int GM) {
  return 1024 + kSkHead + kSkinnyTB * D * 2 + 8 * kSkinnyTB * 64 * 4 + B * GM * 4;
}
__host__ __device__ inline int skinny_proj_smem(int D) {
  return 1024 + kSkHead + kSkinnyTB * D * 2 + 8 * kSkinnyTB * 64 * 4 + (kSkinnyMaxTokens + 1) * 4;
}
__host__ __device__ inline int skinny_out_smem(int D_in) {
  return 1024 + kSkHead + kSkinnyTB * D_in * 2 + 8 * kSkinnyTB * 64 * 4;
}

// The weight-chunk pipeline of a block: kSkBufs buffers, one mbarrier each,
// and how many times each buffer has been filled (its barrier's phase).
struct SkPipe {
  uint8_t* wbuf;
  uint64_t* bar;       // [kSkBufs]
  volatile int* abort_flag;
  uint32_t uses[kSkBufs];
};

// acc[n][c] = sum over rows k < K of xs[n][k] * W[k][col0 + c8 + c], the
// weight slice W[:, col0 .. col0+63] streamed by TMA in chunks of kSkChunk
// rows through the kSkBufs buffers of `pp` (up to kSkBufs chunks in flight,
// the whole slice when K <= kSkBufs * kSkChunk). Thread t reads rows kr, kr + 32, ... of a chunk (kr = t / 8), 16
// bytes each at column c8 = 8 (t % 8); columns at or past ncols are zeros and
// skipped. The 32 row-partials of each (n, c) are summed: lanes 0..7 of every
// warp leave the warp's sums in red[warp]. Returns false if a wait timed out.
// Thread 0 issues the TMA loads of chunk ch of the slice into its buffer.
__device__ __forceinline__ void skinny_issue(const CUtensorMap* tm, int col0, int ch, SkPipe& pp) {
  const int bsel = ch % kSkBufs;
  mbar_arrive_expect_tx(&pp.bar[bsel], kSkChunk * 128);
  tma_load_2d(pp.wbuf + bsel * kSkChunk * 128, tm, &pp.bar[bsel], col0, ch * kSkChunk);
}
// The first kSkBufs chunks (thread 0), so they load before the data they
// multiply is ready (skinny_block then takes preissued = true).
__device__ __forceinline__ void skinny_prefetch(const CUtensorMap* tm, int col0, int K, SkPipe& pp) {
  const int nch = (K + kSkChunk - 1) / kSkChunk;
  if (threadIdx.x == 0)
    for (int ch = 0; ch < kSkBufs && ch < nch; ++ch) skinny_issue(tm, col0, ch, pp);
}

__device__ __forceinline__ bool skinny_block(const CUtensorMap* tm, int col0, int ncols, const __nv_bfloat16* xs,
                                             int K, float* red, SkPipe& pp, bool preissued = false) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c8 = (t & 7) * 8, kr = t >> 3;
  const int nch = (K + kSkChunk - 1) / kSkChunk;
  auto issue = [&](int ch) { skinny_issue(tm, col0, ch, pp); };
  if (!preissued) skinny_prefetch(tm, col0, K, pp);
  float acc[kSkinnyTB][8];
#pragma unroll
  for (int n = 0; n < kSkinnyTB; ++n)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[n][c] = 0.f;
  bool ok = true;
  for (int ch = 0; ch < nch; ++ch) {
    const int bsel = ch % kSkBufs;
    ok = mbar_wait(&pp.bar[bsel], pp.uses[bsel] & 1, pp.abort_flag);
    ++pp.uses[bsel];
    if (!__syncthreads_and(ok)) return false;
    if (c8 < ncols) {
      const uint32_t base = smem_u32(pp.wbuf + bsel * kSkChunk * 128);
#pragma unroll
      for (int i = 0; i < kSkChunk / 32; ++i) {
        const int r = kr + 32 * i, k = ch * kSkChunk + r;
        if (k >= K) break;
        uint32_t w4[4];
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                     : "r"(base + r * 128 + ((((c8 >> 3) ^ (r & 7))) << 4)));
        float wf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          wf[2 * e] = bf16lo_to_f32(w4[e]);
          wf[2 * e + 1] = bf16hi_to_f32(w4[e]);
        }
#pragma unroll
        for (int n = 0; n < kSkinnyTB; ++n) {
          const float xv = __bfloat162float(xs[n * K + k]);
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[n][c] = fmaf(xv, wf[c], acc[n][c]);
        }
      }
    }
    __syncthreads();  // every thread is done with this buffer
    if (t == 0 && ch + kSkBufs < nch) issue(ch + kSkBufs);
  }
#pragma unroll
  for (int n = 0; n < kSkinnyTB; ++n)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      acc[n][c] += __shfl_xor_sync(0xffffffffu, acc[n][c], 8);
      acc[n][c] += __shfl_xor_sync(0xffffffffu, acc[n][c], 16);
    }
  if (lane < 8)
#pragma unroll
    for (int n = 0; n < kSkinnyTB; ++n)
#pragma unroll
      for (int c = 0; c < 8; ++c) red[(warp * kSkinnyTB + n) * 64 + c8 + c] = acc[n][c];
  __syncthreads();
  return true;
}

// The pipeline's buffers and barriers at the start of the block's shared
// memory (aligned to 1024 bytes, as the 128-byte swizzle of the TMA needs).
__device__ __forceinline__ SkPipe skinny_pipe_init(uint8_t* smem) {
  SkPipe pp;
  pp.wbuf = smem;
  pp.bar = reinterpret_cast<uint64_t*>(smem + kSkWbuf);
  pp.abort_flag = reinterpret_cast<volatile int*>(smem + kSkWbuf + 8 * kSkBufs);
  for (int i = 0; i < kSkBufs; ++i) pp.uses[i] = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSkBufs; ++i) mbar_init(&pp.bar[i], 1);
    *pp.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  return pp;
}

// Sum of the 8 warps' partials for token n, column c (after skinny_block).
__device__ __forceinline__ float skinny_sum(const float* red, int n, int c) {
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red[(w * kSkinnyTB + n) * 64 + c];
  return s;
}

// Stage rows of x (tokens tok[0..nt), zeros past nt) into xs [TB][D]: four
// 16-byte pieces per thread are loaded before any is stored, so the loads are
// in flight together.
__device__ __forceinline__ void skinny_stage_x(const DecodeProjParams& p, const int* tok, int nt, __nv_bfloat16* xs) {
  const int per = p.D / 8;  // 16-byte pieces per row
  const int total = kSkinnyTB * per;
  for (int i0 = threadIdx.x; i0 < total; i0 += 4 * kSkinnyThreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kSkinnyThreads;
      const int n = i / per, c = i % per;
      v[u] = (i < total && n < nt) ? reinterpret_cast<const uint4*>(p.x + (size_t)tok[n] * p.D)[c]
                                   : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kSkinnyThreads;
      if (i < total) reinterpret_cast<uint4*>(xs)[i] = v[u];
    }
  }
  __syncthreads();
}

// Router logits x Wr + br of the B new tokens, then the decisions, written to
// sel, w and margin.
template <int RM>
__device__ bool skinny_route(const DecodeProjParams& p, __nv_bfloat16* xs, float* logits, float* red, SkPipe& pp) {
  const int GM = p.G * RM;
  bool pre = true;  // the first slice's chunks were issued by the caller
  for (int n0 = 0; n0 < p.B; n0 += kSkinnyTB) {
    int tok[kSkinnyTB];
#pragma unroll
    for (int n = 0; n < kSkinnyTB; ++n) tok[n] = n0 + n;
    skinny_stage_x(p, tok, min(kSkinnyTB, p.B - n0), xs);
    for (int c0 = 0; c0 < GM; c0 += 64) {
      if (!skinny_block(&p.tmWr, c0, GM - c0, xs, p.D, red, pp, pre)) return false;
      pre = false;
      for (int i = threadIdx.x; i < kSkinnyTB * 64; i += kSkinnyThreads) {
        const int n = i / 64, c = i % 64;
        if (n0 + n < p.B && c0 + c < GM)
          logits[(n0 + n) * GM + c0 + c] = skinny_sum(red, n, c) + (p.br ? p.br[c0 + c] : 0.f);
      }
      __syncthreads();
    }
  }
  // decisions: one thread per (token, group)
  for (int i = threadIdx.x; i < p.B * p.G; i += kSkinnyThreads) {
    const int n = i / p.G, g = i % p.G;
    float l[RM];
#pragma unroll
    for (int e = 0; e < RM; ++e) l[e] = logits[n * GM + g * RM + e];
    int32_t sl[8];
    float wl[8];
    float mg;
    route_decide<RM, false>(l, p.k, true, sl, wl, &mg);
    for (int j = 0; j < p.k; ++j) {
      p.sel[((size_t)n * p.G + g) * p.k + j] = sl[j];
      p.w[((size_t)n * p.G + g) * p.k + j] = wl[j];
    }
    if (p.margin) p.margin[(size_t)n * p.G + g] = mg;
  }
  __syncthreads();
  return true;
}

// One CTA: the routing decisions of the B new tokens (sel, w, margin).
__global__ void __launch_bounds__(kSkinnyThreads) decode_route_kernel(const __grid_constant__ DecodeProjParams p) {
  extern __shared__ uint8_t sk_raw[];
  uint8_t* sk = sk_raw + ((1024u - (smem_u32(sk_raw) & 1023u)) & 1023u);
  SkPipe pp = skinny_pipe_init(sk);
  skinny_prefetch(&p.tmWr, 0, p.D, pp);  // Wr depends on no launch
  // the previous step's output kernel reads w: wait before writing it (and
  // before letting the projection launch in)
  pdl_wait();
  pdl_trigger();
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sk + kSkHead);
  float* red = reinterpret_cast<float*>(sk + kSkHead + kSkinnyTB * p.D * 2);
  float* logits = red + 8 * kSkinnyTB * 64;
  bool ok = true;
  switch (p.M) {
    case 1: ok = skinny_route<1>(p, xs, logits, red, pp); break;
    case 2: ok = skinny_route<2>(p, xs, logits, red, pp); break;
    case 4: ok = skinny_route<4>(p, xs, logits, red, pp); break;
    default: ok = skinny_route<8>(p, xs, logits, red, pp); break;
  }
  if (!ok) {  // a wait ran out: let copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

// The projections of the new tokens. The weight slice starts loading before
// the wait for the routing launch (weights depend on no launch); routed
// blocks read sel after the wait.
__global__ void __launch_bounds__(kSkinnyThreads) decode_proj_kernel(const __grid_constant__ DecodeProjParams p) {
  pdl_trigger();
  extern __shared__ uint8_t sk_raw[];
  // aligned by pointer arithmetic on the shared array itself, so the
  // compiler keeps it in the shared space (its stores cannot alias the
  // global loads, which may then be issued ahead of them)
  uint8_t* sk = sk_raw + ((1024u - (smem_u32(sk_raw) & 1023u)) & 1023u);
  SkPipe pp = skinny_pipe_init(sk);
  const int GM = p.G * p.M;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sk + kSkHead);
  float* red = reinterpret_cast<float*>(sk + kSkHead + kSkinnyTB * p.D * 2);
  int* tlist = reinterpret_cast<int*>(red + 8 * kSkinnyTB * 64);
  const int blk = blockIdx.x;
  const int Ha = p.G * p.k + 1;
  const bool routed = blk > 2 * p.G;
  // this block's weight slice
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
  skinny_prefetch(W, col0, p.D, pp);
  // The K/V and shared-query blocks compute their first pass before the
  // wait (x and the weights depend on no launch) and wait before writing;
  // the routed blocks need sel first.
  bool waited = false;
  int ntok;
  if (!routed) {
    ntok = p.B;
    for (int i = threadIdx.x; i < p.B; i += kSkinnyThreads) tlist[i] = i;
  } else {
    pdl_wait();
    waited = true;
  }
  if (routed && threadIdx.x == 0) {
    // the tokens that selected expert e of group g, in order
    int c = 0;
    for (int n = 0; n < p.B; ++n)
      for (int j = 0; j < p.k; ++j)
        if (p.sel[((size_t)n * p.G + g) * p.k + j] == e) tlist[c++] = n;
    tlist[kSkinnyMaxTokens] = c;
  }
  __syncthreads();
  if (routed) ntok = tlist[kSkinnyMaxTokens];
  bool ok = true;
  bool pre = true;  // the first chunks were issued above
  for (int n0 = 0; ok && n0 < ntok; n0 += kSkinnyTB) {
    const int nt = min(kSkinnyTB, ntok - n0);
    skinny_stage_x(p, tlist + n0, nt, xs);
    if (!(ok = skinny_block(W, col0, 64, xs, p.D, red, pp, pre))) break;
    pre = false;
    if (!waited) {
      pdl_wait();  // earlier launches are done with the rows written below
      waited = true;
    }
    for (int i = threadIdx.x; i < nt * 64; i += kSkinnyThreads) {
      const int n = i / 64, c = i % 64;
      const int tok = tlist[n0 + n];
      const __nv_bfloat16 v = __float2bfloat16_rn(skinny_sum(red, n, c));
      if (blk < 2 * p.G) {
        const int L = p.cache_len[tok];
        if (L < 0 || L >= p.T) {
          if (c == 0) flag_bounds_error();
          continue;
        }
        (blk < p.G ? p.Kc : p.Vc)[(((size_t)tok * p.T + L) * p.G + g) * 64 + c] = v;
      } else if (!routed) {
        p.Q[((size_t)tok * Ha + p.G * p.k) * 64 + c] = v;
      } else {
        // slot of expert e among the token's selections (ascending experts)
        int j = 0;
        for (int jj = 0; jj < p.k; ++jj)
          if (p.sel[((size_t)tok * p.G + g) * p.k + jj] == e) j = jj;
        p.Q[((size_t)tok * Ha + g * p.k + j) * 64 + c] = v;
      }
    }
    __syncthreads();
  }
  pdl_wait();  // on every path, so this grid completes after the ones it depends on
  if (ntok == 0) {
    // nothing consumed the chunks issued before the wait: let them land
    for (int ch = 0; ch < kSkBufs && ch * kSkChunk < p.D; ++ch)
      ok = ok && mbar_wait(&pp.bar[ch], 0, pp.abort_flag);
  }
  if (!ok) {  // a wait ran out: let copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

// y = A Wo for the new tokens; A from O and w (see the file comment).
__global__ void __launch_bounds__(kSkinnyThreads) decode_out_kernel(const __grid_constant__ DecodeProjParams p) {
  pdl_trigger();
  extern __shared__ uint8_t sk_raw[];
  // aligned by pointer arithmetic on the shared array itself, so the
  // compiler keeps it in the shared space (its stores cannot alias the
  // global loads, which may then be issued ahead of them)
  uint8_t* sk = sk_raw + ((1024u - (smem_u32(sk_raw) & 1023u)) & 1023u);
  SkPipe pp = skinny_pipe_init(sk);
  const int Gk = p.G * p.k, Ha = Gk + 1;
  const int Ka = (Gk + p.G + 1) * 64;
  __nv_bfloat16* As = reinterpret_cast<__nv_bfloat16*>(sk + kSkHead);
  float* red = reinterpret_cast<float*>(sk + kSkHead + kSkinnyTB * Ka * 2);
  const int col0 = blockIdx.x * 64;
  skinny_prefetch(&p.tmWo, col0, Ka, pp);  // Wo does not depend on the earlier launches
  pdl_wait();
  bool ok = true;
  bool pre = true;
  for (int n0 = 0; ok && n0 < p.B; n0 += kSkinnyTB) {
    const int nt = min(kSkinnyTB, p.B - n0);
    // A rows: 64-wide blocks [concat (G*k) | slot (G) | shared], built in
    // 16-byte pieces of 8 columns; a thread loads all of a piece's inputs
    // before storing it (loads of consecutive pieces overlap)
    const int per = Ka / 8;
    for (int i = threadIdx.x; i < kSkinnyTB * per; i += kSkinnyThreads) {
      const int n = i / per, col = (i % per) * 8, blkc = col / 64, d = col % 64;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (n < nt) {
        const size_t orow = (size_t)(n0 + n) * Ha;
        if (blkc < Gk || blkc >= Gk + p.G) {
          const int src = blkc < Gk ? blkc : Gk;  // concatenation, or the shared head
          v = *reinterpret_cast<const uint4*>(p.O + (orow + src) * 64 + d);
        } else {
          const int g = blkc - Gk;
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int j = 0; j < p.k; ++j) {
            const float wj = p.w[((size_t)(n0 + n) * p.G + g) * p.k + j];
            const uint4 o = *reinterpret_cast<const uint4*>(p.O + (orow + g * p.k + j) * 64 + d);
            const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[2 * e] = fmaf(wj, bf16lo_to_f32(ou[e]), acc[2 * e]);
              acc[2 * e + 1] = fmaf(wj, bf16hi_to_f32(ou[e]), acc[2 * e + 1]);
            }
          }
          v = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                         pack_bf16x2(acc[6], acc[7]));
        }
      }
      reinterpret_cast<uint4*>(As)[i] = v;
    }
    __syncthreads();
    if (!(ok = skinny_block(&p.tmWo, col0, 64, As, Ka, red, pp, pre))) break;
    pre = false;
    for (int i = threadIdx.x; i < nt * 64; i += kSkinnyThreads) {
      const int n = i / 64, c = i % 64;
      p.y[(size_t)(n0 + n) * p.D + col0 + c] = __float2bfloat16_rn(skinny_sum(red, n, c));
    }
    __syncthreads();
  }
  if (!ok) {  // a wait ran out: let copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

}  // namespace gqe
