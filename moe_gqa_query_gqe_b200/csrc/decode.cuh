// decode.cuh -- one generation step of the GQE layer against a key/value cache.
//
// Method: the layer of the gist.science summary ("Architecture and routing")
// and the animattoys.com article (section 4) applied to one new token per
// sequence; aiboss88.com wiki on grouped-query attention, inference section
// (a decoder caches the key/value heads and re-reads them at every step, so
// the step is bound by reading the cache). The new token of sequence b sits at
// position L_b = cache_len[b]: its K/V row is appended there and each of its
// query rows (the k selected experts of every group, plus the shared head on
// KV head 0) attends positions 0..L_b.
//
// Routing, the projections and the output projection reuse the prefill
// kernels with the B new tokens seen as one sequence of B tokens. This file
// holds the cache-side kernels:
//   decode_append_kernel : K/V row of the new token -> cache position L_b
//   decode_attn_kernel   : split-K attention. CTA (split s, group g, seq b)
//                          takes keys [s*chunk, min((s+1)*chunk, L_b+1)) for
//                          the R = k (+1 shared in group 0) query rows of the
//                          group: scores in shared memory (log2 domain), the
//                          chunk's max m and sum l per row, and the partial
//                          output sum_s 2^(score - m) V_s. CUDA cores: at
//                          R <= 9 rows per key the tensor cores would idle;
//                          the bound is the cache read (2 * 128 B per key).
//   decode_merge_kernel  : one warp per (sequence, query slot) merges the
//                          chunks: O = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kDecChunk = 1024;    // keys per attention CTA
constexpr int kDecThreads = 128;

struct DecodeParams {
  const __nv_bfloat16* Q;    // [B, Ha, 64]: slot g*k+j routed, slot G*k shared
  const __nv_bfloat16* Kn;   // [B, G, 64] the new tokens' keys
  const __nv_bfloat16* Vn;   // [B, G, 64]
  __nv_bfloat16* Kc;         // [B, T, G, 64] caches (T = capacity)
  __nv_bfloat16* Vc;
  const int32_t* cache_len;  // [B] device
  float* part_ml;            // [B, G, rmax, nsplit] x {m, l}
  float* part_o;             // [B, G, rmax, nsplit, 64]
  __nv_bfloat16* O;          // [B, Ha, 64]
  int B, T, G, k, Ha, rmax, nsplit;
  float scale_log2;          // log2(e) / sqrt(64)
};

// Cache length of sequence b, or -1 (and the bounds flag) if it is outside [0, T).
__device__ __forceinline__ int dec_len(const DecodeParams& p, int b) {
  const int L = p.cache_len[b];
  if (L < 0 || L >= p.T) {
    flag_bounds_error();
    return -1;
  }
  return L;
}

__global__ void __launch_bounds__(256) decode_append_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  const int per = p.G * 64 / 8;  // 16-byte pieces of one K (or V) row
  const int total = p.B * per * 2;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int which = i / (p.B * per);
    const int r = i % (p.B * per);
    const int b = r / per, c = r % per;
    const int L = dec_len(p, b);
    if (L < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>((which ? p.Vn : p.Kn) + (size_t)b * p.G * 64) + c;
    uint4* dst = reinterpret_cast<uint4*>((which ? p.Vc : p.Kc) + ((size_t)b * p.T + L) * p.G * 64) + c;
    *dst = *src;
  }
}

__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float dsm[];
  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = p.k + (g == 0 ? 1 : 0);
  float* q = dsm;                       // [rmax][64], scaled to the log2 domain
  float* sc = q + p.rmax * 64;          // [rmax][kDecChunk]
  float* red = sc + p.rmax * kDecChunk;  // [4][rmax][64] partial outputs / [4][rmax] reductions
  const int L = dec_len(p, b);
  const int nkeys = L + 1;
  const int k0 = s * kDecChunk, k1 = min(k0 + kDecChunk, nkeys);
  const size_t base = ((size_t)(b * p.G + g) * p.rmax) * p.nsplit + s;  // + r * nsplit
  if (L < 0 || k0 >= k1) {
    for (int i = tid; i < p.rmax; i += kDecThreads) {
      p.part_ml[(base + (size_t)i * p.nsplit) * 2] = -INFINITY;
      p.part_ml[(base + (size_t)i * p.nsplit) * 2 + 1] = 0.f;
    }
    return;
  }
  for (int i = tid; i < R * 64; i += kDecThreads) {
    const int r = i / 64, d = i % 64;
    const int slot = r < p.k ? g * p.k + r : p.G * p.k;
    q[i] = __bfloat162float(p.Q[((size_t)b * p.Ha + slot) * 64 + d]) * p.scale_log2;
  }
  __syncthreads();

  // scores: each thread takes two keys per pass (both rows' loads in flight
  // before the math), kDecThreads * 2 keys per pass over the chunk
  float mloc[9];
#pragma unroll
  for (int r = 0; r < 9; ++r) mloc[r] = -INFINITY;
  for (int i0 = k0 + tid; i0 < k1; i0 += 2 * kDecThreads) {
    const int i1 = i0 + kDecThreads;
    uint4 u[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = h ? i1 : i0;
      if (i < k1) {
        const uint4* kp = reinterpret_cast<const uint4*>(p.Kc + (((size_t)b * p.T + i) * p.G + g) * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) u[h][c] = kp[c];
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = h ? i1 : i0;
      if (i >= k1) break;
      float kv[64];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t w4[4] = {u[h][c].x, u[h][c].y, u[h][c].z, u[h][c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kv[c * 8 + 2 * e] = bf16lo_to_f32(w4[e]);
          kv[c * 8 + 2 * e + 1] = bf16hi_to_f32(w4[e]);
        }
      }
#pragma unroll
      for (int r = 0; r < 9; ++r) {
        if (r >= R) break;
        float acc = 0.f;
#pragma unroll
        for (int d = 0; d < 64; ++d) acc = fmaf(q[r * 64 + d], kv[d], acc);
        sc[r * kDecChunk + (i - k0)] = acc;
        mloc[r] = fmaxf(mloc[r], acc);
      }
    }
  }
  // chunk max per row
#pragma unroll
  for (int r = 0; r < 9; ++r) {
    if (r >= R) break;
    float v = mloc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp * p.rmax + r] = v;
  }
  __syncthreads();
  float m[9], l[9];
#pragma unroll
  for (int r = 0; r < 9; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
    if (r < R)
      for (int w = 0; w < 4; ++w) m[r] = fmaxf(m[r], red[w * p.rmax + r]);
  }
  __syncthreads();
  // probabilities (unnormalised) and their sum per row
  float lloc[9];
#pragma unroll
  for (int r = 0; r < 9; ++r) lloc[r] = 0.f;
  for (int i = tid; i < k1 - k0; i += kDecThreads) {
#pragma unroll
    for (int r = 0; r < 9; ++r) {
      if (r >= R) break;
      const float e = exp2f(sc[r * kDecChunk + i] - m[r]);
      sc[r * kDecChunk + i] = e;
      lloc[r] += e;
    }
  }
#pragma unroll
  for (int r = 0; r < 9; ++r) {
    if (r >= R) break;
    float v = lloc[r];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp * p.rmax + r] = v;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 9; ++r)
    if (r < R)
      for (int w = 0; w < 4; ++w) l[r] += red[w * p.rmax + r];
  __syncthreads();
  // P.V: warp w takes keys k0+w, k0+w+4, ... (32 rows per batch); lane owns
  // dims 2*lane, 2*lane+1
  float o0[9], o1[9];
#pragma unroll
  for (int r = 0; r < 9; ++r) o0[r] = o1[r] = 0.f;
  for (int i0 = k0 + warp; i0 < k1; i0 += 4 * 32) {
    uint32_t v2[32];  // 32 V rows per warp in flight
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int i = i0 + 4 * u;
      v2[u] = i < k1 ? reinterpret_cast<const uint32_t*>(p.Vc + (((size_t)b * p.T + i) * p.G + g) * 64)[lane] : 0u;
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int i = i0 + 4 * u;
      if (i >= k1) break;
      const float v0 = bf16lo_to_f32(v2[u]), v1 = bf16hi_to_f32(v2[u]);
#pragma unroll
      for (int r = 0; r < 9; ++r) {
        if (r >= R) break;
        const float pr = sc[r * kDecChunk + (i - k0)];
        o0[r] = fmaf(pr, v0, o0[r]);
        o1[r] = fmaf(pr, v1, o1[r]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < 9; ++r) {
    if (r >= R) break;
    red[(warp * p.rmax + r) * 64 + 2 * lane] = o0[r];
    red[(warp * p.rmax + r) * 64 + 2 * lane + 1] = o1[r];
  }
  __syncthreads();
  for (int i = tid; i < R * 64; i += kDecThreads) {
    const int r = i / 64, d = i % 64;
    float acc = 0.f;
    for (int w = 0; w < 4; ++w) acc += red[(w * p.rmax + r) * 64 + d];
    p.part_o[(base + (size_t)r * p.nsplit) * 64 + d] = acc;
  }
  if (tid < R) {
    float mr = 0.f, lr = 0.f;
#pragma unroll
    for (int r = 0; r < 9; ++r)
      if (r == tid) {
        mr = m[r];
        lr = l[r];
      }
    p.part_ml[(base + (size_t)tid * p.nsplit) * 2] = mr;
    p.part_ml[(base + (size_t)tid * p.nsplit) * 2 + 1] = lr;
  }
}

// One warp per (sequence b, query slot).
__global__ void __launch_bounds__(256) decode_merge_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (wid >= p.B * p.Ha) return;
  const int b = wid / p.Ha, slot = wid % p.Ha;
  const int g = slot < p.G * p.k ? slot / p.k : 0;
  const int r = slot < p.G * p.k ? slot % p.k : p.k;
  const size_t base = ((size_t)(b * p.G + g) * p.rmax + r) * p.nsplit;
  float M = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) M = fmaxf(M, p.part_ml[(base + s) * 2]);
  float acc0 = 0.f, acc1 = 0.f, lsum = 0.f;
  for (int s = 0; s < p.nsplit; ++s) {
    const float ms = p.part_ml[(base + s) * 2];
    if (ms == -INFINITY) continue;
    const float f = exp2f(ms - M);
    lsum += f * p.part_ml[(base + s) * 2 + 1];
    const float2 o = reinterpret_cast<const float2*>(p.part_o + (base + s) * 64)[lane];
    acc0 = fmaf(f, o.x, acc0);
    acc1 = fmaf(f, o.y, acc1);
  }
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  reinterpret_cast<uint32_t*>(p.O + ((size_t)b * p.Ha + slot) * 64)[lane] = pack_bf16x2(acc0 * inv, acc1 * inv);
}

}  // namespace gqe
