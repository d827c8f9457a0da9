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
//   decode_attn_kernel   : split-K attention. CTA (split s, seq b) takes
//                          keys [s*chunk, min((s+1)*chunk, L_b+1)) of all
//                          groups (one contiguous range of the cache) for
//                          every query row: scores in shared memory (log2
//                          domain), the chunk's max m and sum l per row, and
//                          the partial output sum_s 2^(score - m) V_s. CUDA
//                          cores: at <= 9 rows per key the tensor cores would
//                          idle; the bound is the cache read (2 * 128 B per
//                          key and group).
//   decode_merge_kernel  : one warp per (sequence, query slot) merges the
//                          chunks: O = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kDecChunk = 256;    // keys per attention CTA
constexpr int kDecThreads = 256;  // 8 warps
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecUnroll = 8;     // key quads whose loads each lane keeps in flight

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

// Shared memory of decode_attn_kernel, in floats: queries q [Ha][64] (log2
// domain), scores / probabilities sc [Ha][kDecChunk], chunk max and sum
// ml [Ha][2], per-warp partial outputs red [kDecWarps][rmax][64].
__host__ __device__ inline int dec_smem_floats(int Ha, int rmax) {
  return Ha * 64 + Ha * kDecChunk + Ha * 2 + kDecWarps * rmax * 64;
}

// Query slot of row j of group g: the group's k selected experts, then (group
// 0 only) the shared head.
__device__ __forceinline__ int dec_slot(const DecodeParams& p, int g, int j) {
  return j < p.k ? g * p.k + j : p.G * p.k;
}

// CTA (split s, sequence b): keys [s*kDecChunk, min((s+1)*kDecChunk, L_b+1))
// of ALL groups, so the CTA streams one contiguous range of the cache
// ([key][group][64] rows). Warp w takes groups g = w % gs + gs*t (gs =
// min(G, 8)) and, when G < 8, every (8/G)-th quad of keys. A quad is 4 keys;
// lane l reads 16 bytes (dims 8c..8c+7, c = l % 8) of key l / 8 of the quad,
// so one warp load moves four whole 128-byte rows. KR bounds the rows of a
// group (k, plus the shared head in group 0).
template <int KR>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float dsm[];
  const int s = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane & 7, kq = lane >> 3;  // 16-byte piece of a row, key within the quad
  float* q = dsm;
  float* sc = q + p.Ha * 64;
  float* ml = sc + p.Ha * kDecChunk;
  float* red = ml + p.Ha * 2;
  const int L = dec_len(p, b);
  const int k0 = s * kDecChunk, k1 = min(k0 + kDecChunk, L + 1);
  if (L < 0 || k0 >= k1) {
    for (int i = tid; i < p.G * p.rmax; i += kDecThreads) {
      const size_t at = ((size_t)(b * p.G) * p.rmax + i) * p.nsplit + s;
      p.part_ml[at * 2] = -INFINITY;
      p.part_ml[at * 2 + 1] = 0.f;
    }
    return;
  }
  const int n = k1 - k0, nq = (n + 3) >> 2;
  const int gs = min(p.G, kDecWarps), wpg = kDecWarps / gs;  // warps per group
  for (int i = tid; i < p.Ha * 64; i += kDecThreads)
    q[i] = __bfloat162float(p.Q[(size_t)b * p.Ha * 64 + i]) * p.scale_log2;
  __syncthreads();

  // ---- scores: sc[slot][key] = q[slot] . K[key, group of slot] ------------------
  for (int g = warp % gs; g < p.G; g += gs) {
    const int R = p.k + (g == 0 ? 1 : 0);
    float qr[KR][8];
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) qr[j][e] = j < R ? q[dec_slot(p, g, j) * 64 + 8 * c + e] : 0.f;
    for (int qa = warp / gs; qa < nq; qa += wpg * kDecUnroll) {
      uint4 u[kDecUnroll];
#pragma unroll
      for (int t = 0; t < kDecUnroll; ++t) {
        const int i = k0 + 4 * (qa + t * wpg) + kq;
        u[t] = i < k1 ? reinterpret_cast<const uint4*>(p.Kc + (((size_t)b * p.T + i) * p.G + g) * 64)[c]
                      : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int t = 0; t < kDecUnroll; ++t) {
        const int key = 4 * (qa + t * wpg) + kq;  // within the chunk
        const uint32_t w4[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kf[2 * e] = bf16lo_to_f32(w4[e]);
          kf[2 * e + 1] = bf16hi_to_f32(w4[e]);
        }
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          if (j >= R) break;
          float part = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) part = fmaf(qr[j][e], kf[e], part);
          part += __shfl_xor_sync(0xffffffffu, part, 1);
          part += __shfl_xor_sync(0xffffffffu, part, 2);
          part += __shfl_xor_sync(0xffffffffu, part, 4);
          if (c == 0 && key < n) sc[dec_slot(p, g, j) * kDecChunk + key] = part;
        }
      }
    }
  }
  __syncthreads();

  // ---- per row: chunk max, 2^(score - max), their sum ---------------------------
  for (int r = warp; r < p.Ha; r += kDecWarps) {
    float* row = sc + r * kDecChunk;
    float m = -INFINITY;
    for (int i = lane; i < n; i += 32) m = fmaxf(m, row[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float e = exp2f(row[i] - m);
      row[i] = e;
      l += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      ml[r * 2] = m;
      ml[r * 2 + 1] = l;
    }
  }
  __syncthreads();

  // ---- P.V: partial output of every row over this chunk -------------------------
  for (int g = warp % gs; g < p.G; g += gs) {
    const int R = p.k + (g == 0 ? 1 : 0);
    float acc[KR][8];
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    for (int qa = warp / gs; qa < nq; qa += wpg * kDecUnroll) {
      uint4 u[kDecUnroll];
#pragma unroll
      for (int t = 0; t < kDecUnroll; ++t) {
        const int i = k0 + 4 * (qa + t * wpg) + kq;
        u[t] = i < k1 ? reinterpret_cast<const uint4*>(p.Vc + (((size_t)b * p.T + i) * p.G + g) * 64)[c]
                      : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int t = 0; t < kDecUnroll; ++t) {
        const int key = 4 * (qa + t * wpg) + kq;
        const uint32_t w4[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
        float vf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          vf[2 * e] = bf16lo_to_f32(w4[e]);
          vf[2 * e + 1] = bf16hi_to_f32(w4[e]);
        }
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          if (j >= R) break;
          const float pr = key < n ? sc[dec_slot(p, g, j) * kDecChunk + key] : 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j][e] = fmaf(pr, vf[e], acc[j][e]);
        }
      }
    }
    // sum over the four keys of a quad (lanes c, c+8, c+16, c+24)
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[j][e] += __shfl_xor_sync(0xffffffffu, acc[j][e], 8);
        acc[j][e] += __shfl_xor_sync(0xffffffffu, acc[j][e], 16);
      }
    if (kq == 0) {
#pragma unroll
      for (int j = 0; j < KR; ++j) {
        if (j >= R) break;
        if (wpg == 1) {
          float* dst = p.part_o + (((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s) * 64 + 8 * c;
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = acc[j][e];
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) red[(warp * p.rmax + j) * 64 + 8 * c + e] = acc[j][e];
        }
      }
    }
  }
  if (wpg > 1) {
    // groups shared by several warps (G < 8): warps g, g + G, ... hold partial sums
    __syncthreads();
    for (int i = tid; i < p.G * p.rmax * 64; i += kDecThreads) {
      const int g = i / (p.rmax * 64), j = (i / 64) % p.rmax, d = i % 64;
      if (j >= p.k + (g == 0 ? 1 : 0)) continue;
      float a = 0.f;
      for (int t = 0; t < wpg; ++t) a += red[((g + t * gs) * p.rmax + j) * 64 + d];
      p.part_o[(((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s) * 64 + d] = a;
    }
  }
  for (int i = tid; i < p.G * p.rmax; i += kDecThreads) {
    const int g = i / p.rmax, j = i % p.rmax;
    const size_t at = ((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s;
    const bool used = j < p.k + (g == 0 ? 1 : 0);
    p.part_ml[at * 2] = used ? ml[dec_slot(p, g, j) * 2] : -INFINITY;
    p.part_ml[at * 2 + 1] = used ? ml[dec_slot(p, g, j) * 2 + 1] : 0.f;
  }
}

// ---------------------------------------------------------------------------
// decode_attn_ring_kernel: the same split-K attention, with the chunk's cache
// rows brought in by bulk copies through a ring of kDecRingStages shared-memory
// stages of kDecStageBytes (a stage is SK whole keys of all groups, one
// contiguous range of the cache). The stage sequence is the chunk's K stages
// and then its V stages, so the first V stages load while the last scores are
// computed; each CTA keeps up to kDecRingStages stages in flight, and the
// loads cost no registers. Scores, softmax and P.V read the staged rows.
// ---------------------------------------------------------------------------
constexpr int kDecRingStages = 3;
constexpr int kDecStageBytes = 32768;

// Keys per stage for G groups (a power of two, at most the chunk).
__host__ __device__ inline int dec_stage_keys(int G) {
  int sk = kDecStageBytes / (G * 128);
  int p2 = 1;
  while (p2 * 2 <= sk) p2 *= 2;
  return p2 < kDecChunk ? p2 : kDecChunk;
}
// Shared memory: ring (1024-aligned), barriers + abort flag, then the floats
// of dec_smem_floats.
__host__ __device__ inline int dec_ring_smem(int Ha, int rmax) {
  return 1024 + kDecRingStages * kDecStageBytes + 256 + dec_smem_floats(Ha, rmax) * 4;
}

template <int KR>
__global__ void __launch_bounds__(kDecThreads) decode_attn_ring_kernel(const DecodeParams p) {
  pdl_trigger();
  extern __shared__ uint8_t dr_raw[];
  uint8_t* ring = dr_raw + ((1024u - (smem_u32(dr_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kDecRingStages * kDecStageBytes);  // [kDecRingStages]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kDecRingStages);
  float* q = reinterpret_cast<float*>(ring + kDecRingStages * kDecStageBytes + 256);
  float* sc = q + p.Ha * 64;
  float* ml = sc + p.Ha * kDecChunk;
  float* red = ml + p.Ha * 2;
  const int s = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane & 7, kq = lane >> 3;  // 16-byte piece of a row, key within the quad
  // cache_len and the cache rows before the new token's depend on no launch
  // of this step: a chunk without row L starts loading before the wait for
  // the projection launch (which writes row L and the queries)
  const int L = dec_len(p, b);
  const int k0 = s * kDecChunk, k1 = min(k0 + kDecChunk, L + 1);
  if (L < 0 || k0 >= k1) {
    pdl_wait();
    for (int i = tid; i < p.G * p.rmax; i += kDecThreads) {
      const size_t at = ((size_t)(b * p.G) * p.rmax + i) * p.nsplit + s;
      p.part_ml[at * 2] = -INFINITY;
      p.part_ml[at * 2 + 1] = 0.f;
    }
    return;
  }
  const int n = k1 - k0;
  const int SK = dec_stage_keys(p.G);
  const int nst = (n + SK - 1) / SK;  // stages per pass (K, then V)
  const size_t row_bytes = (size_t)p.G * 128;
  const bool has_new = k1 == L + 1;  // the chunk holds row L
  // stage i: pass i / nst (K or V), keys [k0 + (i % nst) * SK, +SK) clipped
  auto issue = [&](int i) {
    const int st = i % nst, key0 = k0 + st * SK, nk = min(SK, k1 - key0);
    const __nv_bfloat16* src = (i < nst ? p.Kc : p.Vc) + ((size_t)b * p.T + key0) * p.G * 64;
    uint64_t* bar = &full[i % kDecRingStages];
    mbar_arrive_expect_tx(bar, (uint32_t)(nk * row_bytes));
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(ring + (i % kDecRingStages) * kDecStageBytes)),
                 "l"(src), "r"((uint32_t)(nk * row_bytes)), "r"(smem_u32(bar))
                 : "memory");
  };
  if (tid == 0) {
    for (int i = 0; i < kDecRingStages; ++i) mbar_init(&full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (!has_new)
      for (int i = 0; i < kDecRingStages && i < 2 * nst; ++i) issue(i);
  }
  pdl_wait();
  if (tid == 0 && has_new)
    for (int i = 0; i < kDecRingStages && i < 2 * nst; ++i) issue(i);
  for (int i = tid; i < p.Ha * 64; i += kDecThreads)
    q[i] = __bfloat162float(p.Q[(size_t)b * p.Ha * 64 + i]) * p.scale_log2;
  __syncthreads();
  const int gs = min(p.G, kDecWarps), wpg = kDecWarps / gs;  // warps per group
  bool ok = true;
  uint32_t uses[kDecRingStages] = {};
  // waits for stage i, returns its buffer (all threads; false if a wait ran out)
  auto acquire = [&](int i, const uint8_t*& buf) -> bool {
    const int r = i % kDecRingStages;
    bool w = mbar_wait(&full[r], uses[r] & 1, abort_flag);
    ++uses[r];
    buf = ring + r * kDecStageBytes;
    return __syncthreads_and(w);
  };
  auto release = [&](int i) {
    __syncthreads();  // every thread is done with stage i's buffer
    if (tid == 0 && i + kDecRingStages < 2 * nst) issue(i + kDecRingStages);
  };

  // ---- scores: sc[slot][key] = q[slot] . K[key, group of slot] ------------------
  for (int st = 0; ok && st < nst; ++st) {
    const uint8_t* buf;
    if (!(ok = acquire(st, buf))) break;
    const int key0 = st * SK, nk = min(SK, n - key0);  // within the chunk
    for (int g = warp % gs; g < p.G; g += gs) {
      const int R = p.k + (g == 0 ? 1 : 0);
      float qr[KR][8];
#pragma unroll
      for (int j = 0; j < KR; ++j)
#pragma unroll
        for (int e = 0; e < 8; ++e) qr[j][e] = j < R ? q[dec_slot(p, g, j) * 64 + 8 * c + e] : 0.f;
      for (int qa = warp / gs; 4 * qa < nk; qa += wpg) {
        const int kl = 4 * qa + kq;  // key within the stage
        const uint4 u = kl < nk ? reinterpret_cast<const uint4*>(buf + ((size_t)kl * p.G + g) * 128)[c]
                                : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        float kf[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kf[2 * e] = bf16lo_to_f32(w4[e]);
          kf[2 * e + 1] = bf16hi_to_f32(w4[e]);
        }
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          if (j >= R) break;
          float part = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) part = fmaf(qr[j][e], kf[e], part);
          part += __shfl_xor_sync(0xffffffffu, part, 1);
          part += __shfl_xor_sync(0xffffffffu, part, 2);
          part += __shfl_xor_sync(0xffffffffu, part, 4);
          if (c == 0 && kl < nk) sc[dec_slot(p, g, j) * kDecChunk + key0 + kl] = part;
        }
      }
    }
    release(st);
  }

  // ---- per row: chunk max, 2^(score - max), their sum ---------------------------
  if (ok) {
    for (int r = warp; r < p.Ha; r += kDecWarps) {
      float* row = sc + r * kDecChunk;
      float m = -INFINITY;
      for (int i = lane; i < n; i += 32) m = fmaxf(m, row[i]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
      for (int i = lane; i < n; i += 32) {
        const float e = exp2f(row[i] - m);
        row[i] = e;
        l += e;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        ml[r * 2] = m;
        ml[r * 2 + 1] = l;
      }
    }
    __syncthreads();
  }

  // ---- P.V: partial output of every row over this chunk -------------------------
  // every warp keeps its groups' accumulators across the V stages
  float acc[2][KR][8];  // a warp serves at most two groups (G <= 16 here; more groups loop below)
  const int gpw = (p.G + gs - 1) / gs;  // groups per warp
  const bool acc_fits = gpw <= 2;
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[a][j][e] = 0.f;
  for (int st = 0; ok && st < nst; ++st) {
    const uint8_t* buf;
    if (!(ok = acquire(nst + st, buf))) break;
    const int key0 = st * SK, nk = min(SK, n - key0);
    if (acc_fits) {
#pragma unroll
      for (int a = 0; a < 2; ++a) {
        const int g = warp % gs + a * gs;
        if (g >= p.G) break;
        const int R = p.k + (g == 0 ? 1 : 0);
        for (int qa = warp / gs; 4 * qa < nk; qa += wpg) {
          const int kl = 4 * qa + kq;
          const uint4 u = kl < nk ? reinterpret_cast<const uint4*>(buf + ((size_t)kl * p.G + g) * 128)[c]
                                  : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
          float vf[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            vf[2 * e] = bf16lo_to_f32(w4[e]);
            vf[2 * e + 1] = bf16hi_to_f32(w4[e]);
          }
#pragma unroll
          for (int j = 0; j < KR; ++j) {
            if (j >= R) break;
            const float pr = kl < nk ? sc[dec_slot(p, g, j) * kDecChunk + key0 + kl] : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[a][j][e] = fmaf(pr, vf[e], acc[a][j][e]);
          }
        }
      }
    }
    release(nst + st);
  }
  if (!acc_fits && ok) flag_bounds_error();  // the host never launches this case
  // sum over the four keys of a quad (lanes c, c+8, c+16, c+24), then over the
  // warps sharing a group, into part_o
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < KR; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc[a][j][e] += __shfl_xor_sync(0xffffffffu, acc[a][j][e], 8);
        acc[a][j][e] += __shfl_xor_sync(0xffffffffu, acc[a][j][e], 16);
      }
  if (ok) {
    for (int a = 0; a < 2; ++a) {
      const int g = warp % gs + a * gs;
      if (g >= p.G) break;
      const int R = p.k + (g == 0 ? 1 : 0);
      if (kq == 0) {
#pragma unroll
        for (int j = 0; j < KR; ++j) {
          if (j >= R) break;
          if (wpg == 1) {
            float* dst = p.part_o + (((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s) * 64 + 8 * c;
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = acc[a][j][e];
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) red[(warp * p.rmax + j) * 64 + 8 * c + e] = acc[a][j][e];
          }
        }
      }
    }
    if (wpg > 1) {
      // groups shared by several warps (G < 8): warps g, g + G, ... hold partial sums
      __syncthreads();
      for (int i = tid; i < p.G * p.rmax * 64; i += kDecThreads) {
        const int g = i / (p.rmax * 64), j = (i / 64) % p.rmax, d = i % 64;
        if (j >= p.k + (g == 0 ? 1 : 0)) continue;
        float a = 0.f;
        for (int t = 0; t < wpg; ++t) a += red[((g + t * gs) * p.rmax + j) * 64 + d];
        p.part_o[(((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s) * 64 + d] = a;
      }
    }
    for (int i = tid; i < p.G * p.rmax; i += kDecThreads) {
      const int g = i / p.rmax, j = i % p.rmax;
      const size_t at = ((size_t)(b * p.G + g) * p.rmax + j) * p.nsplit + s;
      const bool used = j < p.k + (g == 0 ? 1 : 0);
      p.part_ml[at * 2] = used ? ml[dec_slot(p, g, j) * 2] : -INFINITY;
      p.part_ml[at * 2 + 1] = used ? ml[dec_slot(p, g, j) * 2 + 1] : 0.f;
    }
  } else {
    // a wait ran out: let the copies in flight land before the block exits
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
}

// One block per (sequence b, query slot): all the key chunks' partial results
// are combined in parallel. Thread t takes dims d = t % 64 and every
// (blockDim/64)-th chunk; the chunk maxima are reduced first, then each
// thread accumulates 2^(m_s - M) o_s[d] and 2^(m_s - M) l_s over its chunks,
// and the partial sums are added through shared memory.
constexpr int kDecMergeThreads = 256;
__global__ void __launch_bounds__(kDecMergeThreads) decode_merge_kernel(const DecodeParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_red[kDecMergeThreads];
  __shared__ float s_l[kDecMergeThreads / 64];
  const int b = blockIdx.x / p.Ha, slot = blockIdx.x % p.Ha;
  const int g = slot < p.G * p.k ? slot / p.k : 0;
  const int r = slot < p.G * p.k ? slot % p.k : p.k;
  const size_t base = ((size_t)(b * p.G + g) * p.rmax + r) * p.nsplit;
  const int tid = threadIdx.x, d = tid & 63, part = tid >> 6;
  constexpr int kParts = kDecMergeThreads / 64;
  // the maximum over all chunks
  float M = -INFINITY;
  for (int s = tid; s < p.nsplit; s += kDecMergeThreads) M = fmaxf(M, p.part_ml[(base + s) * 2]);
  s_red[tid] = M;
  __syncthreads();
  for (int w = kDecMergeThreads / 2; w > 0; w >>= 1) {
    if (tid < w) s_red[tid] = fmaxf(s_red[tid], s_red[tid + w]);
    __syncthreads();
  }
  M = s_red[0];
  __syncthreads();
  float acc = 0.f, lsum = 0.f;
  if (M != -INFINITY) {
    // loads without branches, eight chunks at a time, so they are in flight
    // together; an empty chunk (m = -inf) contributes nothing and its partial
    // output (never written) is not used
    for (int s0 = part; s0 < p.nsplit; s0 += 8 * kParts) {
      float ms[8], ls[8], os[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s0 + u * kParts;
        const bool in = s < p.nsplit;
        ms[u] = in ? p.part_ml[(base + s) * 2] : -INFINITY;
        ls[u] = in ? p.part_ml[(base + s) * 2 + 1] : 0.f;
        os[u] = in ? p.part_o[(base + s) * 64 + d] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool live = ms[u] != -INFINITY;
        const float f = live ? exp2f(ms[u] - M) : 0.f;
        acc = fmaf(f, live ? os[u] : 0.f, acc);
        lsum = fmaf(f, live ? ls[u] : 0.f, lsum);
      }
    }
  }
  s_red[tid] = acc;
  if (d == 0) s_l[part] = lsum;
  __syncthreads();
  if (tid < 64) {
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int q = 0; q < kParts; ++q) {
      o += s_red[q * 64 + tid];
      l += s_l[q];
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    p.O[((size_t)b * p.Ha + slot) * 64 + tid] = __float2bfloat16_rn(o * inv);
  }
}

}  // namespace gqe
