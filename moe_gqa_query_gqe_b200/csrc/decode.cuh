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
// The token-side work (routing, projections, output projection) is in
// decode_proj.cuh for a few new tokens, else the prefill kernels with the B
// new tokens seen as one sequence of B tokens. This file holds the cache side:
//   decode_append_kernel   : K/V row of the new token -> cache position L_b
//                            (the prefill route only; decode_proj_kernel
//                            writes the rows itself)
//   decode_attn_mma_kernel : split-K attention over the caches, persistent,
//                            one contiguous key range per CTA, per-warp TMA
//                            rings, the dot products on mma.sync m16n8k16;
//                            the bound is the cache read (2 x 128 B per key
//                            and group)
//   decode_merge_kernel    : one block per (sequence, query slot) merges the
//                            partials: O = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
#pragma once

#include "sm100.cuh"

namespace gqe {

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

// Query slot of row j of group g: the group's k selected experts, then (group
// 0 only) the shared head.
__device__ __forceinline__ int dec_slot(const DecodeParams& p, int g, int j) {
  return j < p.k ? g * p.k + j : p.G * p.k;
}

// ---------------------------------------------------------------------------
// decode_attn_mma_kernel: the split-K attention with the dot products on the
// tensor cores. Persistent, one CTA per SM: the B sequences' keys, cut into
// items of kDmItem keys (sequence-major), are split into gridDim.x contiguous
// ranges of equal item count; CTA c takes range c, i.e. one key range in each
// sequence it touches. Each of its eight warps streams the cache rows of its
// own group through a private ring of kDmStages stages (a stage: kDmSK keys
// of K and of V of one group, 4 KB each, by two TMA tile loads with 128-byte
// swizzle), so the warps never wait on one another, and the ring runs on
// from one sequence's range to the next. Per stage, on mma.sync m16n8k16
// (bf16 in, fp32 accumulate):
//   S^T = Q K^T   query rows (the group's k experts, + the shared head in
//                 group 0) padded to 16, 8 keys per tile, 16 dims per step
//   online softmax over the stage's keys in the log2 domain (row maximum by
//                 two shuffles, running sum and output rescaled)
//   O  += P V     P in bf16; the score tile's accumulator fragments are the
//                 P operand's fragments (same thread layout), so P stays in
//                 registers; V by transposing matrix loads.
// With fewer than eight groups, wpg = 8 / G warps share a group and take
// every wpg-th stage of the range; with more, a warp takes groups w, w + 8,
// ... in turn. A warp leaves one partial (m, l, O) per (sequence, group, row)
// of its range, at split (c - c_first(b)) * wpg + sub, where c_first(b) is
// the first CTA whose range touches sequence b; the last such CTA also marks
// the sequence's remaining splits empty (m = -inf, l = 0) for
// decode_merge_kernel.
// ---------------------------------------------------------------------------
constexpr int kDmWarps = 8;
constexpr int kDmThreads = kDmWarps * 32;
constexpr int kDmSK = 32;                       // keys per stage
constexpr int kDmItem = 64;                     // keys per item (the unit of the split)
// ring depth per warp: 2 keeps the CTA at 129 KB of shared memory, so it
// fits on an SM beside two of the projection launch's CTAs and starts
// streaming the cache while they run (3 stages: 8 us slower per step)
constexpr int kDmStages = 2;
constexpr int kDmGridMax = 148;                 // CTAs at most (one per SM of a B200)
constexpr int kDmBlock = kDmSK * 128;           // one K (or V) block of a stage, bytes
constexpr int kDmStageBytes = 2 * kDmBlock;
constexpr int kDmWarpBytes = kDmStages * kDmStageBytes;
__host__ __device__ inline int dm_wpg(int G) { return G < kDmWarps ? kDmWarps / G : 1; }
__host__ __device__ inline int dm_smem() { return 1024 + kDmWarps * kDmWarpBytes + kDmWarps * kDmStages * 8 + 64; }
// Splits per (sequence, group, row): CTAs whose range touches one sequence
// (at most ceil(grid / B) + 1), times wpg.
__host__ __device__ inline int dm_nsplit(long long B, int G, int grid) {
  const long long per = (grid + B - 1) / B + 1;
  return (int)(per < grid ? per : grid) * dm_wpg(G);
}

struct DecodeMmaParams {
  CUtensorMap tmK, tmV;  // the caches as [B*T keys][G][64], box (64, 1, kDmSK)
  DecodeParams d;        // d.nsplit = dm_nsplit(B, G, gridDim.x)
  long long items;       // B * nitem
  int nitem;             // items per sequence
  int wpg;               // warps per group (G < 8), else 1
  int gpw;               // groups per warp (G > 8), else 1
};

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// First item of CTA c's range, and the CTA whose range holds item i.
__device__ __forceinline__ long long dm_start(long long items, int grid, int c) { return (long long)c * items / grid; }
__device__ __forceinline__ int dm_cta_of(long long items, int grid, long long i) {
  return (int)(((i + 1) * grid - 1) / items);
}

// The keys [k0, k1) of sequence b in CTA c's range, clipped to the new
// token's row L (k1 <= k0: none); L = -1 if cache_len[b] is out of range.
struct DmRange {
  int b, k0, k1, L;
};
__device__ __forceinline__ DmRange dm_range(const DecodeMmaParams& P, long long i0, long long i1, int b) {
  DmRange r;
  r.b = b;
  const int L = P.d.cache_len[b];
  r.L = (L < 0 || L >= P.d.T) ? -1 : L;
  if (r.L < 0) flag_bounds_error();
  const long long a = i0 > (long long)b * P.nitem ? i0 : (long long)b * P.nitem;
  const long long e = i1 < (long long)(b + 1) * P.nitem ? i1 : (long long)(b + 1) * P.nitem;
  r.k0 = (int)(a - (long long)b * P.nitem) * kDmItem;
  const int kend = (int)(e - (long long)b * P.nitem) * kDmItem;
  r.k1 = r.L < 0 ? 0 : min(kend, r.L + 1);
  return r;
}

__global__ void __launch_bounds__(kDmThreads, 1) decode_attn_mma_kernel(const __grid_constant__ DecodeMmaParams P) {
  pdl_trigger();
  const DecodeParams& p = P.d;
  extern __shared__ uint8_t dm_raw[];
  uint8_t* base = dm_raw + ((1024u - (smem_u32(dm_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* ring = base + warp * kDmWarpBytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + kDmWarps * kDmWarpBytes) + warp * kDmStages;
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(base + kDmWarps * kDmWarpBytes + kDmWarps * kDmStages * 8) + warp;
  const int grid = gridDim.x, cta = blockIdx.x;
  const long long i0 = dm_start(P.items, grid, cta), i1 = dm_start(P.items, grid, cta + 1);
  const int b_first = (int)(i0 / P.nitem), b_last = (int)((i1 - 1) / P.nitem);
  const int sub = P.wpg > 1 ? warp / p.G : 0;    // this warp's share of a group's stages
  const int g0 = P.wpg > 1 ? warp % p.G : warp;  // first group; then g0 + 8, ... (gpw of them)
  const int ngr = P.gpw;
  if (lane == 0) {
    for (int i = 0; i < kDmStages; ++i) mbar_init(&bar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&P.tmK);
    tma_prefetch_desc(&P.tmV);
  }
  __syncwarp();

  // ---- producer cursor (lane 0): the next stage to load -------------------------
  // order: sequence b, group ordinal gi, stage st = sub, sub + wpg, ...
  int pb = b_first, pgi = 0, pst = sub;
  bool pdone = false;
  DmRange pr = dm_range(P, i0, i1, pb);
  auto p_settle = [&]() {  // move the cursor to an existing stage, or finish
    while (true) {
      const int nst = pr.k0 < pr.k1 ? (pr.k1 - pr.k0 + kDmSK - 1) / kDmSK : 0;
      if (pst < nst) return;
      pst = sub;
      if (++pgi == ngr) {
        pgi = 0;
        if (++pb > b_last) {
          pdone = true;
          return;
        }
        pr = dm_range(P, i0, i1, pb);
      }
    }
  };
  uint32_t issued = 0;
  auto p_issue = [&]() {  // load the cursor's stage into the next slot, advance
    const int slot = issued % kDmStages;
    const int key0 = pr.k0 + pst * kDmSK;
    const int g = g0 + 8 * pgi;
    uint8_t* dst = ring + slot * kDmStageBytes;
    mbar_arrive_expect_tx(&bar[slot], 2 * kDmBlock);
    tma_load_3d(dst, &P.tmK, &bar[slot], 0, g, pr.b * p.T + key0);
    tma_load_3d(dst + kDmBlock, &P.tmV, &bar[slot], 0, g, pr.b * p.T + key0);
    ++issued;
    pst += P.wpg;
    p_settle();
  };
  auto p_has_new = [&]() {  // the cursor's stage holds the new token's row
    return pr.k1 == pr.L + 1 && pr.k0 + (pst + 1) * kDmSK > pr.L;
  };
  if (lane == 0) {
    // rows before the new token's depend on no launch of this step: they load
    // before the wait for the projection launch, which writes row L and Q
    p_settle();
    while (!pdone && issued < kDmStages && !p_has_new()) p_issue();
  }
  pdl_wait();
  if (lane == 0)
    while (!pdone && issued < kDmStages) p_issue();

  // ---- consumer: the same (sequence, group, stage) order ------------------------
  const int r = lane >> 2, c = lane & 3;    // fragment row (query row) and column pair
  const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix and row this lane addresses
  const uint32_t ring_s = smem_u32(ring);
  uint32_t consumed = 0;
  bool ok = true;
  for (int b = b_first; ok && b <= b_last; ++b) {
    const DmRange rg = dm_range(P, i0, i1, b);
    const int nkeys = rg.k1 - rg.k0;
    const int nst = nkeys > 0 ? (nkeys + kDmSK - 1) / kDmSK : 0;
    const int c_first = dm_cta_of(P.items, grid, (long long)b * P.nitem);
    const int c_last = dm_cta_of(P.items, grid, (long long)(b + 1) * P.nitem - 1);
    const int split = (cta - c_first) * P.wpg + sub;
    for (int gi = 0; ok && gi < ngr; ++gi) {
      const int g = g0 + 8 * gi;
      const int R = p.k + (g == 0 ? 1 : 0);  // query rows of this group
      const bool any = nst > sub;            // this warp has stages here
      // query A fragments: rows r and r + 8 (zero past R), dims 16 kk + 2c (+1, +8, +9)
      uint32_t qa[4][4];
      {
        const __nv_bfloat16* q0 = p.Q + ((size_t)b * p.Ha + dec_slot(p, g, r)) * 64;
        const __nv_bfloat16* q1 = p.Q + ((size_t)b * p.Ha + dec_slot(p, g, r + 8)) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int d0 = 16 * kk + 2 * c;
          qa[kk][0] = (any && r < R) ? *reinterpret_cast<const uint32_t*>(q0 + d0) : 0u;
          qa[kk][1] = (any && r + 8 < R) ? *reinterpret_cast<const uint32_t*>(q1 + d0) : 0u;
          qa[kk][2] = (any && r < R) ? *reinterpret_cast<const uint32_t*>(q0 + d0 + 8) : 0u;
          qa[kk][3] = (any && r + 8 < R) ? *reinterpret_cast<const uint32_t*>(q1 + d0 + 8) : 0u;
        }
      }
      float o[8][4];
#pragma unroll
      for (int dt = 0; dt < 8; ++dt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[dt][e] = 0.f;
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      for (int st = sub; st < nst; st += P.wpg) {
        const int slot = consumed % kDmStages;
        ok = mbar_wait(&bar[slot], (consumed / kDmStages) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        const int nk = min(kDmSK, nkeys - st * kDmSK);  // valid keys of the stage
        const uint32_t kb = ring_s + slot * kDmStageBytes, vb = kb + kDmBlock;
        if (nk < kDmSK) {
          // rows past the new token (another sequence's, or never written):
          // their V must not reach P V (0 x NaN), so zero them
          uint4* vz = reinterpret_cast<uint4*>(ring + slot * kDmStageBytes + kDmBlock);
          for (int i = nk * 8 + lane; i < kDmSK * 8; i += 32) vz[i] = make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();  // before the slot is refilled by TMA
          __syncwarp();
        }
        // ---- S^T = Q K^T: 4 tiles of 8 keys ---------------------------------------
        float sc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int np = 0; np < 2; ++np) {
            const int key = np * 16 + (mi >> 1) * 8 + mr, ch = 2 * kk + (mi & 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kb + key * 128 + ((ch ^ (key & 7)) << 4), b0, b1, b2, b3);
            mma_bf16_16816(sc[2 * np], qa[kk], b0, b1);
            mma_bf16_16816(sc[2 * np + 1], qa[kk], b2, b3);
          }
        // ---- online softmax (log2 domain) -----------------------------------------
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool valid = nt * 8 + 2 * c + e < nk;
            sc[nt][e] = valid ? sc[nt][e] * p.scale_log2 : -INFINITY;
            sc[nt][2 + e] = valid ? sc[nt][2 + e] * p.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, sc[nt][e]);
            mx1 = fmaxf(mx1, sc[nt][2 + e]);
          }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            sc[nt][e] = exp2f(sc[nt][e] - mn0);
            sc[nt][2 + e] = exp2f(sc[nt][2 + e] - mn1);
            ls0 += sc[nt][e];
            ls1 += sc[nt][2 + e];
          }
        l0 = fmaf(l0, al0, ls0);
        l1 = fmaf(l1, al1, ls1);
#pragma unroll
        for (int dt = 0; dt < 8; ++dt) {
          o[dt][0] *= al0;
          o[dt][1] *= al0;
          o[dt][2] *= al1;
          o[dt][3] *= al1;
        }
        // ---- O += P V: 2 steps of 16 keys, 8 tiles of 8 dims ----------------------
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
          const uint32_t pa[4] = {pack_bf16x2(sc[2 * ks][0], sc[2 * ks][1]), pack_bf16x2(sc[2 * ks][2], sc[2 * ks][3]),
                                  pack_bf16x2(sc[2 * ks + 1][0], sc[2 * ks + 1][1]),
                                  pack_bf16x2(sc[2 * ks + 1][2], sc[2 * ks + 1][3])};
#pragma unroll
          for (int dp = 0; dp < 4; ++dp) {
            const int key = ks * 16 + (mi & 1) * 8 + mr, ch = 2 * dp + (mi >> 1);
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vb + key * 128 + ((ch ^ (key & 7)) << 4), b0, b1, b2, b3);
            mma_bf16_16816(o[2 * dp], pa, b0, b1);
            mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
          }
        }
        ++consumed;
        __syncwarp();  // every lane is done with the slot
        if (lane == 0 && !pdone) p_issue();
      }
      if (!ok) break;
      // ---- this warp's partial of (b, g) over the range -----------------------------
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = r + 8 * h;
        if (j >= p.rmax) continue;
        const bool live = j < R && any;
        const size_t row = (size_t)(b * p.G + g) * p.rmax + j;
        const size_t at = row * p.nsplit + split;
        if (c == 0) {
          p.part_ml[at * 2] = live ? (h ? m1 : m0) : -INFINITY;
          p.part_ml[at * 2 + 1] = live ? (h ? l1 : l0) : 0.f;
          if (cta == c_last)  // the sequence's splits no CTA writes: empty
            for (int sp = (c_last - c_first + 1) * P.wpg + sub; sp < p.nsplit; sp += P.wpg) {
              p.part_ml[(row * p.nsplit + sp) * 2] = -INFINITY;
              p.part_ml[(row * p.nsplit + sp) * 2 + 1] = 0.f;
            }
        }
        if (live) {
          float* dst = p.part_o + at * 64;
#pragma unroll
          for (int dt = 0; dt < 8; ++dt)
            *reinterpret_cast<float2*>(dst + dt * 8 + 2 * c) = make_float2(o[dt][2 * h], o[dt][2 * h + 1]);
        }
      }
    }
  }
  if (!ok) {
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
