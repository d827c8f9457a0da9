// gemm2sm.cuh -- dense projection GEMM on CTA pairs (tcgen05 .cta_group::2):
// C = A * B, bf16 in, fp32 accumulate in TMEM, bf16 out. Used for the K/V (and
// shared-head Q) projection, the output projection Wo and the dense GQA
// baseline's projections.
//
//   A [rows, K] row-major (K-major operand), B [K, N] row-major weight
//   (MN-major operand), both by TMA with 128-byte swizzle; up to three output
//   segments (weights) per launch, as in gemm2.cuh.
//
// Why pairs: a 128 x 256 tile on one SM needs 48 KB of operands per 64-deep
// k-block for 512 tensor-core cycles, more than one SM pulls from L2. A pair
// of SMs computes a 256 x 256 tile: each SM loads its 128 rows of A and half
// (128 columns) of B, 32 KB per k-block for the same 512 cycles, and the MMA
// issued by the even CTA reads both CTAs' shared memory.
//
// Per pair tile (256 rows x up to 256 columns; narrow segment tails are
// rounded up to 128 columns so both halves of B are whole 64-column boxes):
//   warp 0 (both CTAs)   TMA producer: A rows [m0 + 128*rank, +128) and B
//                        columns [n0 + rank*N/2, +N/2); the bytes of both CTAs
//                        are counted on the even CTA's stage barrier
//   warp 1 (even CTA)    TMEM owner + MMA issue (M=256, N, K=16 per MMA);
//                        its commits release the stage in both CTAs and mark
//                        the accumulator full in both
//   warps 2..5 (both)    epilogue: this CTA's 128 rows from its own TMEM,
//                        converted to bf16 into swizzled shared-memory rows
//                        (one row per lane) and written by TMA stores of 32
//                        rows x 64 columns, then one arrival per warp on the
//                        even CTA's accumulator-empty barrier
// TMEM: two 256-column accumulators per CTA (double buffer), so the epilogue
// of one tile overlaps the main loop of the next.
#pragma once

#include "gemm.cuh"
#include "route.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kPairBM = 256;  // rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;  // columns per pair tile (B: 128 per CTA)
constexpr int kPairStages = 6;
constexpr int kPairThreads = 192;

struct PairSmem {
  static constexpr int kABytes = 128 * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = 128 * kGemmBK * 2;  // two 64-column boxes of 8 KB
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kBar = kPairStages * kStage;  // (end of the stages)
  static constexpr int kStageOut = kBar;               // epilogue staging: 4 warps x 2 x (32 rows x 128 B)
  static constexpr int kOutBytes = 4096;
  static constexpr int kBarOff = kStageOut + 4 * 2 * kOutBytes;
  static constexpr int kTot = kBarOff + 256;          // routing epilogue: 8 groups x 4 warps of u64
  static constexpr int kBytes = kTot + 256 + 1024;    // + alignment slack
};

struct PairTile {
  int m0;      // first row of the pair tile
  int seg;     // output segment; -1: routing tile
  int n0;      // first column within the segment; routing tile: block of 256 tokens
  int nvalid;  // MMA N: multiple of 128, <= 256
  int rb;      // routing tile: sequence
};

__device__ __forceinline__ PairTile pair_decode(const GemmParams& p, int tile) {
  PairTile t;
  if (tile >= p.r_tile0) {
    const int rt = tile - p.r_tile0;
    t.rb = rt / p.r_nblk;
    t.n0 = rt % p.r_nblk;
    t.m0 = t.rb * p.r_T + t.n0 * kPairBM;
    t.seg = -1;
    t.nvalid = 128;  // G*M <= 64 logits in the even CTA's half; the odd half reads zeros
    return t;
  }
  const int mt = tile / p.ntn, nt = tile % p.ntn;
  t.m0 = mt * kPairBM;
  t.seg = 0;
  for (int s = 1; s < p.nseg; ++s)
    if (nt >= p.seg[s].tile_start) t.seg = s;
  t.n0 = (nt - p.seg[t.seg].tile_start) * kPairBN;
  const int rem = p.seg[t.seg].n_cols - t.n0;
  t.nvalid = rem >= kPairBN ? kPairBN : ((rem + 127) / 128) * 128;
  t.rb = 0;
  return t;
}

// RM (1, 2, 4 or 8) consecutive fp32 TMEM columns of this warp's 32 lanes.
template <int RM>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float (&f)[RM]) {
  if constexpr (RM == 1) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\ttcgen05.wait::ld.sync.aligned;"
                 : "=f"(f[0]) : "r"(taddr) : "memory");
  } else if constexpr (RM == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];\n\ttcgen05.wait::ld.sync.aligned;"
                 : "=f"(f[0]), "=f"(f[1]) : "r"(taddr) : "memory");
  } else if constexpr (RM == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];\n\ttcgen05.wait::ld.sync.aligned;"
                 : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]) : "r"(taddr) : "memory");
  } else {
    static_assert(RM == 8, "RM");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\ttcgen05.wait::ld.sync.aligned;"
        : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]), "=f"(f[4]), "=f"(f[5]), "=f"(f[6]), "=f"(f[7])
        : "r"(taddr)
        : "memory");
  }
}

// Routing epilogue of one CTA of a routing pair tile: its 128 rows are chunk c
// of sequence b (one thread per token). Per group: logits from TMEM (+ br),
// the decision (route.cuh), then a block scan over the chunk of packed 8-bit
// per-expert flags gives each token its rank in its experts' lists and the
// chunk's per-expert counts. Groups go eight at a time through s_tot.
template <int RM, bool PR>
__device__ void pair_route_epilogue(const GemmParams& p, uint32_t tm, int b, int c, int q, int lane,
                                    unsigned long long* s_tot) {
  const int row = q * 32 + lane;
  const int t = c * kRouteChunk + row;
  const bool valid = t < p.r_T;
  const size_t n = (size_t)b * p.r_T + (valid ? t : 0);
  const int G = p.G, k = p.k, GM = G * RM;
  for (int g0 = 0; g0 < G; g0 += 8) {
    const int gn = min(8, G - g0);
    unsigned long long mine[8], incl[8];
    uint32_t chosen[8];
#pragma unroll
    for (int gi = 0; gi < 8; ++gi) {
      mine[gi] = 0;
      chosen[gi] = 0;
      if (gi < gn) {
        const int g = g0 + gi;
        float l[RM];
        tmem_ld_cols<RM>(tm + g * RM, l);
#pragma unroll
        for (int e = 0; e < RM; ++e) l[e] += p.r_br ? p.r_br[g * RM + e] : 0.f;
        const size_t o = (n * G + g) * k;
        chosen[gi] = route_decide<RM, PR>(l, k, valid, p.r_sel + o, p.r_w + o,
                                          p.r_margin ? p.r_margin + n * G + g : nullptr, PR ? p.r_p + o : nullptr);
        if (valid)
#pragma unroll
          for (int e = 0; e < RM; ++e)
            if (chosen[gi] & (1u << e)) mine[gi] += 1ull << (8 * e);
      }
      incl[gi] = mine[gi];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long u = __shfl_up_sync(0xffffffffu, incl[gi], o);
        if (lane >= o) incl[gi] += u;
      }
      if (lane == 31) s_tot[gi * 4 + q] = incl[gi];
    }
    named_barrier_sync(1, 128);
#pragma unroll
    for (int gi = 0; gi < 8; ++gi) {
      if (gi >= gn) break;
      const int g = g0 + gi;
      unsigned long long base = 0, total = 0;
      for (int w = 0; w < 4; ++w) {
        if (w < q) base += s_tot[gi * 4 + w];
        total += s_tot[gi * 4 + w];
      }
      const unsigned long long excl = base + incl[gi] - mine[gi];
      if (valid) {
        int j = 0;
#pragma unroll
        for (int e = 0; e < RM; ++e) {
          if (!(chosen[gi] & (1u << e))) continue;
          const int rank = static_cast<int>((excl >> (8 * e)) & 0xFFull);
          p.r_sel[(n * G + g) * k + j] = e | (rank << 8);
          ++j;
        }
      }
      if (row < RM) p.r_counts[((size_t)b * p.r_nch + c) * GM + g * RM + row] = static_cast<int>((total >> (8 * row)) & 0xFFull);
    }
    named_barrier_sync(1, 128);
  }
}

// The same decisions as plain expert ids, without ranks and counts (for a
// forward pass that does not build segment lists).
template <int RM, bool PR>
__device__ void pair_route_plain(const GemmParams& p, uint32_t tm, int b, int c, int q, int lane) {
  const int t = c * kRouteChunk + q * 32 + lane;
  const bool valid = t < p.r_T;
  const size_t n = (size_t)b * p.r_T + (valid ? t : 0);
  const int G = p.G, k = p.k;
  for (int g = 0; g < G; ++g) {
    float l[RM];
    tmem_ld_cols<RM>(tm + g * RM, l);
#pragma unroll
    for (int e = 0; e < RM; ++e) l[e] += p.r_br ? p.r_br[g * RM + e] : 0.f;
    const size_t o = (n * G + g) * k;
    route_decide<RM, PR>(l, k, valid, p.r_sel + o, p.r_w + o, p.r_margin ? p.r_margin + n * G + g : nullptr,
                         PR ? p.r_p + o : nullptr);
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p, int total_tiles) {
  // A selected-query launch reads only inputs (x, Wq) in its main loop: the
  // wait for the routing launch is left to the epilogue, before it reads sel.
  if (p.sel_seg < 0) pdl_wait();
  pdl_trigger();
  using L = PairSmem;
  extern __shared__ uint8_t smem_raw[];
  // same offset in both CTAs: the MMA addresses the peer's operands by it
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);  // [stages], used in the even CTA
  uint64_t* empty = full + kPairStages;                           // [stages]
  uint64_t* acc_full = empty + kPairStages;                       // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2], used in the even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  unsigned long long* s_tot = reinterpret_cast<unsigned long long*>(smem + L::kTot);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nk = (p.K + kGemmBK - 1) / kGemmBK;

  if (tid == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);   // the even producer's arrive.expect_tx
      mbar_init(&empty[s], 1);  // the MMA commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 8);  // 4 epilogue warps x 2 CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, 2 * kPairBN);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    for (int s = 0; s < p.nseg; ++s) tma_prefetch_desc(&p.tmB[s]);
    if (p.r_tile0 < total_tiles || p.r_merge_seg >= 0) tma_prefetch_desc(&p.tmR);
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer (both CTAs) --------------------------------------------
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += npairs) {
        const PairTile t = pair_decode(p, tile);
        const int half = t.nvalid / 2;  // columns of B this CTA holds
        const int nbox = half / 64;
        // routing tile, or the odd CTA's half of a tile carrying the router
        const bool rt = t.seg < 0 || (t.seg == p.r_merge_seg && rank == 1);
        const int b_col = t.seg < 0 ? (int)rank * half : (rt ? 0 : p.seg[t.seg].b_col0 + t.n0 + (int)rank * half);
        const CUtensorMap* tmb = rt ? &p.tmR : &p.tmB[t.seg];
        const int a_row = t.m0 + (int)rank * 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPairStages;
          if (!(ok = mbar_wait(&empty[s], ((it / kPairStages) & 1) ^ 1, abort_flag))) break;
          const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
          // the even CTA announces both CTAs' bytes; the odd CTA's copies may
          // land first (the count then dips below zero until the announcement)
          if (leader) mbar_arrive_expect_tx(&full[s], 2 * (L::kABytes + nbox * 8192));
          int a_col = kb * kGemmBK;
          if (p.amap_G > 0) {
            // k = 1 combine: A = [concat (G) | slot (G) | shared] read from O,
            // the slot of group g being O's block g itself (weight exactly 1)
            const int blk = kb < 2 * p.amap_G ? kb % p.amap_G : p.amap_G;
            a_col = blk * kGemmBK;
          }
          uint8_t* a_s = smem + s * L::kStage;
          uint8_t* b_s = a_s + L::kABytes;
          tma_load_2d_pair(a_s, &p.tmA, fb, a_col, a_row);
          for (int nb = 0; nb < nbox; ++nb) tma_load_2d_pair(b_s + nb * 8192, tmb, fb, b_col + nb * 64, kb * kGemmBK);
        }
      }
      // wait until the MMA has released every stage in flight, so no commit
      // arrival can reach this CTA after it has left
      for (uint32_t i = it; ok && i < it + kPairStages; ++i)
        ok = mbar_wait(&empty[i % kPairStages], ((i / kPairStages) & 1) ^ 1, abort_flag);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      // ---- MMA issue (even CTA) -------------------------------------------------
      // cluster addresses of the stage-empty and accumulator-full barriers of
      // both CTAs (a CTA's shared memory is contiguous in the cluster window)
      const uint32_t empty_c0 = mapa_shared(smem_u32(empty), 0), empty_c1 = mapa_shared(smem_u32(empty), 1);
      const uint32_t accf_c0 = mapa_shared(smem_u32(acc_full), 0), accf_c1 = mapa_shared(smem_u32(acc_full), 1);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total_tiles; tile += npairs, ++tcount) {
        const PairTile t = pair_decode(p, tile);
        const uint32_t a = tcount & 1;
        if (!(ok = mbar_wait(&acc_empty[a], ((tcount >> 1) & 1) ^ 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * kPairBN;
        const uint32_t idesc = idesc_bf16(kPairBM, t.nvalid, false, true);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPairStages;
          if (!(ok = mbar_wait(&full[s], (it / kPairStages) & 1, abort_flag))) break;
          tc_fence_after();
          const uint32_t a_addr = smem_base + s * L::kStage;
          const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            umma_ss_pair(d_tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), sdesc_sw128(b_addr + kk * 2048, 8192, 1024),
                         idesc, (kb | kk) != 0);
          umma_commit_pair(empty_c0 + 8 * s);
          umma_commit_pair(empty_c1 + 8 * s);
        }
        if (!ok) break;
        umma_commit_pair(accf_c0 + 8 * a);
        umma_commit_pair(accf_c1 + 8 * a);
      }
    }
  } else {
    // ---- epilogue (both CTAs): this CTA's 128 rows ----------------------------------
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    if (p.sel_seg >= 0) pdl_wait();
    const uint32_t acce_c = mapa_shared(smem_u32(acc_empty), 0);
    uint8_t* stage_out = smem + L::kStageOut + q * 2 * L::kOutBytes;  // this warp's two staging buffers
    uint32_t nstore = 0;                                               // chunks staged by this warp
    uint32_t tcount = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs, ++tcount) {
      const PairTile t = pair_decode(p, tile);
      const uint32_t a = tcount & 1;
      const bool ok = mbar_wait(&acc_full[a], (tcount >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // routing decisions of this CTA's 128 tokens (chunk c of sequence b)
      // from the logits at TMEM column tm
      auto route = [&](uint32_t tm, int b, int c) {
        if (p.r_counts == nullptr) {
          if (p.r_p == nullptr) {
            switch (p.M) {
              case 1: pair_route_plain<1, false>(p, tm, b, c, q, lane); break;
              case 2: pair_route_plain<2, false>(p, tm, b, c, q, lane); break;
              case 4: pair_route_plain<4, false>(p, tm, b, c, q, lane); break;
              default: pair_route_plain<8, false>(p, tm, b, c, q, lane); break;
            }
          } else {
            switch (p.M) {
              case 1: pair_route_plain<1, true>(p, tm, b, c, q, lane); break;
              case 2: pair_route_plain<2, true>(p, tm, b, c, q, lane); break;
              case 4: pair_route_plain<4, true>(p, tm, b, c, q, lane); break;
              default: pair_route_plain<8, true>(p, tm, b, c, q, lane); break;
            }
          }
        } else if (p.r_p == nullptr) {
          switch (p.M) {
            case 1: pair_route_epilogue<1, false>(p, tm, b, c, q, lane, s_tot); break;
            case 2: pair_route_epilogue<2, false>(p, tm, b, c, q, lane, s_tot); break;
            case 4: pair_route_epilogue<4, false>(p, tm, b, c, q, lane, s_tot); break;
            default: pair_route_epilogue<8, false>(p, tm, b, c, q, lane, s_tot); break;
          }
        } else {  // the weighted-concatenation variant also writes the probabilities
          switch (p.M) {
            case 1: pair_route_epilogue<1, true>(p, tm, b, c, q, lane, s_tot); break;
            case 2: pair_route_epilogue<2, true>(p, tm, b, c, q, lane, s_tot); break;
            case 4: pair_route_epilogue<4, true>(p, tm, b, c, q, lane, s_tot); break;
            default: pair_route_epilogue<8, true>(p, tm, b, c, q, lane, s_tot); break;
          }
        }
      };
      if (t.seg < 0) {
        const uint32_t tm = tmem_base + a * kPairBN + (static_cast<uint32_t>(q * 32) << 16);
        const int c = t.n0 * 2 + (int)rank;  // this CTA's chunk of 128 tokens
        if (c < p.r_nch) route(tm, t.rb, c);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_c + 8 * a);
        continue;
      }
      const GemmSeg& sg = p.seg[t.seg];
      const int wrow0 = t.m0 + (int)rank * 128 + q * 32;  // first row of this warp
      const int ncols = min(t.nvalid, sg.n_cols - t.n0);
      const uint32_t tm = tmem_base + a * kPairBN + (static_cast<uint32_t>(q * 32) << 16);
      if (t.seg == p.sel_seg) {
        // routed heads: lane = token n; head h's 64 columns go to Q slot
        // g*k + j if the token selected expert e = h % M of group g = h / M
        // (slot j), else nowhere. Each lane stores its own 128-byte row.
        const int n = wrow0 + lane;
#pragma unroll 1
        for (int ch = 0; ch < t.nvalid / 64; ++ch) {
          uint32_t r[64];
          tmem_ld64(tm + ch * 64, r);
          if (ch * 64 >= ncols || n >= p.rows) continue;
          const int h = (sg.b_col0 + t.n0) / 64 + ch;
          const int g = h / p.M, e = h % p.M;
          const int32_t* sl = p.sel + ((size_t)n * p.G + g) * p.k;
          int j = -1;
          for (int jj = 0; jj < p.k; ++jj)
            if ((sl[jj] & 0xff) == e) j = jj;
          if (j < 0) continue;
          uint4* dst = reinterpret_cast<uint4*>(p.Q + ((size_t)n * p.Ha + g * p.k + j) * 64);
#pragma unroll
          for (int c = 0; c < 8; ++c)
            dst[c] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * c]), __uint_as_float(r[8 * c + 1])),
                                pack_bf16x2(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3])),
                                pack_bf16x2(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5])),
                                pack_bf16x2(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7])));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acce_c + 8 * a);
        continue;
      }
      // 64-column chunks: TMEM -> registers -> bf16 -> swizzled staging rows (one
      // row per lane, conflict-free) -> one TMA store of 32 rows x 64 columns
      for (int ch = 0; ch < t.nvalid / 64; ++ch) {
        uint32_t r[64];
        tmem_ld64(tm + ch * 64, r);
        if (ch * 64 >= ncols || wrow0 >= p.rows) continue;  // warp-uniform
        uint8_t* sb = stage_out + (nstore & 1) * L::kOutBytes;
        // the store issued two chunks ago from this buffer must have read it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        const uint32_t rb = smem_u32(sb) + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4(rb + ((c ^ (lane & 7)) << 4), pack_bf16x2(__uint_as_float(r[8 * c]), __uint_as_float(r[8 * c + 1])),
                       pack_bf16x2(__uint_as_float(r[8 * c + 2]), __uint_as_float(r[8 * c + 3])),
                       pack_bf16x2(__uint_as_float(r[8 * c + 4]), __uint_as_float(r[8 * c + 5])),
                       pack_bf16x2(__uint_as_float(r[8 * c + 6]), __uint_as_float(r[8 * c + 7])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmC[t.seg], sb, sg.c_col0 + t.n0 + ch * 64, wrow0);
          bulk_commit();
        }
        ++nstore;
      }
      if (t.seg == p.r_merge_seg) {
        // columns 64..127 are this CTA's tokens' router logits (one chunk)
        const int row0 = t.m0 + (int)rank * 128;
        if (row0 < p.rows) route(tm + 64, row0 / p.r_T, (row0 % p.r_T) / kRouteChunk);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acce_c + 8 * a);
    }
  }

  if (warp >= 2 && lane == 0) bulk_wait_all();  // this warp's output stores have landed
  tc_fence_before();
  if (*abort_flag) {
    // copies of either CTA may still be landing on this CTA's buffers
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
  __syncwarp();  // lanes that skipped a single-lane role wait for it, so every warp arrives whole
  cluster_sync();  // no CTA leaves while its peer's MMAs or arrivals may still reach it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kPairBN);
  }
}

}  // namespace gqe
