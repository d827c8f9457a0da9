// gemm2.cuh -- persistent single-CTA tcgen05 GEMM for the selected-expert
// query projection when the head's weight slice is too large to stay resident
// in shared memory (D > 1024; qgather.cuh covers D <= 1024): for every expert
// segment s = (b, g, e), Q rows of the tokens that picked expert e of group g
// are x[token] * Wq[:, head g*M+e], written to token-major Q at slot (g, j).
//
//   A [rows, K] (K-major operand): rows gathered by the segment's token list
//     with 16-byte cp.async by eight copier warps, so only tokens that picked
//     the expert are multiplied.
//   B [K, 64] slice of the row-major weight (MN-major operand), streamed in
//     64 x 64 TMA boxes with 128-byte swizzle alongside the A rows.
//   Tiles of 128 rows of one segment; persistent CTAs walk the tile list
//   round-robin. The TMEM accumulator is double-buffered (2 x BN columns),
//   so the epilogue of one tile overlaps the main loop of the next.
//
// Warp roles (one CTA per SM, 448 threads):
//   warp 0     : TMA producer of the weight boxes (lane 0)
//   warp 1     : TMEM allocation + MMA issue (lane 0)
//   warps 2..5 : epilogue (TMEM lanes 32*(warp%4) .. +31), rows scattered to Q
//   warps 6..13: A copiers
#pragma once

#include "gemm.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kG2MaxSegsSmem = 8192;  // gather mode: segment tile prefix kept in shared memory

template <int BN, int STAGES>
struct G2Cfg {
  static constexpr int kThreads = 448;  // 8 of the 14 warps copy the gathered A rows
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = BN * kGemmBK * 2;       // BN/64 boxes of 8 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kPrefixOffset = kBarOffset + 256;
  static constexpr int kBytesBase = kPrefixOffset + 1024;  // + (nsegs+1)*4 for the tile prefix
};

struct G2Tile {
  int m0;             // first compacted row offset within the segment
  int seg;            // expert segment
  int nvalid;         // columns computed (64: one head)
  int row0, row_end;  // compacted row range of the tile
};

__device__ __forceinline__ G2Tile g2_decode(const GemmParams& p, int tile, const int* s_prefix) {
  G2Tile t;
  // largest s with s_prefix[s] <= tile
  int lo = 0, hi = p.nsegs_q - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  t.seg = lo;
  const int mt = tile - s_prefix[lo];
  t.m0 = mt * kGemmBM;
  t.row0 = p.seg_off[lo] + t.m0;
  t.row_end = min(p.seg_off[lo + 1], p.seg_off[p.nsegs_q]);
  t.nvalid = 64;
  return t;
}

template <int BN, int STAGES>
__global__ void __launch_bounds__(G2Cfg<BN, STAGES>::kThreads, 1)
    gemm2_kernel(const __grid_constant__ GemmParams p, int total_tiles) {
  pdl_wait();
  pdl_trigger();
  using C = G2Cfg<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(smem + C::kPrefixOffset);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = (p.K + kGemmBK - 1) / kGemmBK;

  // tile prefix over the expert segments: s_prefix[s] = tiles before segment s
  if (warp == 0) {
    int before = 0;
    for (int s0 = 0; s0 < p.nsegs_q; s0 += 32) {
      const int s = s0 + lane;
      const int len = s < p.nsegs_q ? p.seg_off[s + 1] - p.seg_off[s] : 0;
      const int nt = (len + kGemmBM - 1) / kGemmBM;
      int incl = nt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (s < p.nsegs_q) s_prefix[s] = before + incl - nt;
      before += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_prefix[p.nsegs_q] = before;
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1 + 256);  // the weight boxes' arrival + one per copier thread
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * BN);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB[0]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);
  const int ntiles = min(total_tiles, s_prefix[p.nsegs_q]);
  const int* prefix = s_prefix;

  if (warp == 0) {
    // ---- TMA producer: the weight boxes of every stage ---------------------------
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      const G2Tile t = g2_decode(p, tile, prefix);
      const int b_col = (t.seg % (p.G * p.M)) * 64;  // head h = g*M + e of segment (b, g, e)
      const CUtensorMap* tmb = &p.tmB[0];
      const int nbox = t.nvalid / 64;
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        bool w_ok = true;
        if (lane == 0) w_ok = mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag);
        if (!(ok = __shfl_sync(0xffffffffu, w_ok, 0))) break;
        uint8_t* b_s = smem + s * C::kStageBytes + C::kABytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], nbox * 8192);
          for (int nb = 0; nb < nbox; ++nb)
            tma_load_2d(b_s + nb * 8192, tmb, &full[s], b_col + nb * 64, kb * kGemmBK);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issue ------------------------------------------------------------
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++tcount) {
        const G2Tile t = g2_decode(p, tile, prefix);
        const uint32_t a = tcount & 1;
        if (!(ok = mbar_wait(&acc_empty[a], ((tcount >> 1) & 1) ^ 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * BN;
        const uint32_t idesc = idesc_bf16(kGemmBM, t.nvalid, false, true);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % STAGES;
          if (!(ok = mbar_wait(&full[s], (it / STAGES) & 1, abort_flag))) break;
          // rows copied by cp.async (generic proxy) are read by the MMA (async proxy)
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a_addr = smem_base + s * C::kStageBytes;
          const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            umma_ss(d_tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), sdesc_sw128(b_addr + kk * 2048, 8192, 1024),
                    idesc, (kb | kk) != 0);
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[a]);
      }
    }
  } else if (warp >= 6) {
    // ---- A copiers (warps 6..13): 16-byte chunk c of rows r = i*32 + ct/8 -------
    // The token rows of the next tile are fetched while this tile's copies run,
    // so no copier waits on a token-list load at a tile boundary.
    const int ct = tid - 192;  // 0..255
    const int c = ct & 7;
    uint32_t it = 0;
    bool ok = true;
    auto fetch_rows = [&](int tile, int (&tk)[4]) {
      const G2Tile t = g2_decode(p, tile, prefix);
      const int first = p.seg_tok[t.row0];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = i * 32 + (ct >> 3);
        tk[i] = (t.row0 + r < t.row_end) ? p.seg_tok[t.row0 + r] : first;
      }
    };
    int tk_cur[4] = {0, 0, 0, 0}, tk_next[4] = {0, 0, 0, 0};
    if ((int)blockIdx.x < ntiles) fetch_rows(blockIdx.x, tk_cur);
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      if (tile + (int)gridDim.x < ntiles) fetch_rows(tile + gridDim.x, tk_next);
      uint32_t dst_off[4];
      const __nv_bfloat16* src[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = i * 32 + (ct >> 3);
        int v = tk_cur[i];
        if (v < 0 || v >= p.ntok) {
          flag_bounds_error();
          v = 0;
        }
        src[i] = p.x + (size_t)v * p.K + c * 8;
        dst_off[i] = r * 128 + ((c ^ (r & 7)) << 4);
      }
      for (int kb = 0; kb < nk; ++kb, ++it) {
        const int s = it % STAGES;
        if (!(ok = mbar_wait(&empty[s], ((it / STAGES) & 1) ^ 1, abort_flag))) break;
        const uint32_t a_addr = smem_base + s * C::kStageBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async_16_full(a_addr + dst_off[i], src[i] + kb * kGemmBK);
        cp_async_mbar_arrive_noinc(&full[s]);  // arrives when these copies land; no wait here
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) tk_cur[i] = tk_next[i];
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing may be in flight when the CTA exits
  } else {
    // ---- epilogue ---------------------------------------------------------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tcount) {
      const G2Tile t = g2_decode(p, tile, prefix);
      const uint32_t a = tcount & 1;
      const bool ok = mbar_wait(&acc_full[a], (tcount >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      __nv_bfloat16* dst_row = nullptr;
      const int ci = t.row0 + row;
      if (ci < t.row_end) {
        const int GM = p.G * p.M;
        const int n = p.seg_tok[ci];
        const int g = (t.seg % GM) / p.M, e = t.seg % p.M;
        if (n >= 0 && n < p.ntok) {
          int j = 0;
          for (int jj = 0; jj < p.k; ++jj)
            if (p.sel[((size_t)n * p.G + g) * p.k + jj] == e) j = jj;
          dst_row = p.Q + ((size_t)n * p.Ha + g * p.k + j) * 64;
        } else {
          flag_bounds_error();
        }
      }
      const int ncols = t.nvalid;
      const uint32_t tm = tmem_base + a * BN + (static_cast<uint32_t>(q * 32) << 16);
      for (int cc = 0; cc < t.nvalid / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tm + cc * 32, r);
        if (dst_row != nullptr && cc * 32 < ncols) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          __nv_bfloat16* d = dst_row + cc * 32;
#pragma unroll
          for (int i = 0; i < 4; ++i) st_global_v4(d + i * 8, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[a]);
    }
  }

  __syncwarp();  // lanes that skipped a single-lane role wait for it, so every warp arrives whole
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * BN);
  }
}

}  // namespace gqe
