// gemm.cuh -- tcgen05 GEMM for the GQE projections: C = A * B, bf16 in,
// fp32 accumulate in TMEM, bf16 out.
//
//   A [rows, K] row-major (K-major operand). Loaded by TMA (dense rows) or,
//     for the selected-expert query projection, gathered row by row with
//     cp.async from the token list of a segment.
//   B [K, N] row-major weight (MN-major operand), loaded by TMA in 64x64
//     boxes with the 128-byte swizzle.
//   Tile 128 x BN x 64, a STAGES-deep mbarrier ring between the producers and
//   the single MMA-issuing thread; the accumulator is read back from TMEM by
//   four epilogue warps.
//
// Warp roles (non-persistent, one output tile per CTA):
//   warp 0     : TMA producer (lane 0)
//   warp 1     : TMEM allocation + MMA issue (lane 0)
//   warps 2..5 : A gatherers during the main loop (gather mode), then the
//                epilogue (TMEM lanes 32*(warp%4) .. +31)
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;
constexpr int kMaxGemmSegs = 3;

enum GemmAMode : int { kATma = 0, kAGather = 1 };

// One output segment of a dense (TMA-A) launch: columns [b_col0, b_col0+n_cols)
// of the weight behind tmB[seg], written to C[:, c_col0 + ...] with row stride ldc.
struct GemmSeg {
  int n_cols;
  int b_col0;
  int c_col0;
  int tile_start;  // first global n-tile of this segment
  long long ldc;
  __nv_bfloat16* C;
};

struct GemmParams {
  CUtensorMap tmA;
  CUtensorMap tmB[kMaxGemmSegs];
  GemmSeg seg[kMaxGemmSegs];
  int nseg;
  int ntn;   // n-tiles over all segments
  int rows;  // rows of A / C
  int K;
  // gather mode (selected-expert query projection)
  const __nv_bfloat16* x;  // A rows source, row stride K
  const int32_t* seg_off;  // [nsegs_q + 1]
  const int32_t* seg_tok;
  const int32_t* sel;      // [B*T, G, k]
  __nv_bfloat16* Q;        // [B*T, Ha, dh]
  int nsegs_q, G, M, k, Ha;
  int ntok;  // B*T: bound of every token index read from seg_tok
};

template <int BN, int STAGES>
struct GemmSmem {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;  // 16 KB
  static constexpr int kBBytes = BN * kGemmBK * 2;       // BN/64 boxes of 8 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kBytes = kBarOffset + 256 + 1024;  // + barriers + alignment slack
};

template <int BN, int STAGES, int AMODE>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_bf16_kernel(const __grid_constant__ GemmParams p) {
  using L = GemmSmem<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  uint64_t* accum_full = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tile = const_cast<int*>(reinterpret_cast<volatile int*>(abort_flag + 1));  // [seg, mtile]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = (p.K + kGemmBK - 1) / kGemmBK;

  // ---- tile decode ------------------------------------------------------
  int m0, seg_i = 0, n0 = 0, qseg = 0, qrow0 = 0, qrow_end = 0;
  if constexpr (AMODE == kATma) {
    const int mt = blockIdx.x / p.ntn, nt = blockIdx.x % p.ntn;
    m0 = mt * kGemmBM;
    for (int s = 1; s < p.nseg; ++s)
      if (nt >= p.seg[s].tile_start) seg_i = s;
    n0 = (nt - p.seg[seg_i].tile_start) * BN;
  } else {
    // global tile index -> (segment, m-tile) by a warp scan over ceil(len/128)
    if (warp == 0) {
      int found_s = -1, found_mt = 0, before = 0;
      for (int s0 = 0; s0 < p.nsegs_q && found_s < 0; s0 += 32) {
        const int s = s0 + lane;
        const int len = s < p.nsegs_q ? p.seg_off[s + 1] - p.seg_off[s] : 0;
        const int nt = (len + kGemmBM - 1) / kGemmBM;
        int incl = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        const int lo = before + incl - nt;
        const bool mine = (int)blockIdx.x >= lo && (int)blockIdx.x < lo + nt;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        if (bal) {
          const int src = __ffs(bal) - 1;
          found_s = s0 + src;
          found_mt = (int)blockIdx.x - __shfl_sync(0xffffffffu, lo, src);
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) {
        s_tile[0] = found_s;
        s_tile[1] = found_mt;
      }
    }
    __syncthreads();
    qseg = s_tile[0];
    if (qseg < 0) return;  // beyond the last tile: uniform exit before any setup
    const int mt = s_tile[1];
    qrow0 = p.seg_off[qseg] + mt * kGemmBM;
    qrow_end = min(p.seg_off[qseg + 1], p.seg_off[p.nsegs_q]);
    m0 = mt * kGemmBM;
  }

  // ---- setup --------------------------------------------------------------
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], AMODE == kAGather ? 1 + 128 : 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, BN < 32 ? 32 : BN);
  if (warp == 0 && lane == 0) {
    if constexpr (AMODE == kATma) tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB[seg_i]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const uint32_t smem_base = smem_u32(smem);
  int b_col = 0, b_map = 0;
  if constexpr (AMODE == kATma) {
    b_col = p.seg[seg_i].b_col0 + n0;
    b_map = seg_i;
  } else {
    const int GM = p.G * p.M;
    b_col = (qseg % GM) * 64;  // head h = g*M + e of segment (b, g, e)
  }

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ---------------------------------------------------
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&empty[s], ((kb / STAGES) & 1) ^ 1, abort_flag)) break;
        uint8_t* a_s = smem + s * L::kStageBytes;
        uint8_t* b_s = a_s + L::kABytes;
        mbar_arrive_expect_tx(&full[s], (AMODE == kATma ? L::kABytes : 0) + L::kBBytes);
        if constexpr (AMODE == kATma) tma_load_2d(a_s, &p.tmA, &full[s], kb * kGemmBK, m0);
#pragma unroll
        for (int nb = 0; nb < BN / 64; ++nb)
          tma_load_2d(b_s + nb * 8192, &p.tmB[b_map], &full[s], b_col + nb * 64, kb * kGemmBK);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issue ------------------------------------------------------
      constexpr uint32_t idesc = idesc_bf16(kGemmBM, BN, false, true);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&full[s], (kb / STAGES) & 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_base + s * L::kStageBytes;
        const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b_addr + kk * 2048, 8192, 1024);
          umma_ss(tmem_base, ad, bd, idesc, (kb | kk) != 0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum_full);
    }
  } else {
    // ---- warps 2..5 ---------------------------------------------------------
    const int et = tid - 64;  // 0..127
    if constexpr (AMODE == kAGather) {
      // Gather: element chunk c (16 B) of rows r = i*16 + et/8, i = 0..7
      const int c = et & 7;
      int tok[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = i * 16 + (et >> 3);
        tok[i] = (qrow0 + r < qrow_end) ? p.seg_tok[qrow0 + r] : -1;
        if (tok[i] >= p.ntok) {
          flag_bounds_error();
          tok[i] = -1;
        }
      }
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        if (!mbar_wait(&empty[s], ((kb / STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
        const uint32_t a_addr = smem_base + s * L::kStageBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = i * 16 + (et >> 3);
          const uint32_t dst = a_addr + r * 128 + ((c ^ (r & 7)) << 4);
          const __nv_bfloat16* src = p.x + (tok[i] >= 0 ? (size_t)tok[i] * p.K + kb * kGemmBK + c * 8 : 0);
          cp_async_16(dst, src, tok[i] >= 0 ? 16u : 0u);
        }
        cp_async_commit();
        if (kb >= 1) {
          cp_async_wait<1>();
          fence_proxy_async_smem();
          mbar_arrive(&full[(kb - 1) % STAGES]);
        }
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      if (ok && nk >= 1) mbar_arrive(&full[(nk - 1) % STAGES]);
    }

    // ---- epilogue -----------------------------------------------------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool ok = mbar_wait(accum_full, 0, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      __nv_bfloat16* dst_row = nullptr;
      int ncols_valid = BN;
      if constexpr (AMODE == kATma) {
        const GemmSeg& sg = p.seg[seg_i];
        if (m0 + row < p.rows) dst_row = sg.C + (size_t)(m0 + row) * sg.ldc + sg.c_col0 + n0;
        ncols_valid = min(BN, sg.n_cols - n0);
      } else {
        const int ci = qrow0 + row;
        if (ci < qrow_end) {
          const int GM = p.G * p.M;
          const int n = p.seg_tok[ci];
          const int g = (qseg % GM) / p.M, e = qseg % p.M;
          if (n >= 0 && n < p.ntok) {
            int j = 0;
            for (int jj = 0; jj < p.k; ++jj)
              if (p.sel[((size_t)n * p.G + g) * p.k + jj] == e) j = jj;
            dst_row = p.Q + ((size_t)n * p.Ha + g * p.k + j) * 64;
          } else {
            flag_bounds_error();
          }
        }
        ncols_valid = 64;
      }
#pragma unroll
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tmem_base, q * 32, cc * 32), r);
        if (dst_row != nullptr && cc * 32 < ncols_valid) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
          __nv_bfloat16* d = dst_row + cc * 32;
#pragma unroll
          for (int i = 0; i < 4; ++i) st_global_v4(d + i * 8, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // let any copy or MMA still in flight land before the memory is released
    const unsigned long long t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000ull) {}
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, BN < 32 ? 32 : BN);
  }
}

}  // namespace gqe
