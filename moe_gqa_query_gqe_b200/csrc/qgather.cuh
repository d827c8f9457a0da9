// qgather.cuh -- query projection of the selected experts only (GQE step a3):
// for every segment s = (b, g, e), Q rows of the tokens that selected expert
// e of group g are x[token] * Wq[:, head g*M+e], written to token-major Q at
// slot (g, j) where j is e's rank among the token's selected experts.
//
// Method: gist.science summary of "Grouped Query Experts", "Architecture and
// routing" (query-side sparsity, dense K/V); animattoys.com article, section 4
// (each expert has its own query projection).
//
// Design (one CTA per SM, persistent, blocked tile assignment):
//   * a tile is 128 compacted rows of one segment; CTA c takes a contiguous
//     run of tiles, so its tiles mostly share one segment and thus one head;
//   * the head's whole weight slice Wq[:, h*64 .. h*64+63] (D x 64 bf16,
//     D/64 boxes of 8 KB) stays resident in shared memory and is reloaded by
//     TMA only when the segment changes;
//   * the A rows are gathered by eight copier warps with 16-byte cp.async,
//     whose completion arrives on the stage mbarrier
//     (cp.async.mbarrier.arrive.noinc); the MMA thread fences the generic to
//     async proxy before reading a stage;
//   * tcgen05 SS MMA (M=128, N=64, K=16) into a double-buffered TMEM
//     accumulator; the epilogue scatters rows to Q.
// Warps: 0 TMA (weights), 1 TMEM + MMA, 2..5 epilogue, 6..13 copiers.
#pragma once

#include "gemm.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kQgMaxStages = 12;
constexpr int kQgMinStages = 4;
constexpr int kQgThreads = 448;
constexpr int kQgMaxK = 1024;  // resident weight slice: K x 64 bf16 <= 128 KB
constexpr int kQgBarBytes = 512;

// Shared memory: `stages` A stages of 16 KB, the resident weight slice (nk
// boxes of 8 KB), barriers, the tile prefix over the segments and a copy of
// the segment offsets. As many stages as fit (the gather is bound by the
// bytes in flight).
struct QgLayout {
  int stages, nk;
  __host__ __device__ int a_off(int s) const { return s * 16384; }
  __host__ __device__ int b_off() const { return stages * 16384; }
  __host__ __device__ int bar_off() const { return b_off() + nk * 8192; }
  __host__ __device__ int prefix_off() const { return bar_off() + kQgBarBytes; }
  __host__ __device__ int segoff_off(int nsegs) const { return prefix_off() + (nsegs + 1) * 4; }
  __host__ __device__ int bytes(int nsegs) const { return segoff_off(nsegs) + (nsegs + 1) * 4 + 1024; }
};

__global__ void __launch_bounds__(kQgThreads, 1) qgather_kernel(const __grid_constant__ GemmParams p, int stages) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nk = p.K / kGemmBK;
  const QgLayout L{stages, nk};
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bar_off());  // [stages]
  uint64_t* empty = full + kQgMaxStages;                              // [stages]
  uint64_t* acc_full = empty + kQgMaxStages;                          // [2]
  uint64_t* acc_empty = acc_full + 2;                             // [2]
  uint64_t* b_full = acc_empty + 2;
  uint64_t* b_empty = b_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(b_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_prefix = reinterpret_cast<int*>(smem + L.prefix_off());
  int* s_segoff = reinterpret_cast<int*>(smem + L.segoff_off(p.nsegs_q));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int GM = p.G * p.M;

  // Segment offsets into shared memory, all loads in flight at once (the
  // copiers and the epilogue then find every tile's rows without a
  // dependent global load at the tile boundary).
  for (int s = tid; s <= p.nsegs_q; s += kQgThreads) s_segoff[s] = p.seg_off[s];
  __syncthreads();
  if (warp == 0) {
    // tile prefix over the expert segments: s_prefix[s] = tiles before segment s
    int before = 0;
    for (int s0 = 0; s0 < p.nsegs_q; s0 += 32) {
      const int s = s0 + lane;
      const int len = s < p.nsegs_q ? s_segoff[s + 1] - s_segoff[s] : 0;
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
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 256);  // one cp.async-tracked arrival per copier thread
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    mbar_init(b_full, 1);
    mbar_init(b_empty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 128);
  if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tmB[0]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  // blocked assignment: CTA c takes tiles [first, last)
  const int ntiles = s_prefix[p.nsegs_q];
  const int per = (ntiles + (int)gridDim.x - 1) / (int)gridDim.x;
  const int first = min(ntiles, (int)blockIdx.x * per), last = min(ntiles, first + per);
  auto seg_of = [&](int tile) {  // largest s with s_prefix[s] <= tile
    int lo = 0, hi = p.nsegs_q - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    return lo;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---- weight slices: loaded once per run of tiles of the same segment -------
      int cur_head = -1;
      uint32_t loads = 0;
      for (int tile = first; tile < last; ++tile) {
        const int head = seg_of(tile) % GM;
        if (head == cur_head) continue;
        if (loads > 0 && !mbar_wait(b_empty, (loads - 1) & 1, abort_flag)) break;
        mbar_arrive_expect_tx(b_full, nk * 8192);
        for (int kb = 0; kb < nk; ++kb)
          tma_load_2d(smem + L.b_off() + kb * 8192, &p.tmB[0], b_full, head * 64, kb * kGemmBK);
        cur_head = head;
        ++loads;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issue ------------------------------------------------------------
      constexpr uint32_t idesc = idesc_bf16(kGemmBM, 64, false, true);
      int cur_head = -1;
      uint32_t loads = 0, tcount = 0;
      int s = 0;
      uint32_t ph = 0;  // stage s and the parity of its current use (no division in the loop)
      bool ok = true;
      for (int tile = first; ok && tile < last; ++tile, ++tcount) {
        const int head = seg_of(tile) % GM;
        if (head != cur_head) {
          if (!(ok = mbar_wait(b_full, loads & 1, abort_flag))) break;
          cur_head = head;
          ++loads;
        }
        const uint32_t a = tcount & 1;
        if (!(ok = mbar_wait(&acc_empty[a], ((tcount >> 1) & 1) ^ 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + a * 64;
        for (int kb = 0; kb < nk; ++kb) {
          if (!(ok = mbar_wait(&full[s], ph, abort_flag))) break;
          fence_proxy_async_smem();  // rows copied by cp.async (generic proxy) feed the MMA (async proxy)
          tc_fence_after();
          const uint32_t a_addr = smem_base + L.a_off(s);
          const uint32_t b_addr = smem_base + L.b_off() + kb * 8192;
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            umma_ss(d_tmem, sdesc_sw128(a_addr + kk * 32, 16, 1024), sdesc_sw128(b_addr + kk * 2048, 8192, 1024),
                    idesc, (kb | kk) != 0);
          umma_commit(&empty[s]);
          if (++s == stages) {
            s = 0;
            ph ^= 1;
          }
        }
        umma_commit(&acc_full[a]);
        // the weight slice may be replaced once this run's last tile is issued
        if (tile + 1 >= last || seg_of(tile + 1) % GM != head) umma_commit(b_empty);
      }
    }
  } else if (warp < 6) {
    // ---- epilogue: scatter rows to token-major Q ----------------------------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint32_t tcount = 0;
    for (int tile = first; tile < last; ++tile, ++tcount) {
      const int seg = seg_of(tile);
      const int row0 = s_segoff[seg] + (tile - s_prefix[seg]) * kGemmBM;
      const int row_end = min(s_segoff[seg + 1], s_segoff[p.nsegs_q]);
      // destination row first: its dependent loads overlap the accumulation
      __nv_bfloat16* dst_row = nullptr;
      const int ci = row0 + row;
      if (ci < row_end) {
        const int n = p.seg_tok[ci];
        const int g = (seg % GM) / p.M, e = seg % p.M;
        if (n >= 0 && n < p.ntok) {
          int j = 0;
          for (int jj = 0; jj < p.k; ++jj)
            if (p.sel[((size_t)n * p.G + g) * p.k + jj] == e) j = jj;
          dst_row = p.Q + ((size_t)n * p.Ha + g * p.k + j) * 64;
        } else {
          flag_bounds_error();
        }
      }
      const uint32_t a = tcount & 1;
      const bool ok = mbar_wait(&acc_full[a], (tcount >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tm = tmem_base + a * 64 + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t r[32];
        tmem_ld32(tm + cc * 32, r);
        if (dst_row != nullptr) {
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
  } else {
    // ---- copiers (warps 6..13): 16-byte chunk c of rows r = i*32 + ct/8 ---------------
    const int ct = tid - 192;  // 0..255
    const int c = ct & 7;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    // The next tile's token rows are loaded while this tile's copies run. Rows
    // past the segment re-read its first row (their results are never
    // stored); the row index is clamped before the load and nothing reads the
    // loaded values until the tile boundary, so the loads do not stall here.
    auto fetch_rows = [&](int tile, int (&tk)[4]) {
      const int seg = seg_of(tile);
      const int row0 = s_segoff[seg] + (tile - s_prefix[seg]) * kGemmBM;
      const int row_end = min(s_segoff[seg + 1], s_segoff[p.nsegs_q]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = i * 32 + (ct >> 3);
        tk[i] = p.seg_tok[row0 + r < row_end ? row0 + r : row0];
      }
    };
    int tk_cur[4] = {0, 0, 0, 0}, tk_next[4] = {0, 0, 0, 0};
    if (first < last) fetch_rows(first, tk_cur);
    for (int tile = first; ok && tile < last; ++tile) {
      if (tile + 1 < last) fetch_rows(tile + 1, tk_next);
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
      for (int kb = 0; kb < nk; ++kb) {
        if (!(ok = mbar_wait(&empty[s], ph ^ 1, abort_flag))) break;
        const uint32_t a_addr = smem_base + L.a_off(s);
#pragma unroll
        for (int i = 0; i < 4; ++i) cp_async_16_full(a_addr + dst_off[i], src[i] + kb * kGemmBK);
        cp_async_mbar_arrive_noinc(&full[s]);  // arrives when these copies land
        if (++s == stages) {
          s = 0;
          ph ^= 1;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) tk_cur[i] = tk_next[i];
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // nothing may be in flight when the CTA exits
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
    tmem_dealloc(tmem_base, 128);
  }
}

}  // namespace gqe
