// attn.cuh -- causal attention of GQE's selected experts (and of the dense
// GQA baseline) on Blackwell tensor cores.
//
// Method: animattoys.com article on "Grouped Query Experts", section 4 (each
// selected expert computes attention on its own, against the K/V shared by its
// group; the shared head is always computed); gist.science technical summary,
// "Architecture and routing" (K/V stay dense and unchanged).
//
// Work decomposition. The query rows of one KV group form a "row set": for
// every token t there are rr rows (the k selected experts of the group, or
// all M heads in the dense baseline), stored contiguously as Q[n, h0 .. h0+rr).
// Because every token contributes exactly rr rows regardless of which experts
// it picked, the routed attention of a group is plain causal attention with rr
// query rows per position: the routing skew never unbalances this kernel.
// A CTA owns 128 consecutive rows (128/rr tokens) of one row set and streams
// the group's K/V in 128-position blocks up to the diagonal.
//
// Per CTA (192 threads, one CTA per SM):
//   warp 0     TMA: Q tile once, then K/V blocks into a STAGES-deep ring
//   warp 1     TMEM owner; lane 0 issues S_j = Q K_j^T (M=128, N=128, K=64)
//              into a double-buffered S in TMEM and O += P_j V_j (N=64, K=128)
//   warps 2..5 softmax, one thread per row: reads S_j from TMEM, online
//              softmax in the exp2 domain with a lazily updated running max
//              (O in TMEM is rescaled only when the max grows by more than
//              2^8), writes P_j (bf16) to shared memory, final O / l.
// TMEM columns: S0 [0,128), S1 [128,256), O [256,320); 512 allocated.
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kAttnStages = 3;
constexpr int kAttnThreads = 192;
constexpr int kMaxRowSets = 72;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnRowSet {
  int h0;   // first Q/O head of the set
  int rr;   // rows per token (1, 2, 4 or 8)
  int kvg;  // KV head the set attends
  int tm;   // which Q tensor map (box height rr)
};

struct AttnParams {
  CUtensorMap tmQ[2];  // [B*T, Ha, 64] boxes (64, rr, 128/rr)
  CUtensorMap tmK;     // [B*T, G, 64] box (64, 1, 128)
  CUtensorMap tmV;
  __nv_bfloat16* O;    // [B*T, Ha, 64]
  int B, T, Ha, nrs, nqt_max;
  float scale_log2;    // log2(e) / sqrt(dh)
  AttnRowSet rs[kMaxRowSets];
};

struct AttnSmem {
  static constexpr int kQ = 0;
  static constexpr int kK = 16384;
  static constexpr int kV = kK + kAttnStages * 16384;
  static constexpr int kP = kV + kAttnStages * 16384;
  static constexpr int kBar = kP + 32768;
  static constexpr int kBytes = kBar + 256 + 1024;
};

__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  using L = AttnSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                     // [STAGES]
  uint64_t* v_full = k_full + kAttnStages;         // [STAGES]
  uint64_t* kv_empty = v_full + kAttnStages;       // [STAGES]
  uint64_t* s_full = kv_empty + kAttnStages;       // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- tile decode (heaviest tiles first: blockIdx.y counts from the end) ---
  const int rsi = blockIdx.x % p.nrs;
  const int b = blockIdx.x / p.nrs;
  const AttnRowSet rs = p.rs[rsi];
  const int tpt = 128 / rs.rr;                     // tokens per tile
  const int nqt = (p.T + tpt - 1) / tpt;
  const int qt = nqt - 1 - (int)blockIdx.y;
  if (qt < 0) return;
  const int t0 = qt * tpt;
  const int t_last = min(t0 + tpt, p.T) - 1;
  const int nblk = t_last / 128 + 1;
  const int row_base = b * p.T;                    // flat token of t = 0

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmQ[rs.tm]);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ---- producer ----------------------------------------------------------
      mbar_arrive_expect_tx(q_full, 16384);
      tma_load_3d(smem + L::kQ, &p.tmQ[rs.tm], q_full, 0, rs.h0, row_base + t0);
      for (int j = 0; j < nblk; ++j) {
        const int s = j % kAttnStages;
        if (!mbar_wait(&kv_empty[s], ((j / kAttnStages) & 1) ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(&k_full[s], 16384);
        tma_load_3d(smem + L::kK + s * 16384, &p.tmK, &k_full[s], 0, rs.kvg, row_base + j * 128);
        mbar_arrive_expect_tx(&v_full[s], 16384);
        tma_load_3d(smem + L::kV + s * 16384, &p.tmV, &v_full[s], 0, rs.kvg, row_base + j * 128);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issue ---------------------------------------------------------
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_bf16(128, 64, false, true);    // P K-major, V MN-major
      const uint32_t tm_s[2] = {tmem_base, tmem_base + 128};
      const uint32_t tm_o = tmem_base + 256;
      auto issue_s = [&](int j) {
        const int s = j % kAttnStages;
        const uint32_t qa = sbase + L::kQ, ka = sbase + L::kK + s * 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tm_s[j & 1], sdesc_sw128(qa + kk * 32, 16, 1024), sdesc_sw128(ka + kk * 32, 16, 1024), idesc_s,
                  kk != 0);
        umma_commit(&s_full[j & 1]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&k_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; ok && j < nblk; ++j) {
        if (j + 1 < nblk) {
          const int s1 = (j + 1) % kAttnStages;
          if (!(ok = mbar_wait(&k_full[s1], ((j + 1) / kAttnStages) & 1, abort_flag))) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        const int s = j % kAttnStages;
        if (!(ok = mbar_wait(p_full, j & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&v_full[s], (j / kAttnStages) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t pa = sbase + L::kP, va = sbase + L::kV + s * 16384;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tm_o, sdesc_sw128(pa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(va + kk * 2048, 8192, 1024), idesc_o, (j | kk) != 0);
        umma_commit(pv_done);
        umma_commit(&kv_empty[s]);
      }
    }
  } else {
    // ---- softmax: one thread per row ------------------------------------------
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int tok = t0 + row / rs.rr;          // token of this row (may be >= T: not stored)
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[128];
      {
        uint32_t r[64];
        tmem_ld64(tmem_base + lane_off + (j & 1) * 128, r);
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(r[i]);
        tmem_ld64(tmem_base + lane_off + (j & 1) * 128 + 64, r);
#pragma unroll
        for (int i = 0; i < 64; ++i) s[64 + i] = __uint_as_float(r[i]);
      }
      const int kv0 = j * 128;
      if (kv0 + 127 > t0) {
        const int lim = tok - kv0;  // columns c > lim are in the future
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c > lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      const float m_use = (m_new > m_run + kRescaleThreshold) ? m_new : m_run;
      const float alpha = ex2_approx(m_run - m_use);  // 0 on the first block, 1 when unchanged
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        s[c] = ex2_approx(fmaf(s[c], sl2, -m_use));
        sum += s[c];
      }
      l_run = l_run * alpha + sum;
      const bool rescale = (j > 0) && (m_use != m_run);
      m_run = m_use;
      tc_fence_before();

      if (j > 0) {
        ok = mbar_wait(pv_done, (j - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale)) {
          uint32_t o[32];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tmem_ld32(tmem_base + lane_off + 256 + h * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem_base + lane_off + 256 + h * 32, o);
          }
        }
      }
      // P (bf16) -> shared memory, K-major 128B-swizzled, two 64-column halves
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t prow = sbase + L::kP + h * 16384 + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const int c = h * 64 + ch * 8;
          st_shared_v4(prow + ((ch ^ (row & 7)) << 4), pack_bf16x2(s[c], s[c + 1]), pack_bf16x2(s[c + 2], s[c + 3]),
                       pack_bf16x2(s[c + 4], s[c + 5]), pack_bf16x2(s[c + 6], s[c + 7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok) {
      ok = mbar_wait(pv_done, (nblk - 1) & 1, abort_flag);
      if (__all_sync(0xffffffffu, ok)) {
        tc_fence_after();
        const float inv = 1.f / l_run;
        __nv_bfloat16* dst = (tok < p.T)
            ? p.O + ((size_t)(row_base + tok) * p.Ha + rs.h0 + (row % rs.rr)) * 64
            : nullptr;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t o[32];
          tmem_ld32(tmem_base + lane_off + 256 + h * 32, o);
          if (dst) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_global_v4(dst + h * 32 + i * 8, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    const unsigned long long t0n = globaltimer_ns();
    while (globaltimer_ns() - t0n < 100000ull) {}
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace gqe
