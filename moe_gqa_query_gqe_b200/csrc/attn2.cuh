// attn2.cuh -- causal attention of GQE's selected experts (and of the dense
// GQA baseline), second-generation Blackwell kernel.
//
// Method: animattoys.com article on "Grouped Query Experts", section 4 (each
// selected expert computes attention on its own against the K/V shared by its
// group; the shared head is always computed); gist.science technical summary,
// "Architecture and routing" (dense, unchanged K/V).
//
// Row sets (see attn.cuh): the query rows of one KV group, rr rows per token
// (the k selected experts of the group, or all M heads in the dense baseline),
// so the routed attention of a group is causal attention with rr rows per
// position and stays balanced under any routing skew.
//
// Per CTA (persistent, one per SM), work item = two adjacent 128-row Q tiles
// (A, B) of one row set; items are visited heaviest first:
//   warp 0      TMA producer: Q_A, Q_B once per item (two item buffers, so
//               the next item's Q arrives while this one runs), K/V blocks of
//               128 positions through a STAGES-deep ring
//   warps 1, 2  lane 0 issues the MMAs of tile A (warp 1, also the TMEM owner)
//               or tile B (warp 2), per K/V block j:
//                 S_t(j+1) = Q_t K_{j+1}^T  (SS MMA, M=128 N=128 K=64)
//                 O_t     += P_t(j) V_j     (TS MMA: P read from TMEM, N=64)
//               so neither tile's pipeline waits on the other's barriers
//   warp 3      idle
//   warps 4..   softmax: S read from TMEM (then released at once so the next
//               S can be computed under this block's softmax), lazily
//               rescaled online softmax in the exp2 domain, P written back to
//               TMEM as bf16 pairs, final O / l stored as bf16. Row layout:
//               warps 4..11, one thread per row. Quad layout: warps 4..19,
//               16 rows a warp, four threads a row.
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,320) O_B [320,384)
//               P_A [384,448) P_B [448,512).
// Exponentials: MUFU ex2 delivers 16/clk/SM while each score needs 1/32 clk
// of tensor time, so one column pair in kA2PolyEvery (= 8, the best share
// measured) is evaluated on the FMA pipe instead: 2^x = 2^j * p(x - j),
// j = round(x), p a degree-3 minimax polynomial on [-1/2, 1/2] (relative
// error 7.5e-5; coefficients fitted by fit_exp2_poly.py in this directory).
#pragma once

#include "attn.cuh"
#include "sm100.cuh"

namespace gqe {

constexpr int kA2Stages = 3;
// Two softmax layouts (template parameter kQuad of attn2_fwd_kernel):
//   row layout,  384 threads: one thread per row, two softmax warps per SM
//                sub-partition, 88/208 register split after set-up
//                (88*128 + 208*256 = 168*384, the registers of the launch);
//   quad layout, 640 threads: four threads per row, four softmax warps per
//                sub-partition.
// The host takes the quad layout when every row set has one row per token
// (GQE with k = 1): there it measured as fast at 2K tokens and 4% faster at
// 32K. With two rows per token (the dense baseline's M = 2 heads, GQE with
// k = 2) the row layout measured faster from 2K to 16K and equal at 32K.
constexpr int kA2ThreadsRow = 384;
constexpr int kA2ThreadsQuad = 640;
constexpr int kA2RegsLow = 88;
constexpr int kA2RegsHigh = 208;
constexpr int kA2PolyEvery = 8;  // every n-th column pair uses the FMA-pipe exp2 (0: none)

struct Attn2Params {
  CUtensorMap tmQ[2];  // [B*T, Ha, 64] boxes (64, rr, 128/rr)
  CUtensorMap tmK;     // [B*T, G, 64] box (64, 1, 128)
  CUtensorMap tmV;
  __nv_bfloat16* O;    // [B*T, o_ld, 64]: row r of a set goes to block ob + r % rr
  // Fused output construction (GQE with k > 1): when w is set, the routed
  // sets also write each token's slot sum_j w[n,g,j] O[n,g*k+j] to block
  // slot_blk0 + g, so O is the whole operand A = [concat | slots | shared]
  // of the output projection.
  const float* w;      // [B*T, G, k] renormalised weights, or null
  int slot_blk0;       // G*k
  int G;
  int o_ld;            // 64-wide blocks per token row of O
  int B, T, Ha, nrs, npairs_max, total_items;
  float scale_log2;    // log2(e) / sqrt(dh)
  AttnRowSet rs[kMaxRowSets];
};

struct A2Smem {
  static constexpr int kQ = 0;  // two item buffers of [Q_A, Q_B], 16 KB each
  static constexpr int kK = 65536;
  static constexpr int kV = kK + kA2Stages * 16384;
  static constexpr int kBar = kV + kA2Stages * 16384;
  static constexpr int kBytes = kBar + 512 + 1024;
};

// ---- packed fp32 helpers (sm_100 f32x2 instructions) ------------------------
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                      float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair on the FMA pipe: j = round(x) by the 1.5*2^23 shift, f = x - j
// in [-1/2, 1/2], p(f) by Horner, exponent j added to p's bits. x is clamped
// at -125 so the exponent add cannot underflow (2^-125 is zero for bf16 P).
__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
  constexpr float kShift = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 9.999280572e-01f, c1 = 6.932609677e-01f, c2 = 2.426111251e-01f, c3 = 5.517166853e-02f;
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  float t0, t1, j0, j1, f0, f1, p0, p1;
  fadd2(t0, t1, x0, x1, kShift, kShift);
  fadd2(j0, j1, t0, t1, -kShift, -kShift);
  ffma2(f0, f1, j0, j1, -1.0f, -1.0f, x0, x1);
  ffma2(p0, p1, f0, f1, c3, c3, c2, c2);
  ffma2(p0, p1, p0, p1, f0, f1, c1, c1);
  ffma2(p0, p1, p0, p1, f0, f1, c0, c0);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// 32 lanes x 64 columns store of packed bf16 pairs; waits in the same block.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
      "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]),
      "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]),
      "r"(r[41]), "r"(r[42]), "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]),
      "r"(r[49]), "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]),
      "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}


// 16-lane TMEM shapes (the warp reads or writes lanes base .. base+15 of its
// quadrant). Fragment layouts, with g = lane / 4 and c = lane % 4:
//   16x256b, chunk m (8 columns): regs 4m .. 4m+3 hold (row g, col 8m+2c),
//     (g, 8m+2c+1), (g+8, 8m+2c), (g+8, 8m+2c+1);
//   16x128b, chunk m (4 columns): regs 2m, 2m+1 hold (g, 4m+c), (g+8, 4m+c).
#define GQE_R32(r)                                                                                              \
  "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),   \
      "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),     \
      "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),    \
      "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define GQE_W32(r)                                                                                              \
  "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),  \
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), \
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), \
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
#define GQE_V32 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}"
#define GQE_V32B "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32}"

// 16 lanes x 128 columns (16x256b.x16), fp32.
__device__ __forceinline__ void tmem_ld16x128f(uint32_t taddr, float (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7]), "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]), "=f"(r[14]), "=f"(r[15]), "=f"(r[16]), "=f"(r[17]), "=f"(r[18]), "=f"(r[19]), "=f"(r[20]), "=f"(r[21]), "=f"(r[22]), "=f"(r[23]), "=f"(r[24]), "=f"(r[25]), "=f"(r[26]), "=f"(r[27]), "=f"(r[28]), "=f"(r[29]), "=f"(r[30]), "=f"(r[31]), "=f"(r[32]), "=f"(r[33]), "=f"(r[34]), "=f"(r[35]), "=f"(r[36]), "=f"(r[37]), "=f"(r[38]), "=f"(r[39]), "=f"(r[40]), "=f"(r[41]), "=f"(r[42]), "=f"(r[43]), "=f"(r[44]), "=f"(r[45]), "=f"(r[46]), "=f"(r[47]), "=f"(r[48]), "=f"(r[49]), "=f"(r[50]), "=f"(r[51]), "=f"(r[52]), "=f"(r[53]), "=f"(r[54]), "=f"(r[55]), "=f"(r[56]), "=f"(r[57]), "=f"(r[58]), "=f"(r[59]), "=f"(r[60]), "=f"(r[61]), "=f"(r[62]), "=f"(r[63])
      : "r"(taddr)
      : "memory");
}
// 16 lanes x 64 columns (16x256b.x8).
__device__ __forceinline__ void tmem_ld16x64(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x8.b32 " GQE_V32 ", [%32];\n\ttcgen05.wait::ld.sync.aligned;"
               : GQE_R32(r) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_st16x64(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], " GQE_V32B ";\n\ttcgen05.wait::st.sync.aligned;"
               ::"r"(taddr), GQE_W32(r) : "memory");
}
// 16 lanes x 64 columns in the 16x128b layout (16x128b.x16).
__device__ __forceinline__ void tmem_st16x64_n(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile("tcgen05.st.sync.aligned.16x128b.x16.b32 [%0], " GQE_V32B ";\n\ttcgen05.wait::st.sync.aligned;"
               ::"r"(taddr), GQE_W32(r) : "memory");
}
#undef GQE_R32
#undef GQE_W32
#undef GQE_V32
#undef GQE_V32B

__device__ __forceinline__ void st_global_b32(void* p, uint32_t v) {
  asm volatile("st.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

struct A2Item {
  int valid;         // 0: no work for this item index
  int b, t0, tpt;    // batch, first token of tile A, tokens per tile
  int nA, nB, nmax;  // K/V blocks of tile A, tile B (0 if empty), max
  AttnRowSet rs;
};

__device__ __forceinline__ A2Item a2_decode(const Attn2Params& p, int item) {
  A2Item it;
  const int per_level = p.B * p.nrs;
  const int level = item / per_level, rem = item % per_level;
  const int rsi = rem % p.nrs;
  it.b = rem / p.nrs;
  it.rs = p.rs[rsi];
  it.tpt = 128 / it.rs.rr;
  const int npairs = (p.T + 2 * it.tpt - 1) / (2 * it.tpt);
  const int pair = npairs - 1 - level;  // heaviest pair of every row set first
  it.valid = pair >= 0;
  if (!it.valid) return it;
  it.t0 = pair * 2 * it.tpt;
  it.nA = (min(it.t0 + it.tpt, p.T) - 1) / 128 + 1;
  it.nB = (it.t0 + it.tpt < p.T) ? (min(it.t0 + 2 * it.tpt, p.T) - 1) / 128 + 1 : 0;
  it.nmax = max(it.nA, it.nB);
  return it;
}

// Static schedule over the heaviest-first item list: round r hands items
// r*G .. r*G+G-1 to the G CTAs in forward order when r is even and in reverse
// order when r is odd, so every CTA's heavy and light items pair up.
__device__ __forceinline__ int a2_item_of(int round) {
  const int g = gridDim.x;
  return round * g + ((round & 1) ? (g - 1 - (int)blockIdx.x) : (int)blockIdx.x);
}

template <bool kQuad>
__global__ void __launch_bounds__(kQuad ? kA2ThreadsQuad : kA2ThreadsRow, 1)
    attn2_fwd_kernel(const __grid_constant__ Attn2Params p) {
  constexpr int kSoftmaxPerTile = kQuad ? 256 : 128;  // softmax threads of one Q tile
  pdl_wait();
  pdl_trigger();
  using L = A2Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars + 0;                   // [2] item buffers
  uint64_t* q_empty = bars + 2;                  // [2]
  uint64_t* k_full = bars + 4;                   // [STAGES]
  uint64_t* v_full = k_full + kA2Stages;         // [STAGES]
  uint64_t* kv_empty = v_full + kA2Stages;       // [STAGES]
  uint64_t* s_full = kv_empty + kA2Stages;       // [2] (tile A, B)
  uint64_t* s_free = s_full + 2;                 // [2]
  uint64_t* p_full = s_free + 2;                 // [2]
  uint64_t* pv_done = p_full + 2;                // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int qb = 0; qb < 2; ++qb) {
      mbar_init(&q_full[qb], 1);
      mbar_init(&q_empty[qb], 2);  // one commit from each tile's MMA thread
    }
    for (int s = 0; s < kA2Stages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 2);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&s_free[t], kSoftmaxPerTile);
      mbar_init(&p_full[t], kSoftmaxPerTile);
      mbar_init(&pv_done[t], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmQ[0]);
    tma_prefetch_desc(&p.tmQ[1]);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);
  if (warp < 4) {
    if constexpr (!kQuad) setmaxnreg_dec<kA2RegsLow>();
    if (warp == 0 && lane == 0) {
      // ---- producer ------------------------------------------------------------
      uint32_t kv = 0, n_items = 0;
      bool ok = true;
      for (int round = 0, item = a2_item_of(0); ok && item < p.total_items; item = a2_item_of(++round)) {
        const A2Item it = a2_decode(p, item);
        if (!it.valid) continue;
        const int row0 = it.b * p.T;
        const int qb = n_items & 1;
        if (!(ok = mbar_wait(&q_empty[qb], ((n_items >> 1) & 1) ^ 1, abort_flag))) break;
        uint8_t* qs = smem + L::kQ + qb * 32768;
        mbar_arrive_expect_tx(&q_full[qb], it.nB > 0 ? 32768 : 16384);
        tma_load_3d(qs, &p.tmQ[it.rs.tm], &q_full[qb], 0, it.rs.h0, row0 + it.t0);
        if (it.nB > 0) tma_load_3d(qs + 16384, &p.tmQ[it.rs.tm], &q_full[qb], 0, it.rs.h0, row0 + it.t0 + it.tpt);
        for (int j = 0; j < it.nmax; ++j, ++kv) {
          const int s = kv % kA2Stages;
          if (!(ok = mbar_wait(&kv_empty[s], ((kv / kA2Stages) & 1) ^ 1, abort_flag))) break;
          mbar_arrive_expect_tx(&k_full[s], 16384);
          tma_load_3d(smem + L::kK + s * 16384, &p.tmK, &k_full[s], 0, it.rs.kvg, row0 + j * 128);
          mbar_arrive_expect_tx(&v_full[s], 16384);
          tma_load_3d(smem + L::kV + s * 16384, &p.tmV, &v_full[s], 0, it.rs.kvg, row0 + j * 128);
        }
        ++n_items;
      }
    } else if ((warp == 1 || warp == 2) && lane == 0) {
      // ---- MMA issue: warp 1 drives tile A, warp 2 tile B --------------------------
      const int t = warp - 1;
      constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_bf16(128, 64, false, true);    // P from TMEM, V MN-major
      uint32_t kv = 0, n_items = 0;
      uint32_t s_cnt = 0, pv_cnt = 0;  // issued so far by this thread
      bool ok = true;
      uint32_t qa = sbase + L::kQ + t * 16384;
      auto issue_s = [&](uint32_t kvi) -> bool {
        if (s_cnt > 0 && !mbar_wait(&s_free[t], (s_cnt - 1) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t ka = sbase + L::kK + (kvi % kA2Stages) * 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem_base + t * 128, sdesc_sw128(qa + kk * 32, 16, 1024), sdesc_sw128(ka + kk * 32, 16, 1024),
                  idesc_s, kk != 0);
        umma_commit(&s_full[t]);
        ++s_cnt;
        return true;
      };
      auto issue_pv = [&](uint32_t kvi, bool acc) -> bool {
        if (!mbar_wait(&p_full[t], pv_cnt & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t va = sbase + L::kV + (kvi % kA2Stages) * 16384;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem_base + 256 + t * 64, tmem_base + 384 + t * 64 + kk * 8, sdesc_sw128(va + kk * 2048, 8192, 1024),
                  idesc_o, (acc || kk != 0) ? 1u : 0u);
        umma_commit(&pv_done[t]);
        ++pv_cnt;
        return true;
      };
      for (int round = 0, item = a2_item_of(0); ok && item < p.total_items; item = a2_item_of(++round)) {
        const A2Item it = a2_decode(p, item);
        if (!it.valid) continue;
        const int n = t == 0 ? it.nA : it.nB;
        const int qb = n_items & 1;
        if (!(ok = mbar_wait(&q_full[qb], (n_items >> 1) & 1, abort_flag))) break;
        qa = sbase + L::kQ + qb * 32768 + t * 16384;
        const uint32_t kv0 = kv;
        if (n > 0) {
          if (!(ok = mbar_wait(&k_full[kv0 % kA2Stages], (kv0 / kA2Stages) & 1, abort_flag))) break;
          if (!(ok = issue_s(kv0))) break;
        }
        for (int j = 0; ok && j < it.nmax; ++j) {
          const uint32_t kvj = kv0 + j;
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&k_full[(kvj + 1) % kA2Stages], ((kvj + 1) / kA2Stages) & 1, abort_flag))) break;
            if (!(ok = issue_s(kvj + 1))) break;
          }
          // A block this tile does not use (j >= n) is released only after it
          // has arrived: an earlier release could complete the stage's previous
          // phase (the other tile still reading the block before it) and let
          // the producer overwrite that block.
          if (!(ok = mbar_wait(&v_full[kvj % kA2Stages], (kvj / kA2Stages) & 1, abort_flag))) break;
          if (j < n && !(ok = issue_pv(kvj, j > 0))) break;
          umma_commit(&kv_empty[kvj % kA2Stages]);  // this thread is done with block j
        }
        umma_commit(&q_empty[qb]);
        kv += it.nmax;
        ++n_items;
      }
    }
  } else if constexpr (kQuad) {
    // ---- softmax: 16 warps, four on each SM sub-partition -----------------------
    // Warp w (4..19) takes lane quadrant q = w % 4 (the TMEM lanes it may
    // access), tile t = ((w - 4) / 4) % 2 and half h = (w - 4) / 8 of the
    // quadrant: rows q*32 + h*16 .. +15 of its tile. Each row is spread over
    // four threads (16x256b fragments): thread (g, c) = (lane / 4, lane % 4)
    // holds rows g and g+8 of the warp's 16, columns 8m+2c and 8m+2c+1 of
    // every 8-column chunk m. Row maxima and sums combine over the four
    // threads by shuffles.
    const int sw = warp - 4;
    const int q = warp & 3;
    const int t = (sw >> 2) & 1;
    const int h = sw >> 3;
    const int g = lane >> 2, c4 = lane & 3;
    const int row0 = q * 32 + h * 16 + g;  // tile rows of this thread: row0, row0 + 8
    const uint32_t lane_off = static_cast<uint32_t>(q * 32 + h * 16) << 16;
    const uint32_t tm_s = tmem_base + lane_off + t * 128;
    const uint32_t tm_o = tmem_base + lane_off + 256 + t * 64;
    const uint32_t tm_p = tmem_base + lane_off + 384 + t * 64;
    const float sl2 = p.scale_log2;
    uint32_t cnt = 0;  // blocks processed by this tile so far (barrier phases)
    bool ok = true;
    for (int round = 0, item = a2_item_of(0); ok && item < p.total_items; item = a2_item_of(++round)) {
      const A2Item it = a2_decode(p, item);
      if (!it.valid) continue;
      const int nblk = t == 0 ? it.nA : it.nB;
      if (nblk == 0) continue;
      const int tfirst = it.t0 + t * it.tpt;  // first token of this tile
      const int rr = it.rs.rr;
      const int tok0 = tfirst + row0 / rr, tok1 = tfirst + (row0 + 8) / rr;  // >= T: not stored
      float m_run0 = -INFINITY, m_run1 = -INFINITY, l_run0 = 0.f, l_run1 = 0.f;
      for (int j = 0; j < nblk; ++j, ++cnt) {
        bool w_ok = mbar_wait(&s_full[t], cnt & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        float s[64];
        tmem_ld16x128f(tm_s, s);
        tc_fence_before();
        mbar_arrive(&s_free[t]);  // S may be overwritten by the next block's QK^T now

        const int kv0 = j * 128;
        if (kv0 + 127 > tfirst) {
          const int lim0 = tok0 - kv0, lim1 = tok1 - kv0;
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const int c = 8 * m + 2 * c4;
            if (c > lim0) s[4 * m] = -INFINITY;
            if (c + 1 > lim0) s[4 * m + 1] = -INFINITY;
            if (c > lim1) s[4 * m + 2] = -INFINITY;
            if (c + 1 > lim1) s[4 * m + 3] = -INFINITY;
          }
        }
        float a0 = fmaxf(s[0], s[1]), b0 = fmaxf(s[4], s[5]), a1 = fmaxf(s[2], s[3]), b1 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int m = 2; m < 16; m += 2) {
          a0 = fmax3(a0, s[4 * m], s[4 * m + 1]);
          b0 = fmax3(b0, s[4 * m + 4], s[4 * m + 5]);
          a1 = fmax3(a1, s[4 * m + 2], s[4 * m + 3]);
          b1 = fmax3(b1, s[4 * m + 6], s[4 * m + 7]);
        }
        float mx0 = fmaxf(a0, b0), mx1 = fmaxf(a1, b1);
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float m_new0 = fmaxf(m_run0, mx0 * sl2), m_new1 = fmaxf(m_run1, mx1 * sl2);
        const float m_use0 = (m_new0 > m_run0 + kRescaleThreshold) ? m_new0 : m_run0;
        const float m_use1 = (m_new1 > m_run1 + kRescaleThreshold) ? m_new1 : m_run1;
        const float alpha0 = ex2_approx(m_run0 - m_use0), alpha1 = ex2_approx(m_run1 - m_use1);
        const bool rescale = (j > 0) && (m_use0 != m_run0 || m_use1 != m_run1);
        m_run0 = m_use0;
        m_run1 = m_use1;

        // x = s * scale_log2 - m, then 2^x: MUFU for most pairs, FMA pipe for some
        float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // row 0: sm[0..3], row 1: sm[4..7]
        uint32_t pk[32];  // 16x128b layout: pk[2m] row 0, pk[2m+1] row 1, P column 4m + c4
#pragma unroll
        for (int pi = 0; pi < 32; ++pi) {
          const int m = pi >> 1, r = pi & 1;
          const float mu = r ? m_use1 : m_use0;
          float x0, x1, y0, y1;
          ffma2(x0, x1, s[4 * m + 2 * r], s[4 * m + 2 * r + 1], sl2, sl2, -mu, -mu);
          bool poly = false;
          if constexpr (kA2PolyEvery > 0) poly = (pi % kA2PolyEvery) == kA2PolyEvery - 1;
          if (poly) {
            exp2_poly2(y0, y1, x0, x1);
          } else {
            y0 = ex2_approx(x0);
            y1 = ex2_approx(x1);
          }
          const int sc = 4 * r + 2 * (m & 1);
          fadd2(sm[sc], sm[sc + 1], sm[sc], sm[sc + 1], y0, y1);
          pk[pi] = pack_bf16x2(y0, y1);
        }
        l_run0 = l_run0 * alpha0 + ((sm[0] + sm[1]) + (sm[2] + sm[3]));
        l_run1 = l_run1 * alpha1 + ((sm[4] + sm[5]) + (sm[6] + sm[7]));

        // P(j) overwrites P(j-1) and O may need rescaling: both need PV(j-1) done
        if (j > 0) {
          w_ok = mbar_wait(&pv_done[t], (cnt - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            uint32_t o[32];
            tmem_ld16x64(tm_o, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * ((i & 2) ? alpha1 : alpha0));
            tmem_st16x64(tm_o, o);
          }
        }
        tmem_st16x64_n(tm_p, pk);
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 ------------------------------------------------
      const int jslot = row0 % rr;  // row0 + 8 has the same slot (rr divides 8)
      const size_t n_tok0 = (size_t)it.b * p.T + (tok0 < p.T ? tok0 : 0);
      const size_t n_tok1 = (size_t)it.b * p.T + (tok1 < p.T ? tok1 : 0);
      // slot weights of the rows' tokens (fused output construction)
      const bool slot = p.w != nullptr && it.rs.ob < p.slot_blk0;
      float wj0[8], wj1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        wj0[i] = (slot && i < rr && tok0 < p.T) ? p.w[(n_tok0 * p.G + it.rs.kvg) * rr + i] : 0.f;
        wj1[i] = (slot && i < rr && tok1 < p.T) ? p.w[(n_tok1 * p.G + it.rs.kvg) * rr + i] : 0.f;
      }
      // row sums over the four threads of each row (the same value on all four)
      l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, 1);
      l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, 1);
      l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, 2);
      l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, 2);
      const bool w_ok = mbar_wait(&pv_done[t], (cnt - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const float inv0 = 1.f / l_run0, inv1 = 1.f / l_run1;
      uint32_t o[32];
      tmem_ld16x64(tm_o, o);
      uint32_t po[16];  // po[2m]: row 0, po[2m+1]: row 1; output columns 8m + 2*c4 and the next
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        po[2 * m] = pack_bf16x2(__uint_as_float(o[4 * m]) * inv0, __uint_as_float(o[4 * m + 1]) * inv0);
        po[2 * m + 1] = pack_bf16x2(__uint_as_float(o[4 * m + 2]) * inv1, __uint_as_float(o[4 * m + 3]) * inv1);
      }
      __nv_bfloat16* dst0 = (tok0 < p.T) ? p.O + (n_tok0 * p.o_ld + it.rs.ob + jslot) * 64 + 2 * c4 : nullptr;
      __nv_bfloat16* dst1 = (tok1 < p.T) ? p.O + (n_tok1 * p.o_ld + it.rs.ob + jslot) * 64 + 2 * c4 : nullptr;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        if (dst0) st_global_b32(dst0 + 8 * m, po[2 * m]);
        if (dst1) st_global_b32(dst1 + 8 * m, po[2 * m + 1]);
      }
      if (slot) {
        // The token's rr rows are this warp's rows g - jslot .. g - jslot + rr - 1
        // (and the same +8), held by lanes lane + 4*(i - jslot) in the same
        // register. Every one of them sums the rr bf16 outputs (fp32, in slot
        // order, as the separate combine kernel does); the first stores.
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          float acc[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) acc[c] = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (i >= rr) break;
            const int src = lane + 4 * (i - jslot);
            const float wi = r ? wj1[i] : wj0[i];
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              const uint32_t u = __shfl_sync(0xffffffffu, po[2 * m + r], src);
              acc[2 * m] = fmaf(wi, bf16lo_to_f32(u), acc[2 * m]);
              acc[2 * m + 1] = fmaf(wi, bf16hi_to_f32(u), acc[2 * m + 1]);
            }
          }
          const int tk = r ? tok1 : tok0;
          if (jslot == 0 && tk < p.T) {
            __nv_bfloat16* sd = p.O + ((r ? n_tok1 : n_tok0) * p.o_ld + p.slot_blk0 + it.rs.kvg) * 64 + 2 * c4;
#pragma unroll
            for (int m = 0; m < 8; ++m) st_global_b32(sd + 8 * m, pack_bf16x2(acc[2 * m], acc[2 * m + 1]));
          }
        }
      }
      tc_fence_before();
    }
  } else {
    setmaxnreg_inc<kA2RegsHigh>();
    // ---- softmax warpgroups: warps 4..7 -> tile A, 8..11 -> tile B --------------
    const int t = (warp - 4) >> 2;
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tm_s = tmem_base + lane_off + t * 128;
    const uint32_t tm_o = tmem_base + lane_off + 256 + t * 64;
    const uint32_t tm_p = tmem_base + lane_off + 384 + t * 64;
    const float sl2 = p.scale_log2;
    uint32_t cnt = 0;  // blocks processed by this tile so far (barrier phases)
    bool ok = true;
    for (int round = 0, item = a2_item_of(0); ok && item < p.total_items; item = a2_item_of(++round)) {
      const A2Item it = a2_decode(p, item);
      if (!it.valid) continue;
      const int nblk = t == 0 ? it.nA : it.nB;
      if (nblk == 0) continue;
      const int tfirst = it.t0 + t * it.tpt;      // first token of this tile
      const int tok = tfirst + row / it.rs.rr;    // token of this row (>= T: not stored)
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nblk; ++j, ++cnt) {
        bool w_ok = mbar_wait(&s_full[t], cnt & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        tmem_ld128f(tm_s, s);
        tc_fence_before();
        mbar_arrive(&s_free[t]);  // S may be overwritten by the next block's QK^T now

        const int kv0 = j * 128;
        if (kv0 + 127 > tfirst) {
          const int lim = tok - kv0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) s[c] = -INFINITY;
        }
        float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 128; c += 8) {
          m4[0] = fmax3(m4[0], s[c], s[c + 1]);
          m4[1] = fmax3(m4[1], s[c + 2], s[c + 3]);
          m4[2] = fmax3(m4[2], s[c + 4], s[c + 5]);
          m4[3] = fmax3(m4[3], s[c + 6], s[c + 7]);
        }
        const float mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const float m_use = (m_new > m_run + kRescaleThreshold) ? m_new : m_run;
        const float alpha = ex2_approx(m_run - m_use);
        const bool rescale = (j > 0) && (m_use != m_run);
        m_run = m_use;

        // x = s * scale_log2 - m, then 2^x: MUFU for most pairs, FMA pipe for some
        float sm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 4 independent pair chains
        uint32_t pk[64];
#pragma unroll
        for (int pi = 0; pi < 64; ++pi) {
          float x0, x1, y0, y1;
          ffma2(x0, x1, s[2 * pi], s[2 * pi + 1], sl2, sl2, -m_use, -m_use);
          bool poly = false;
          if constexpr (kA2PolyEvery > 0) poly = (pi % kA2PolyEvery) == kA2PolyEvery - 1;
          if (poly) {
            exp2_poly2(y0, y1, x0, x1);
          } else {
            y0 = ex2_approx(x0);
            y1 = ex2_approx(x1);
          }
          fadd2(sm[2 * (pi & 3)], sm[2 * (pi & 3) + 1], sm[2 * (pi & 3)], sm[2 * (pi & 3) + 1], y0, y1);
          pk[pi] = pack_bf16x2(y0, y1);
        }
        l_run = l_run * alpha + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));

        // P(j) overwrites P(j-1) and O may need rescaling: both need PV(j-1) done
        if (j > 0) {
          w_ok = mbar_wait(&pv_done[t], (cnt - 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              uint32_t o[16];
              tmem_ld16(tm_o + h * 16, o);
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st16(tm_o + h * 16, o);
            }
          }
        }
        tmem_st64(tm_p, pk);
        tc_fence_before();
        mbar_arrive(&p_full[t]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 ------------------------------------------------
      const int rr = it.rs.rr, jslot = row % rr;
      const size_t n_tok = (size_t)it.b * p.T + (tok < p.T ? tok : 0);
      // slot weights of this row's token (fused output construction)
      const bool slot = p.w != nullptr && it.rs.ob < p.slot_blk0;
      float wj[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        wj[i] = (slot && i < rr && tok < p.T) ? p.w[(n_tok * p.G + it.rs.kvg) * rr + i] : 0.f;
      const bool w_ok = mbar_wait(&pv_done[t], (cnt - 1) & 1, abort_flag);
      if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
      tc_fence_after();
      const float inv = 1.f / l_run;
      __nv_bfloat16* dst = (tok < p.T) ? p.O + (n_tok * p.o_ld + it.rs.ob + jslot) * 64 : nullptr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t o[32];
        tmem_ld32(tm_o + h * 32, o);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (dst) {
#pragma unroll
          for (int i = 0; i < 4; ++i)
            st_global_v4(dst + h * 32 + i * 8, pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
        if (slot) {
          // The token's rr rows are lanes base .. base+rr-1 of this warp.
          // Every one of them sums the rr bf16 outputs (fp32, in slot
          // order, as the separate combine kernel does); the first stores.
          const int base = lane - jslot;
          float acc[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) acc[c] = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (i >= rr) break;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t u = __shfl_sync(0xffffffffu, pk[c], base + i);
              acc[2 * c] = fmaf(wj[i], bf16lo_to_f32(u), acc[2 * c]);
              acc[2 * c + 1] = fmaf(wj[i], bf16hi_to_f32(u), acc[2 * c + 1]);
            }
          }
          if (dst && jslot == 0) {
            __nv_bfloat16* sd = p.O + (n_tok * p.o_ld + p.slot_blk0 + it.rs.kvg) * 64 + h * 32;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              st_global_v4(sd + i * 8, pack_bf16x2(acc[8 * i], acc[8 * i + 1]), pack_bf16x2(acc[8 * i + 2], acc[8 * i + 3]),
                           pack_bf16x2(acc[8 * i + 4], acc[8 * i + 5]), pack_bf16x2(acc[8 * i + 6], acc[8 * i + 7]));
          }
        }
      }
      tc_fence_before();
    }
  }

  __syncwarp();  // lanes that skipped a single-lane role wait for it, so every warp arrives whole
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
