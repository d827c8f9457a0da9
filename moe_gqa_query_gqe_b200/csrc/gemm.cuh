// gemm.cuh -- parameter blocks of the tcgen05 projection GEMM (gemm2.cuh).
//
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kMaxGemmSegs = 3;

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
  CUtensorMap tmC[kMaxGemmSegs];  // CTA-pair GEMM: output of segment s, box 64 cols x 32 rows (TMA stores)
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
  // routing tiles of the CTA-pair GEMM (router logits x Wr on the tensor
  // cores, decisions in the epilogue): pair tiles r_tile0 .. r_tile0 +
  // r_B*r_nblk - 1, tile (b, blk) covering tokens [blk*256, blk*256 + 256) of
  // sequence b; r_tile0 = total tile count when there are none
  CUtensorMap tmR;     // Wr [D, G*M], 64 x 64 boxes (columns past G*M read as zero)
  int r_tile0, r_nblk;
  const float* r_br;   // [G*M] or null
  int32_t* r_sel;      // [B*T, G, k]: expert | rank in the chunk << 8 (see route.cuh)
  float* r_w;          // [B*T, G, k]
  float* r_margin;     // [B*T, G] or null
  float* r_p;          // [B*T, G, k] in-group probabilities of the selected experts, or null
  int32_t* r_counts;   // [B][nch][G*M]
  int r_B, r_T, r_nch;
  // Router merged into a dense segment's tiles instead of separate routing
  // tiles: columns 64..127 of that segment's 128-column tiles are the router
  // logits (B columns from tmR), decided in the same epilogue. Needs every
  // 128-row block to be one chunk of one sequence (T % 128 == 0). -1: none.
  int r_merge_seg;
  // A column remap for the k = 1 combine: A = [O_routed | O_routed | O_shared]
  // read straight from O ([N, (G+1)*64]); 0 disables the remap
  int amap_G;
  // Selected-query segment: this segment's columns are the routed heads
  // h = g*M + e of Wq (64 each); the epilogue writes head h's row of token n
  // to Q slot g*k + j only where sel[n, g, j] is expert e, and drops the
  // rest (sel from an earlier launch, read after the dependency wait). -1: none.
  int sel_seg;
};


}  // namespace gqe
