// combine.cuh -- GQE output construction before the output projection.
//
// Method: gist.science technical summary of "Grouped Query Experts",
// "Architecture and routing", output construction: the hard concatenation of
// the selected experts' outputs, a renormalised weighted sum of them (router
// probabilities renormalised over the selected set), and the always-on shared
// head; animattoys.com article, section 4: the three parts are merged and then
// passed through the final output projection.
//
//   A[n] = [ O[n, 0 .. G*k-1]                 (concat, slot order = ascending expert)
//          | sum_j w[n,g,j] * O[n, g*k+j]  for g = 0..G-1   (fp32 sum, one slot per group)
//          | O[n, G*k] ]                       (shared head)
// and the variants of that construction (the ablation of the animattoys.com
// article, section 6, and of the gist.science summary, "Experimental
// results"; the single-slot reading of the article's section 4):
//   weighted concatenation  [ p[n,g,j] * O[n, g*k+j] | shared ]
//   one global slot         [ concat | sum_{g,j} p[n,g,j] O[n,g*k+j] / sum_{g,j} p[n,g,j] | shared ]
//   no shared head          [ concat | per-group slots ]
// with p the in-group probabilities of the selected experts.
// One warp per token, 16-byte chunks; the projection y = A Wo follows as a
// tcgen05 GEMM.
#pragma once

#include "sm100.cuh"

namespace gqe {

enum CombineSlots : int { kNoSlot = 0, kSlotPerGroup = 1, kGlobalSlot = 2 };

struct CombineParams {
  const __nv_bfloat16* O;  // [N, Ha, 64]
  const float* w;          // [N, G, k]: renormalised weights (per-group slots) or in-group probabilities
  __nv_bfloat16* A;        // [N, KA], KA = (G*k + slot blocks + shared) * 64
  long long N;
  int G, k;
  int scale_concat;        // 1: each concatenated output scaled by its w
  int slots;               // CombineSlots
  int shared;              // 1: the shared head's output is A's last block
};

__host__ __device__ inline int combine_slot_blocks(int G, int slots) {
  return slots == kSlotPerGroup ? G : (slots == kGlobalSlot ? 1 : 0);
}

__global__ void __launch_bounds__(256) combine_build_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int Ha = p.G * p.k + 1;
  const int Gk = p.G * p.k;
  const int n_concat = Gk * 8;  // 16-byte chunks
  const int n_slot = combine_slot_blocks(p.G, p.slots) * 8;
  const int n_all = n_concat + n_slot + (p.shared ? 8 : 0);
  for (long long n = warp0; n < p.N; n += nwarps) {
    const uint4* orow = reinterpret_cast<const uint4*>(p.O + (size_t)n * Ha * 64);
    uint4* arow = reinterpret_cast<uint4*>(p.A + (size_t)n * n_all * 8);
    const float* wrow = p.w + (size_t)n * Gk;
    for (int c = lane; c < n_all; c += 32) {
      uint4 v;
      if (c < n_concat && p.scale_concat) {
        // weighted concatenation: slot (g, j) scaled by its weight
        const float wj = wrow[c >> 3];
        const uint4 o = orow[c];
        const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
        uint32_t r4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) r4[i] = pack_bf16x2(wj * bf16lo_to_f32(ou[i]), wj * bf16hi_to_f32(ou[i]));
        v = make_uint4(r4[0], r4[1], r4[2], r4[3]);
      } else if (c < n_concat) {
        v = orow[c];
      } else if (c < n_concat + n_slot) {
        // per-group slot g: its k outputs; global slot: all G*k outputs,
        // divided by the sum of their weights
        const int d8 = (c - n_concat) & 7;
        const int i0 = p.slots == kGlobalSlot ? 0 : ((c - n_concat) >> 3) * p.k;
        const int i1 = p.slots == kGlobalSlot ? Gk : i0 + p.k;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        float wsum = 0.f;
        for (int i = i0; i < i1; ++i) {
          const float wi = wrow[i];
          const uint4 o = orow[i * 8 + d8];
          const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
          wsum += wi;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(wi, bf16lo_to_f32(ou[e]), acc[2 * e]);
            acc[2 * e + 1] = fmaf(wi, bf16hi_to_f32(ou[e]), acc[2 * e + 1]);
          }
        }
        if (p.slots == kGlobalSlot) {
          const float inv = 1.0f / wsum;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] *= inv;
        }
        v = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
      } else {
        v = orow[n_concat + (c - n_concat - n_slot)];  // the shared head, O's last block
      }
      arow[c] = v;
    }
  }
}

}  // namespace gqe
