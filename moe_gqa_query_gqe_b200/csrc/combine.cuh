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
// One warp per token, 16-byte chunks; the projection y = A Wo follows as a
// tcgen05 GEMM.
#pragma once

#include "sm100.cuh"

namespace gqe {

struct CombineParams {
  const __nv_bfloat16* O;  // [N, Ha, 64]
  const float* w;          // [N, G, k]: renormalised weights (slot) or in-group probabilities (weighted)
  __nv_bfloat16* A;        // [N, (G*k + G + 1) * 64] (slot) or [N, (G*k + 1) * 64] (weighted)
  long long N;
  int G, k;
  int weighted;            // 1: A = [w-scaled concat | shared], no slot
};

__global__ void __launch_bounds__(256) combine_build_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const long long warp0 = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int Ha = p.G * p.k + 1;
  const int KA = (p.G * p.k + (p.weighted ? 0 : p.G) + 1) * 64;
  const int n_concat = p.G * p.k * 8;  // 16-byte chunks
  const int n_slot = p.weighted ? 0 : p.G * 8;
  const int n_all = KA / 8;
  for (long long n = warp0; n < p.N; n += nwarps) {
    const uint4* orow = reinterpret_cast<const uint4*>(p.O + (size_t)n * Ha * 64);
    uint4* arow = reinterpret_cast<uint4*>(p.A + (size_t)n * KA);
    for (int c = lane; c < n_all; c += 32) {
      uint4 v;
      if (c < n_concat && p.weighted) {
        // weighted concatenation: slot (g, j) scaled by its in-group probability
        const float wj = p.w[(size_t)n * p.G * p.k + (c >> 3)];
        const uint4 o = orow[c];
        const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
        uint32_t r4[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) r4[i] = pack_bf16x2(wj * bf16lo_to_f32(ou[i]), wj * bf16hi_to_f32(ou[i]));
        v = make_uint4(r4[0], r4[1], r4[2], r4[3]);
      } else if (c < n_concat) {
        v = orow[c];
      } else if (c < n_concat + n_slot) {
        const int g = (c - n_concat) >> 3, d8 = (c - n_concat) & 7;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < p.k; ++j) {
          const float wj = p.w[((size_t)n * p.G + g) * p.k + j];
          const uint4 o = orow[(g * p.k + j) * 8 + d8];
          const uint32_t ou[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[2 * i] = fmaf(wj, bf16lo_to_f32(ou[i]), acc[2 * i]);
            acc[2 * i + 1] = fmaf(wj, bf16hi_to_f32(ou[i]), acc[2 * i + 1]);
          }
        }
        v = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                       pack_bf16x2(acc[6], acc[7]));
      } else {
        v = orow[p.G * p.k * 8 + (c - n_concat - n_slot)];
      }
      arow[c] = v;
    }
  }
}

}  // namespace gqe
