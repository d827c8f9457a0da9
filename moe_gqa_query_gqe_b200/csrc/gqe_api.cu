// gqe_api.cu -- the C ABI of libgqe (declared in include/gqe.h): argument
// validation, TMA tensor-map construction, workspace carving and kernel
// launches for the GQE forward pass and the dense GQA baseline. Every step of
// the computation runs in the kernels of this translation unit.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include "gqe.h"
#include "sm100.cuh"
#include "route.cuh"
#include "gemm.cuh"
#include "gemm2.cuh"
#include "gemm2sm.cuh"
#include "qgather.cuh"
#include "attn.cuh"
#include "attn2.cuh"
#include "combine.cuh"
#include "decode.cuh"
#include "decode_proj.cuh"

using namespace gqe;

namespace {

inline bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }
inline long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_dims(const gqe_dims* d) {
  if (d == nullptr) return GQE_ERR_INVALID_ARG;
  if (d->B < 1 || d->T < 1 || d->D < 1 || d->G < 1 || d->M < 1 || d->k < 1 || d->dh < 1) return GQE_ERR_INVALID_ARG;
  if (d->k > d->M) return GQE_ERR_INVALID_ARG;
  if (d->dh != 64) return GQE_ERR_UNSUPPORTED;
  if (d->D % 64 != 0) return GQE_ERR_UNSUPPORTED;
  const int GM = d->G * d->M;
  // 8 <= G*M: the router weight's rows must be a multiple of 16 bytes for TMA
  if (GM < 8 || GM > 64 || !pow2(GM)) return GQE_ERR_UNSUPPORTED;
  if (!pow2(d->M) || d->M > 8 || !pow2(d->k) || d->k > 8) return GQE_ERR_UNSUPPORTED;
  if ((long long)d->B * GM > 8192) return GQE_ERR_UNSUPPORTED;
  const long long N = (long long)d->B * d->T;
  if (N * d->G * d->k >= (1ll << 31) || N * (d->G * d->M + 1) >= (1ll << 31)) return GQE_ERR_UNSUPPORTED;
  return GQE_OK;
}

// ---------------------------------------------------------------------------
// TMA tensor maps (driver entry point fetched through the runtime)
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor, 128-byte swizzle; dims/strides innermost first; strides in bytes
// for dims 1..rank-1.
int make_tmap(CUtensorMap* tm, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return GQE_ERR_CUDA;
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides[i];
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), gd, gs, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GQE_OK : GQE_ERR_CUDA;
}

// row-major [rows, cols] bf16 with row stride ld (elements); box 64 cols x box_rows
int tmap_rows(CUtensorMap* tm, const void* base, long long rows, long long cols, long long ld, int box_rows) {
  const uint64_t dims[2] = {(uint64_t)cols, (uint64_t)rows};
  const uint64_t strides[1] = {(uint64_t)ld * 2};
  const uint32_t box[2] = {64, (uint32_t)box_rows};
  return make_tmap(tm, base, 2, dims, strides, box);
}

// [N, H, 64] bf16; box (64, bh, bn)
int tmap_heads(CUtensorMap* tm, const void* base, long long N, int H, int bh, int bn) {
  const uint64_t dims[3] = {64, (uint64_t)H, (uint64_t)N};
  const uint64_t strides[2] = {128, (uint64_t)H * 128};
  const uint32_t box[3] = {64, (uint32_t)bh, (uint32_t)bn};
  return make_tmap(tm, base, 3, dims, strides, box);
}

// ---------------------------------------------------------------------------
// Launch helpers
// ---------------------------------------------------------------------------
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GQE_OK;
  g_last_cuda_error = e;
  return GQE_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream is still finishing (every kernel of
// the library waits on it with griddepcontrol.wait before touching memory).
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...));
}

template <typename K>
int set_smem(K kernel, int bytes) {
  // cheap after the first call on a device; keeps multi-device use correct
  return cuda_status(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
}


constexpr int kG2DenseBN = kPairBN;
constexpr int kG2GatherStages = 8;

int sm_count();

template <int BN, int STAGES>
int launch_gemm2(const GemmParams& p, long long tiles, cudaStream_t st) {
  using C = G2Cfg<BN, STAGES>;
  auto kern = gemm2_kernel<BN, STAGES>;
  const int smem = C::kBytesBase + (p.nsegs_q + 1) * 4;
  if (int e = set_smem(kern, smem)) return e;
  if (tiles <= 0) return GQE_OK;
  if (tiles > 0x7fffffffll) return GQE_ERR_UNSUPPORTED;
  const int grid = (int)std::min<long long>(tiles, sm_count());
  return launch_pdl(kern, dim3(grid), dim3(C::kThreads), smem, st, p, (int)tiles);
}

// Clusters of two CTAs that can be resident at once for a kernel launched with
// `threads` threads and `smem` bytes of dynamic shared memory (a pair needs two
// free SMs of one GPC, so this can be below half the SM count). Kernels with a
// blocked work split must not launch more pairs than this, or the surplus
// would run as a second wave.
template <typename K>
int max_resident_pairs(K kernel, int threads, int smem) {
  struct Entry {
    const void* fn;
    int dev, threads, smem, pairs;
  };
  static std::mutex mu;
  static Entry cache[32];
  static int ncache = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return sm_count() / 2;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < ncache; ++i)
    if (cache[i].fn == (const void*)kernel && cache[i].dev == dev && cache[i].threads == threads &&
        cache[i].smem == smem)
      return cache[i].pairs;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * 1024, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = sm_count() / 2;
  }
  if (ncache < 32) cache[ncache++] = Entry{(const void*)kernel, dev, threads, smem, n};
  return n;
}

int launch_gemm_pair(const GemmParams& p, long long tiles, cudaStream_t st) {
  if (int e = set_smem(gemm_pair_kernel, PairSmem::kBytes)) return e;
  if (tiles <= 0) return GQE_OK;
  if (tiles > 0x7fffffffll) return GQE_ERR_UNSUPPORTED;
  const int pairs = (int)std::min<long long>(tiles, max_resident_pairs(gemm_pair_kernel, kPairThreads, PairSmem::kBytes));
  return launch_pdl(gemm_pair_kernel, dim3(2 * pairs), dim3(kPairThreads), PairSmem::kBytes, st, p, (int)tiles);
}

// Dense multi-segment projection: A [rows, K] times up to three weights.
struct DenseSeg {
  const void* W;     // [K, w_cols]
  int w_cols;        // columns of the weight tensor
  int b_col0;        // first column used
  int n_cols;        // columns used
  void* C;
  long long ldc;
  int c_col0;
};

// Pair-GEMM parameters of a dense multi-segment projection; returns the
// number of pair tiles (no routing tiles yet).
int dense_params(GemmParams& p, const void* A, long long rows, int K, const DenseSeg* segs, int nseg, long long* tiles) {
  memset(&p, 0, sizeof(p));
  if (int e = tmap_rows(&p.tmA, A, rows, K, K, kGemmBM)) return e;
  int nt = 0;
  for (int s = 0; s < nseg; ++s) {
    if (int e = tmap_rows(&p.tmB[s], segs[s].W, K, segs[s].w_cols, segs[s].w_cols, 64)) return e;
    if (int e = tmap_rows(&p.tmC[s], segs[s].C, rows, segs[s].ldc, segs[s].ldc, 32)) return e;
    p.seg[s].n_cols = segs[s].n_cols;
    p.seg[s].b_col0 = segs[s].b_col0;
    p.seg[s].c_col0 = segs[s].c_col0;
    p.seg[s].ldc = segs[s].ldc;
    p.seg[s].C = static_cast<__nv_bfloat16*>(segs[s].C);
    p.seg[s].tile_start = nt;
    nt += (int)cdiv(segs[s].n_cols, kG2DenseBN);
  }
  p.nseg = nseg;
  p.ntn = nt;
  p.rows = (int)rows;
  p.K = K;
  *tiles = nt > 0 ? cdiv(rows, kPairBM) * nt : 0;
  p.r_tile0 = 0x7fffffff;
  p.r_merge_seg = -1;
  p.sel_seg = -1;
  return GQE_OK;
}

int gemm_dense(const void* A, long long rows, int K, const DenseSeg* segs, int nseg, cudaStream_t st) {
  GemmParams p;
  long long tiles = 0;
  if (int e = dense_params(p, A, rows, K, segs, nseg, &tiles)) return e;
  return launch_gemm_pair(p, tiles, st);
}

// ---------------------------------------------------------------------------
// Workspace carving
// ---------------------------------------------------------------------------
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off = align256(off + count * sizeof(T));
    return p;
  }
};

struct RouteWs {
  int32_t* counts;
  int32_t* chunk_base;
};
RouteWs carve_route(Carver& c, const gqe_dims* d) {
  const long long nch = cdiv(d->T, kRouteChunk);
  const size_t n = (size_t)d->B * nch * d->G * d->M;
  RouteWs r;
  r.counts = c.take<int32_t>(n);
  r.chunk_base = c.take<int32_t>(n);
  return r;
}

struct FwdWs {
  int32_t *sel, *seg_off, *seg_tok, *row_map;
  float *w, *margin;
  RouteWs route;
  __nv_bfloat16 *Q, *K, *V, *O, *A;
};
FwdWs carve_forward(Carver& c, const gqe_dims* d) {
  const size_t N = (size_t)d->B * d->T;
  const int Ha = d->G * d->k + 1;
  FwdWs f;
  f.sel = c.take<int32_t>(N * d->G * d->k);
  f.w = c.take<float>(N * d->G * d->k);
  f.margin = c.take<float>(N * d->G);
  f.seg_off = c.take<int32_t>((size_t)d->B * d->G * d->M + 1);
  f.seg_tok = c.take<int32_t>(N * d->G * d->k);
  f.row_map = c.take<int32_t>(N * d->G * d->k);
  f.route = carve_route(c, d);
  f.Q = c.take<__nv_bfloat16>(N * Ha * 64);
  f.K = c.take<__nv_bfloat16>(N * d->G * 64);
  f.V = c.take<__nv_bfloat16>(N * d->G * 64);
  f.O = c.take<__nv_bfloat16>(N * Ha * 64);
  f.A = c.take<__nv_bfloat16>(d->k == 1 ? 0 : N * (size_t)(d->G * d->k + d->G + 1) * 64);
  return f;
}

// Columns of A, i.e. rows of Wo, for an output construction (gqe_combine_mode).
int combine_cols(const gqe_dims* d, int mode) {
  const int Gk = d->G * d->k;
  switch (mode) {
    case GQE_COMBINE_SLOT: return (Gk + d->G + 1) * 64;
    case GQE_COMBINE_HARD:
    case GQE_COMBINE_WEIGHTED: return (Gk + 1) * 64;
    case GQE_COMBINE_GLOBAL_SLOT: return (Gk + 2) * 64;
    case GQE_COMBINE_NO_SHARED: return (Gk + d->G) * 64;
    default: return 0;
  }
}

// The widest A among the variants other than GQE_COMBINE_SLOT (workspace of
// gqe_forward_variant).
int variant_max_cols(const gqe_dims* d) {
  int c = 0;
  for (int m = GQE_COMBINE_HARD; m <= GQE_COMBINE_NO_SHARED; ++m) c = std::max(c, combine_cols(d, m));
  return c;
}

size_t combine_ws_bytes(const gqe_dims* d) {
  if (d->k == 1) return 0;  // A is read straight from O (see do_combine)
  return align256((size_t)d->B * d->T * combine_cols(d, GQE_COMBINE_SLOT) * 2);
}

struct DenseWs {
  __nv_bfloat16 *Q, *K, *V, *O;
};
DenseWs carve_dense(Carver& c, const gqe_dims* d) {
  const size_t N = (size_t)d->B * d->T;
  DenseWs w;
  w.Q = c.take<__nv_bfloat16>(N * d->G * d->M * 64);
  w.K = c.take<__nv_bfloat16>(N * d->G * 64);
  w.V = c.take<__nv_bfloat16>(N * d->G * 64);
  w.O = c.take<__nv_bfloat16>(N * d->G * d->M * 64);
  return w;
}

int check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return GQE_OK;
  if (ws == nullptr || ws_bytes < need) return GQE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255) != 0) return GQE_ERR_WORKSPACE;
  return GQE_OK;
}

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQE_ERR_NO_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return GQE_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return GQE_ERR_NO_DEVICE;
  return (major == 10 && minor == 0) ? GQE_OK : GQE_ERR_NO_DEVICE;
}

#define GQE_TRY(expr)          \
  do {                         \
    const int _e = (expr);     \
    if (_e != GQE_OK) return _e; \
  } while (0)

// ---------------------------------------------------------------------------
// Stage implementations (arguments already validated)
// ---------------------------------------------------------------------------
// Routing tiles (router logits and decisions, gemm2sm.cuh) appended to the
// pair-GEMM launch `p` over x, starting at pair tile `tile0`; returns in
// *tiles the number added. p.tmA must already map x with 128-row boxes.
int add_route_tiles(GemmParams& p, const gqe_dims* d, const void* Wr, const float* br, int32_t* sel, float* w,
                    float* margin, RouteWs rw, long long tile0, long long* tiles) {
  const int GM = d->G * d->M;
  GQE_TRY(tmap_rows(&p.tmR, Wr, d->D, GM, GM, 64));  // 64-wide box: columns past G*M read as zero
  p.K = d->D;
  p.G = d->G;
  p.M = d->M;
  p.k = d->k;
  p.r_br = br;
  p.r_sel = sel;
  p.r_w = w;
  p.r_margin = margin;
  p.r_counts = rw.counts;
  p.r_B = d->B;
  p.r_T = d->T;
  p.r_nch = (int)cdiv(d->T, kRouteChunk);
  p.r_nblk = (int)cdiv(d->T, kPairBM);
  p.r_tile0 = (int)tile0;
  *tiles = (long long)d->B * p.r_nblk;
  return tile0 + *tiles > 0x7fffffffll ? GQE_ERR_UNSUPPORTED : GQE_OK;
}

// After the routing tiles: segment offsets, chunk bases, compacted lists.
int route_finish(const gqe_dims* d, int32_t* sel, int32_t* seg_off, int32_t* seg_tok, int32_t* row_map, RouteWs rw,
                 cudaStream_t st) {
  RouteParams rp;
  rp.sel = sel;
  rp.counts = rw.counts;
  rp.chunk_base = rw.chunk_base;
  rp.seg_off = seg_off;
  rp.seg_tok = seg_tok;
  rp.row_map = row_map;
  rp.B = d->B;
  rp.T = d->T;
  rp.G = d->G;
  rp.M = d->M;
  rp.k = d->k;
  rp.nch = (int)cdiv(d->T, kRouteChunk);
  const int nseg = d->B * d->G * d->M;
  const long long rows = (long long)d->B * d->T * d->G * d->k;
  const long long blocks = std::min<long long>(cdiv(rows, 256), (long long)sm_count() * 8);
  const long long ncnt = (long long)nseg * rp.nch;
  if (ncnt <= kRouteFusedMax) {
    // counts small enough for every block to scan them itself: one launch,
    // one block per SM (each block scans once, then places its share)
    const int smem = (int)(ncnt + nseg + 1) * 4;
    const long long fblocks = std::min<long long>(cdiv(rows, 256), (long long)sm_count());
    return launch_pdl(route_scan_finalize_kernel, dim3((unsigned)std::max<long long>(fblocks, 1)), dim3(1024), smem,
                      st, rp);
  }
  GQE_TRY(launch_pdl(route_scan_kernel, dim3(1), dim3(1024), nseg * 4, st, rp));
  return launch_pdl(route_finalize_kernel, dim3((unsigned)std::max<long long>(blocks, 1)), dim3(256), 0, st, rp);
}

int do_route(const gqe_dims* d, const void* x, const void* Wr, const float* br, int32_t* sel, float* w,
             float* margin, int32_t* seg_off, int32_t* seg_tok, int32_t* row_map, RouteWs rw, cudaStream_t st) {
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.r_merge_seg = -1;
  p.sel_seg = -1;
  const long long N = (long long)d->B * d->T;
  GQE_TRY(tmap_rows(&p.tmA, x, N, d->D, d->D, kGemmBM));
  p.rows = (int)N;
  long long tiles = 0;
  GQE_TRY(add_route_tiles(p, d, Wr, br, sel, w, margin, rw, 0, &tiles));
  GQE_TRY(launch_gemm_pair(p, tiles, st));
  return route_finish(d, sel, seg_off, seg_tok, row_map, rw, st);
}

// The dense part of the query/key/value projections, one launch over x: K,
// V and the shared head's query.
void kv_segments(const gqe_dims* d, const void* Wq, const void* Wk, const void* Wv, void* Q, void* K, void* V,
                 DenseSeg (&segs)[3]) {
  const int G = d->G, M = d->M, k = d->k, Ha = G * k + 1;
  const int wq_cols = (G * M + 1) * 64;
  segs[0] = DenseSeg{Wk, G * 64, 0, G * 64, K, (long long)G * 64, 0};
  segs[1] = DenseSeg{Wv, G * 64, 0, G * 64, V, (long long)G * 64, 0};
  segs[2] = DenseSeg{Wq, wq_cols, G * M * 64, 64, Q, (long long)Ha * 64, G * k * 64};
}

// The selected queries of gqe_forward as one dense product over every
// routed head (Wq columns 0 .. G*M*64), whose epilogue keeps each token's
// selected experts' rows (gemm2sm.cuh, selected-query segment). Chosen when
// M <= 2k: the tensor-core work on the unselected heads (at most as much
// again) then costs less than gathering every (token, group)'s row of x per
// expert, which the gather kernel is bound by. The results are the same
// products, accumulated in the same order.
bool qproj_dense_select(const gqe_dims* d) { return d->M <= 2 * d->k; }

int do_qselect(const gqe_dims* d, const void* x, const void* Wq, const int32_t* sel, void* Q, cudaStream_t st) {
  const int G = d->G, M = d->M, k = d->k, Ha = G * k + 1;
  const int wq_cols = (G * M + 1) * 64;
  const DenseSeg seg = {Wq, wq_cols, 0, G * M * 64, Q, (long long)Ha * 64, 0};
  GemmParams p;
  long long tiles = 0;
  GQE_TRY(dense_params(p, x, (long long)d->B * d->T, d->D, &seg, 1, &tiles));
  p.sel_seg = 0;
  p.sel = sel;
  p.Q = static_cast<__nv_bfloat16*>(Q);
  p.G = G;
  p.M = M;
  p.k = k;
  p.Ha = Ha;
  return launch_gemm_pair(p, tiles, st);
}

// Selected experts: one segment per (b, g, e), rows gathered by seg_tok.
int do_qgather(const gqe_dims* d, const void* x, const void* Wq, const int32_t* sel, const int32_t* seg_off,
               const int32_t* seg_tok, void* Q, cudaStream_t st) {
  const long long N = (long long)d->B * d->T;
  const int G = d->G, M = d->M, k = d->k, Ha = G * k + 1;
  const int wq_cols = (G * M + 1) * 64;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.r_merge_seg = -1;
  p.sel_seg = -1;
  GQE_TRY(tmap_rows(&p.tmB[0], Wq, d->D, wq_cols, wq_cols, 64));
  GQE_TRY(tmap_rows(&p.tmA, x, N, d->D, d->D, 1));  // a valid map for the kernel's descriptor prefetch (rows are copied with cp.async)
  p.K = d->D;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.seg_off = seg_off;
  p.seg_tok = seg_tok;
  p.sel = sel;
  p.Q = static_cast<__nv_bfloat16*>(Q);
  p.nsegs_q = d->B * G * M;
  p.G = G;
  p.M = M;
  p.k = k;
  p.Ha = Ha;
  p.ntok = (int)N;
  const long long tiles_max = cdiv(N * G * k, kGemmBM) + p.nsegs_q;
  const int nk = d->D / kGemmBK;
  const int qg_stages = std::min(kQgMaxStages, (232448 - QgLayout{0, nk}.bytes(p.nsegs_q)) / 16384);
  if (d->D <= kQgMaxK && d->D % kGemmBK == 0 && qg_stages >= kQgMinStages) {
    // the head's weight slice stays resident in shared memory
    const int qg_smem = QgLayout{qg_stages, nk}.bytes(p.nsegs_q);
    GQE_TRY(set_smem(qgather_kernel, qg_smem));
    const int grid = (int)std::min<long long>(tiles_max, sm_count());
    return launch_pdl(qgather_kernel, dim3(grid), dim3(kQgThreads), qg_smem, st, p, qg_stages);
  }
  return launch_gemm2<64, kG2GatherStages>(p, tiles_max, st);
}

int do_qproj(const gqe_dims* d, const void* x, const void* Wq, const void* Wk, const void* Wv, const int32_t* sel,
             const int32_t* seg_off, const int32_t* seg_tok, void* Q, void* K, void* V, cudaStream_t st) {
  DenseSeg segs[3];
  kv_segments(d, Wq, Wk, Wv, Q, K, V, segs);
  GQE_TRY(gemm_dense(x, (long long)d->B * d->T, d->D, segs, 3, st));
  return do_qgather(d, x, Wq, sel, seg_off, seg_tok, Q, st);
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// Persistent two-tile attention (attn2.cuh). With slot_w set (GQE, k > 1),
// O is the output projection's operand A [N, G*k + G + 1, 64]: the routed
// rows in their concatenation blocks, each token's per-group slot (weights
// slot_w) in blocks G*k .. G*k+G-1, the shared head in the last block.
int do_attn2(const gqe_dims* d, const void* Q, int Hq, const void* K, const void* V, void* O, bool dense,
             bool shared, cudaStream_t st, const float* slot_w = nullptr) {
  const long long N = (long long)d->B * d->T;
  Attn2Params p;
  memset(&p, 0, sizeof(p));
  const int rr = dense ? d->M : d->k;
  GQE_TRY(tmap_heads(&p.tmQ[0], Q, N, Hq, rr, 128 / rr));
  GQE_TRY(tmap_heads(&p.tmQ[1], Q, N, Hq, 1, 128));
  GQE_TRY(tmap_heads(&p.tmK, K, N, d->G, 1, 128));
  GQE_TRY(tmap_heads(&p.tmV, V, N, d->G, 1, 128));
  p.O = static_cast<__nv_bfloat16*>(O);
  p.B = d->B;
  p.T = d->T;
  p.Ha = Hq;
  p.w = slot_w;
  p.G = d->G;
  p.slot_blk0 = d->G * d->k;
  p.o_ld = slot_w ? d->G * d->k + d->G + 1 : Hq;
  int nrs = 0;
  for (int g = 0; g < d->G; ++g) p.rs[nrs++] = AttnRowSet{g * rr, rr, g, 0, g * rr};
  if (shared) p.rs[nrs++] = AttnRowSet{d->G * d->k, 1, 0, 1, slot_w ? d->G * d->k + d->G : d->G * d->k};
  p.nrs = nrs;
  p.npairs_max = (int)cdiv((long long)d->T * rr, 256);
  const long long items = (long long)p.npairs_max * d->B * nrs;
  if (items > 0x7fffffffll) return GQE_ERR_UNSUPPORTED;
  p.total_items = (int)items;
  p.scale_log2 = 1.4426950408889634f / sqrtf(64.f);
  const int grid = (int)std::min<long long>(items, sm_count());
  if (rr == 1 && slot_w == nullptr) {  // one row per token in every set, no slots: the quad softmax layout
    GQE_TRY(set_smem(attn2_fwd_kernel<true>, A2Smem::kBytes));
    return launch_pdl(attn2_fwd_kernel<true>, dim3(grid), dim3(kA2ThreadsQuad), A2Smem::kBytes, st, p);
  }
  GQE_TRY(set_smem(attn2_fwd_kernel<false>, A2Smem::kBytes));
  return launch_pdl(attn2_fwd_kernel<false>, dim3(grid), dim3(kA2ThreadsRow), A2Smem::kBytes, st, p);
}

// k = 1: the renormalised weight of the one selected expert is exactly 1, so
// the slot of group g is O[:, g] itself and the projection reads A's blocks
// straight from O (blocks [0, G) and [G, 2G) are O's routed blocks, block 2G
// the shared head). KA is (2G + 1)*64, or 2G*64 without the shared head.
int project_from_o(const gqe_dims* d, const void* O, const void* Wo, void* y, int KA, cudaStream_t st) {
  const long long N = (long long)d->B * d->T;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  const int Ha = d->G + 1;
  GQE_TRY(tmap_rows(&p.tmA, O, N, Ha * 64, Ha * 64, kGemmBM));
  GQE_TRY(tmap_rows(&p.tmB[0], Wo, KA, d->D, d->D, 64));
  p.seg[0] = GemmSeg{d->D, 0, 0, 0, (long long)d->D, static_cast<__nv_bfloat16*>(y)};
  GQE_TRY(tmap_rows(&p.tmC[0], y, N, d->D, d->D, 32));
  p.nseg = 1;
  p.ntn = (int)cdiv(d->D, kG2DenseBN);
  p.rows = (int)N;
  p.K = KA;
  p.amap_G = d->G;
  p.r_tile0 = 0x7fffffff;
  p.r_merge_seg = -1;
  p.sel_seg = -1;
  return launch_gemm_pair(p, cdiv(N, kPairBM) * p.ntn, st);
}

// A = combine(O, w) by combine_build_kernel, then y = A Wo.
int build_and_project(const gqe_dims* d, const CombineParams& cp, int KA, const void* Wo, void* y, cudaStream_t st) {
  const long long blocks = std::min<long long>(cdiv(cp.N * 32, 256), 148ll * 16);
  GQE_TRY(launch_pdl(combine_build_kernel, dim3((unsigned)blocks), dim3(256), 0, st, cp));
  const DenseSeg seg = {Wo, d->D, 0, d->D, y, (long long)d->D, 0};
  return gemm_dense(cp.A, cp.N, KA, &seg, 1, st);
}

int do_combine(const gqe_dims* d, const void* O, const float* w, const void* Wo, void* y, __nv_bfloat16* A,
               cudaStream_t st) {
  const int KA = combine_cols(d, GQE_COMBINE_SLOT);
  if (d->k == 1) return project_from_o(d, O, Wo, y, KA, st);
  const CombineParams cp{static_cast<const __nv_bfloat16*>(O), w, A, (long long)d->B * d->T, d->G, d->k,
                         0, kSlotPerGroup, 1};
  return build_and_project(d, cp, KA, Wo, y, st);
}

// Output construction of the variants (gqe_combine_mode), y = A Wo with Wo of
// combine_cols(d, mode) rows. The hard variant's A is O itself.
int do_combine_variant(const gqe_dims* d, int mode, const void* O, const float* w, const float* p_sel,
                       const void* Wo, void* y, __nv_bfloat16* A, cudaStream_t st) {
  const long long N = (long long)d->B * d->T;
  const int KA = combine_cols(d, mode);
  const __nv_bfloat16* Ob = static_cast<const __nv_bfloat16*>(O);
  switch (mode) {
    case GQE_COMBINE_HARD: {
      const DenseSeg seg = {Wo, d->D, 0, d->D, y, (long long)d->D, 0};
      return gemm_dense(O, N, KA, &seg, 1, st);
    }
    case GQE_COMBINE_WEIGHTED:
      return build_and_project(d, CombineParams{Ob, p_sel, A, N, d->G, d->k, 1, kNoSlot, 1}, KA, Wo, y, st);
    case GQE_COMBINE_GLOBAL_SLOT:
      return build_and_project(d, CombineParams{Ob, p_sel, A, N, d->G, d->k, 0, kGlobalSlot, 1}, KA, Wo, y, st);
    case GQE_COMBINE_NO_SHARED:
      if (d->k == 1) return project_from_o(d, O, Wo, y, KA, st);
      return build_and_project(d, CombineParams{Ob, w, A, N, d->G, d->k, 0, kSlotPerGroup, 0}, KA, Wo, y, st);
    default:
      return GQE_ERR_INVALID_ARG;
  }
}

// Self-test of the bounded waits: one thread waits on an mbarrier that no
// thread arrives on, so the wait runs out, records the timeout and returns.
__global__ void selftest_wait_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag);
}

// Streams and events of the host-buffer entry point, created once per device
// and reused (guarded by g_pipe_mutex while a call enqueues its work).
constexpr int kHostChunks = 8;
constexpr int kPipeDevices = 64;
struct HostPipe {
  cudaStream_t h2d, d2h;
  cudaEvent_t start, done, in[kHostChunks], out[kHostChunks];
  bool ready;
};
std::mutex g_pipe_mutex;
HostPipe g_pipe[kPipeDevices];

int host_pipe(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQE_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kPipeDevices) return GQE_ERR_UNSUPPORTED;
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    HostPipe n;
    GQE_TRY(cuda_status(cudaStreamCreateWithFlags(&n.h2d, cudaStreamNonBlocking)));
    GQE_TRY(cuda_status(cudaStreamCreateWithFlags(&n.d2h, cudaStreamNonBlocking)));
    GQE_TRY(cuda_status(cudaEventCreateWithFlags(&n.start, cudaEventDisableTiming)));
    GQE_TRY(cuda_status(cudaEventCreateWithFlags(&n.done, cudaEventDisableTiming)));
    for (int i = 0; i < kHostChunks; ++i) {
      GQE_TRY(cuda_status(cudaEventCreateWithFlags(&n.in[i], cudaEventDisableTiming)));
      GQE_TRY(cuda_status(cudaEventCreateWithFlags(&n.out[i], cudaEventDisableTiming)));
    }
    n.ready = true;
    hp = n;
  }
  *out = &hp;
  return GQE_OK;
}

// The persistent tensor-core decode attention over the caches (decode.cuh).
// dp.nsplit: the splits the workspace holds; the launch sets its own count
// (*nsplit_used), which the merge must take.
int launch_decode_attn_mma(const DecodeParams& dp, int* nsplit_used, cudaStream_t st) {
  DecodeMmaParams P;
  memset(&P, 0, sizeof(P));
  GQE_TRY(tmap_heads(&P.tmK, dp.Kc, (long long)dp.B * dp.T, dp.G, 1, kDmSK));
  GQE_TRY(tmap_heads(&P.tmV, dp.Vc, (long long)dp.B * dp.T, dp.G, 1, kDmSK));
  P.d = dp;
  P.nitem = (int)cdiv(dp.T, kDmItem);
  P.items = (long long)dp.B * P.nitem;
  P.wpg = dm_wpg(dp.G);
  P.gpw = dp.G > kDmWarps ? dp.G / kDmWarps : 1;
  const int grid = (int)std::min<long long>(std::min<long long>(P.items, kDmGridMax), sm_count());
  // the workspace holds dm_nsplit(B, G, kDmGridMax) splits, at least this grid's
  P.d.nsplit = dm_nsplit(dp.B, dp.G, grid);
  if (P.d.nsplit > dp.nsplit || dp.rmax > 16) return GQE_ERR_UNSUPPORTED;
  *nsplit_used = P.d.nsplit;
  GQE_TRY(set_smem(decode_attn_mma_kernel, dm_smem()));
  return launch_pdl(decode_attn_mma_kernel, dim3(std::max(grid, 1)), dim3(kDmThreads), dm_smem(), st, P);
}

int check_ptrs(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr || !aligned16(p)) return GQE_ERR_INVALID_ARG;
  return GQE_OK;
}

}  // namespace

// ===========================================================================
// exported C ABI
// ===========================================================================
extern "C" {

int gqe_version(void) { return 100; }

int gqe_validate_dims(const gqe_dims* d) { return check_dims(d); }

// Decode step: the B new tokens as one sequence of B tokens for the prefill
// kernels (routing, projections, output projection).
gqe_dims decode_token_dims(const gqe_dims* d) {
  gqe_dims t = *d;
  t.B = 1;
  t.T = d->B;
  return t;
}

struct DecodeWs {
  RouteWs route;
  float* margin;
  int32_t *seg_off, *seg_tok;
  __nv_bfloat16 *Kn, *Vn, *Q, *O, *A;
  float *part_ml, *part_o;
  int nsplit, rmax;
};
DecodeWs carve_decode(Carver& c, const gqe_dims* d) {
  const gqe_dims t = decode_token_dims(d);
  const size_t B = d->B;
  const int Ha = d->G * d->k + 1;
  DecodeWs f;
  f.route = carve_route(c, &t);
  f.margin = c.take<float>(B * d->G);
  f.seg_off = c.take<int32_t>((size_t)d->G * d->M + 1);
  f.seg_tok = c.take<int32_t>(B * d->G * d->k);
  f.Kn = c.take<__nv_bfloat16>(B * d->G * 64);
  f.Vn = c.take<__nv_bfloat16>(B * d->G * 64);
  f.Q = c.take<__nv_bfloat16>(B * Ha * 64);
  f.O = c.take<__nv_bfloat16>(B * Ha * 64);
  f.A = d->k == 1 ? nullptr : c.take<__nv_bfloat16>(B * (size_t)(d->G * d->k + d->G + 1) * 64);
  f.nsplit = dm_nsplit(d->B, d->G, kDmGridMax);
  f.rmax = d->k + 1;
  const size_t parts = B * d->G * f.rmax * (size_t)f.nsplit;
  f.part_ml = c.take<float>(parts * 2);
  f.part_o = c.take<float>(parts * 64);
  return f;
}

size_t gqe_workspace_bytes(const gqe_dims* d, int op) {
  if (check_dims(d) != GQE_OK) return 0;
  Carver c{nullptr};
  switch (op) {
    case GQE_OP_ROUTE: carve_route(c, d); return c.off;
    case GQE_OP_QPROJ: return 0;
    case GQE_OP_ATTN: return 0;
    case GQE_OP_COMBINE: return combine_ws_bytes(d);
    case GQE_OP_FORWARD: carve_forward(c, d); return c.off;
    case GQE_OP_FORWARD_HOST: {
      carve_forward(c, d);
      c.take<__nv_bfloat16>((size_t)d->B * d->T * d->D);
      c.take<__nv_bfloat16>((size_t)d->B * d->T * d->D);
      return c.off;
    }
    case GQE_OP_DENSE: carve_dense(c, d); return c.off;
    case GQE_OP_DECODE: carve_decode(c, d); return c.off;
    case GQE_OP_FORWARD_VARIANT: {
      carve_forward(c, d);
      const size_t N = (size_t)d->B * d->T;
      c.take<float>(N * d->G * d->k);                                      // probabilities
      c.take<__nv_bfloat16>(N * (size_t)variant_max_cols(d));              // variant A
      return c.off;
    }
    default: return 0;
  }
}

int gqe_route(const gqe_dims* d, const void* x, const void* Wr, const float* br, int32_t* sel, float* w,
              float* margin, int32_t* seg_off, int32_t* seg_tok, int32_t* row_map, void* ws, size_t ws_bytes,
              void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({x, Wr, sel, w, seg_off, seg_tok}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  if (margin && !aligned16(margin)) return GQE_ERR_INVALID_ARG;
  if (row_map && !aligned16(row_map)) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_ROUTE)));
  GQE_TRY(check_device());
  Carver c{static_cast<uint8_t*>(ws)};
  RouteWs rw = carve_route(c, d);
  return do_route(d, x, Wr, br, sel, w, margin, seg_off, seg_tok, row_map, rw, static_cast<cudaStream_t>(stream));
}

int gqe_qproj(const gqe_dims* d, const void* x, const void* Wq, const void* Wk, const void* Wv, const int32_t* sel,
              const int32_t* seg_off, const int32_t* seg_tok, void* Q, void* K, void* V, void* ws, size_t ws_bytes,
              void* stream) {
  (void)ws;
  (void)ws_bytes;
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({x, Wq, Wk, Wv, sel, seg_off, seg_tok, Q, K, V}));
  GQE_TRY(check_device());
  return do_qproj(d, x, Wq, Wk, Wv, sel, seg_off, seg_tok, Q, K, V, static_cast<cudaStream_t>(stream));
}

int gqe_attn(const gqe_dims* d, const void* Q, const void* K, const void* V, void* O, void* ws, size_t ws_bytes,
             void* stream) {
  (void)ws;
  (void)ws_bytes;
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({Q, K, V, O}));
  GQE_TRY(check_device());
  return do_attn2(d, Q, d->G * d->k + 1, K, V, O, false, true, static_cast<cudaStream_t>(stream));
}

int gqe_combine(const gqe_dims* d, const void* O, const float* w, const void* Wo, void* y, void* ws, size_t ws_bytes,
                void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({O, w, Wo, y}));
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_COMBINE)));
  GQE_TRY(check_device());
  return do_combine(d, O, w, Wo, y, static_cast<__nv_bfloat16*>(ws), static_cast<cudaStream_t>(stream));
}

// The layer: mode GQE_COMBINE_SLOT is the GQE output construction; the other
// modes are the ablation variants (see gqe_forward_variant).
int do_forward(const gqe_dims* d, int mode_bits, const void* x, const void* Wq, const void* Wk, const void* Wv,
               const void* Wr, const float* br, const void* Wo, void* y, void* ws, cudaStream_t st) {
  const int mode = mode_bits & 0xff, qpath = mode_bits & (GQE_QPROJ_GATHER | GQE_QPROJ_DENSE);
  Carver c{static_cast<uint8_t*>(ws)};
  FwdWs f = carve_forward(c, d);
  const size_t N = (size_t)d->B * d->T;
  float* p_sel = nullptr;
  __nv_bfloat16* A2 = nullptr;
  if (mode != GQE_COMBINE_SLOT) {
    p_sel = c.take<float>(N * d->G * d->k);
    A2 = c.take<__nv_bfloat16>(N * (size_t)variant_max_cols(d));
  }
  // Without the shared head neither its query nor its attention is computed
  // (its column of Q and O is left unwritten and is never read).
  const bool shared = mode != GQE_COMBINE_NO_SHARED;
  // one pair-GEMM launch over x: K, V, the shared head's query and the router
  // (logits and decisions), then the selected queries: a dense product over
  // the routed heads that keeps the selected rows, or (M > 2k) the
  // compaction and the gather
  const bool qsel = qpath == GQE_QPROJ_DENSE || (qpath == GQE_QPROJ_AUTO && qproj_dense_select(d));
  DenseSeg segs[3];
  kv_segments(d, Wq, Wk, Wv, f.Q, f.K, f.V, segs);
  GemmParams p;
  long long dense_tiles = 0, route_tiles = 0;
  GQE_TRY(dense_params(p, x, (long long)d->B * d->T, d->D, segs, shared ? 3 : 2, &dense_tiles));
  GQE_TRY(add_route_tiles(p, d, Wr, br, f.sel, f.w, f.margin, f.route, dense_tiles, &route_tiles));
  if (qsel) p.r_counts = nullptr;  // plain decisions, no segment lists
  p.r_p = (mode == GQE_COMBINE_WEIGHTED || mode == GQE_COMBINE_GLOBAL_SLOT) ? p_sel : nullptr;
  if (shared && d->T % kRouteChunk == 0) {
    // the router logits fill the second half of the shared head's 128-column
    // tiles (the same x tile), so no separate routing tiles are launched
    p.r_merge_seg = 2;
    p.r_tile0 = (int)dense_tiles;
    route_tiles = 0;
  }
  GQE_TRY(launch_gemm_pair(p, dense_tiles + route_tiles, st));
  if (qsel) {
    GQE_TRY(do_qselect(d, x, Wq, f.sel, f.Q, st));
  } else {
    GQE_TRY(route_finish(d, f.sel, f.seg_off, f.seg_tok, f.row_map, f.route, st));
    GQE_TRY(do_qgather(d, x, Wq, f.sel, f.seg_off, f.seg_tok, f.Q, st));
  }
  if (mode == GQE_COMBINE_SLOT && d->k > 1) {
    // the attention writes A itself (concatenation, per-group slots, shared
    // head), then y = A Wo: no separate combine pass over O
    GQE_TRY(do_attn2(d, f.Q, d->G * d->k + 1, f.K, f.V, f.A, false, true, st, f.w));
    const DenseSeg seg = {Wo, d->D, 0, d->D, y, (long long)d->D, 0};
    return gemm_dense(f.A, (long long)d->B * d->T, combine_cols(d, GQE_COMBINE_SLOT), &seg, 1, st);
  }
  GQE_TRY(do_attn2(d, f.Q, d->G * d->k + 1, f.K, f.V, f.O, false, shared, st));
  if (mode == GQE_COMBINE_SLOT) return do_combine(d, f.O, f.w, Wo, y, f.A, st);
  return do_combine_variant(d, mode, f.O, f.w, p_sel, Wo, y, A2, st);
}

int gqe_forward(const gqe_dims* d, const void* x, const void* Wq, const void* Wk, const void* Wv, const void* Wr,
                const float* br, const void* Wo, void* y, void* ws, size_t ws_bytes, void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({x, Wq, Wk, Wv, Wr, Wo, y}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_FORWARD)));
  GQE_TRY(check_device());
  return do_forward(d, GQE_COMBINE_SLOT, x, Wq, Wk, Wv, Wr, br, Wo, y, ws, static_cast<cudaStream_t>(stream));
}

int gqe_forward_variant(const gqe_dims* d, int mode, const void* x, const void* Wq, const void* Wk, const void* Wv,
                        const void* Wr, const float* br, const void* Wo, void* y, void* ws, size_t ws_bytes,
                        void* stream) {
  GQE_TRY(check_dims(d));
  const int cmode = mode & 0xff, qpath = mode & ~0xff;
  if (cmode < GQE_COMBINE_SLOT || cmode > GQE_COMBINE_NO_SHARED) return GQE_ERR_INVALID_ARG;
  if (qpath != GQE_QPROJ_AUTO && qpath != GQE_QPROJ_GATHER && qpath != GQE_QPROJ_DENSE) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ptrs({x, Wq, Wk, Wv, Wr, Wo, y}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_FORWARD_VARIANT)));
  GQE_TRY(check_device());
  return do_forward(d, mode, x, Wq, Wk, Wv, Wr, br, Wo, y, ws, static_cast<cudaStream_t>(stream));
}

int gqe_forward_host(const gqe_dims* d, const void* x_host, const void* Wq, const void* Wk, const void* Wv,
                     const void* Wr, const float* br, const void* Wo, void* y_host, void* ws, size_t ws_bytes,
                     void* stream) {
  GQE_TRY(check_dims(d));
  if (x_host == nullptr || y_host == nullptr) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ptrs({Wq, Wk, Wv, Wr, Wo}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_FORWARD_HOST)));
  GQE_TRY(check_device());
  Carver c{static_cast<uint8_t*>(ws)};
  carve_forward(c, d);
  uint8_t* x_dev = reinterpret_cast<uint8_t*>(c.take<__nv_bfloat16>((size_t)d->B * d->T * d->D));
  uint8_t* y_dev = reinterpret_cast<uint8_t*>(c.take<__nv_bfloat16>((size_t)d->B * d->T * d->D));
  const uint8_t* xh = static_cast<const uint8_t*>(x_host);
  uint8_t* yh = static_cast<uint8_t*>(y_host);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t seq_bytes = (size_t)d->T * d->D * 2;
  const int nch = std::min(d->B, kHostChunks);
  if (nch == 1) {
    GQE_TRY(cuda_status(cudaMemcpyAsync(x_dev, xh, d->B * seq_bytes, cudaMemcpyHostToDevice, st)));
    GQE_TRY(do_forward(d, GQE_COMBINE_SLOT, x_dev, Wq, Wk, Wv, Wr, br, Wo, y_dev, ws, st));
    return cuda_status(cudaMemcpyAsync(yh, y_dev, d->B * seq_bytes, cudaMemcpyDeviceToHost, st));
  }
  // Sequences are independent: chunk ci (whole sequences) is copied in on
  // the h2d stream, projected and attended on `stream`, and copied out on
  // the d2h stream, so the two copy directions and the forward passes of
  // different chunks overlap. The forward passes share the workspace in
  // stream order; x_dev and y_dev lie past the whole batch's forward
  // workspace.
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe* hp = nullptr;
  GQE_TRY(host_pipe(&hp));
  GQE_TRY(cuda_status(cudaEventRecord(hp->start, st)));  // earlier work on `stream` may still read x_dev
  GQE_TRY(cuda_status(cudaStreamWaitEvent(hp->h2d, hp->start, 0)));
  int rc = GQE_OK;
  for (int ci = 0; ci < nch && rc == GQE_OK; ++ci) {
    const int b0 = (int)((long long)d->B * ci / nch), b1 = (int)((long long)d->B * (ci + 1) / nch);
    gqe_dims dc = *d;
    dc.B = b1 - b0;
    const size_t off = (size_t)b0 * seq_bytes, bytes = (size_t)dc.B * seq_bytes;
    if ((rc = cuda_status(cudaMemcpyAsync(x_dev + off, xh + off, bytes, cudaMemcpyHostToDevice, hp->h2d)))) break;
    if ((rc = cuda_status(cudaEventRecord(hp->in[ci], hp->h2d)))) break;
    if ((rc = cuda_status(cudaStreamWaitEvent(st, hp->in[ci], 0)))) break;
    if ((rc = do_forward(&dc, GQE_COMBINE_SLOT, x_dev + off, Wq, Wk, Wv, Wr, br, Wo, y_dev + off, ws, st))) break;
    if ((rc = cuda_status(cudaEventRecord(hp->out[ci], st)))) break;
    if ((rc = cuda_status(cudaStreamWaitEvent(hp->d2h, hp->out[ci], 0)))) break;
    rc = cuda_status(cudaMemcpyAsync(yh + off, y_dev + off, bytes, cudaMemcpyDeviceToHost, hp->d2h));
  }
  // join: `stream` continues only after every copy this call enqueued (also on error)
  const int rj0 = cuda_status(cudaEventRecord(hp->in[0], hp->h2d));
  const int rj1 = rj0 ? rj0 : cuda_status(cudaStreamWaitEvent(st, hp->in[0], 0));
  const int rj2 = cuda_status(cudaEventRecord(hp->done, hp->d2h));
  const int rj3 = rj2 ? rj2 : cuda_status(cudaStreamWaitEvent(st, hp->done, 0));
  return rc ? rc : (rj1 ? rj1 : rj3);
}

int gqe_decode(const gqe_dims* d, const int32_t* cache_len, const void* x_new, const void* Wq, const void* Wk,
               const void* Wv, const void* Wr, const float* br, const void* Wo, void* K_cache, void* V_cache, void* y,
               int32_t* sel, float* w, void* ws, size_t ws_bytes, void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({cache_len, x_new, Wq, Wk, Wv, Wr, Wo, K_cache, V_cache, y, sel, w}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  if (d->B > 65535) return GQE_ERR_UNSUPPORTED;
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_DECODE)));
  GQE_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c{static_cast<uint8_t*>(ws)};
  DecodeWs f = carve_decode(c, d);
  const gqe_dims t = decode_token_dims(d);
  const int ka_cols = (d->G * d->k + d->G + 1) * 64;
  const bool skinny = d->B <= kSkinnyMaxTokens && sk_smem(d->D, true, d->B) <= 232448 && sk_smem(ka_cols, false, d->B) <= 232448;
  DecodeProjParams pp;
  memset(&pp, 0, sizeof(pp));
  pp.x = static_cast<const __nv_bfloat16*>(x_new);
  pp.br = br;
  pp.cache_len = cache_len;
  pp.Kc = static_cast<__nv_bfloat16*>(K_cache);
  pp.Vc = static_cast<__nv_bfloat16*>(V_cache);
  pp.Q = f.Q;
  pp.sel = sel;
  pp.w = w;
  pp.margin = f.margin;
  pp.O = f.O;
  pp.y = static_cast<__nv_bfloat16*>(y);
  pp.B = d->B;
  pp.T = d->T;
  pp.D = d->D;
  pp.G = d->G;
  pp.M = d->M;
  pp.k = d->k;
  if (skinny) {
    // a few new tokens: K/V (written straight into the caches at
    // cache_len), the routing and the queries as skinny products in one
    // launch, one 8-CTA cluster per 64-column weight slice
    const int GM = d->G * d->M, Ka = (d->G * d->k + d->G + 1) * 64;
    GQE_TRY(tmap_rows(&pp.tmWq, Wq, d->D, (GM + 1) * 64, (GM + 1) * 64, kSkBoxRows));
    GQE_TRY(tmap_rows(&pp.tmWk, Wk, d->D, d->G * 64, d->G * 64, kSkBoxRows));
    GQE_TRY(tmap_rows(&pp.tmWv, Wv, d->D, d->G * 64, d->G * 64, kSkBoxRows));
    GQE_TRY(tmap_rows(&pp.tmWr, Wr, d->D, GM, GM, kSkBoxRows));
    GQE_TRY(tmap_rows(&pp.tmWo, Wo, Ka, d->D, d->D, kSkBoxRows));
    const int smem = sk_smem(d->D, true, d->B);
    GQE_TRY(set_smem(decode_proj_kernel, smem));
    GQE_TRY(launch_pdl(decode_proj_kernel, dim3((2 * d->G + 1 + GM) * kSkCluster), dim3(kSkinnyThreads), smem, st,
                       pp));
  }
  // one pair-GEMM launch over the new tokens: K, V, the shared query and the
  // router, then the compaction and the selected queries (prefill kernels)
  DenseSeg segs[3];
  kv_segments(&t, Wq, Wk, Wv, f.Q, f.Kn, f.Vn, segs);
  if (!skinny) {
    GemmParams p;
    long long dense_tiles = 0, route_tiles = 0;
    GQE_TRY(dense_params(p, x_new, d->B, d->D, segs, 3, &dense_tiles));
    GQE_TRY(add_route_tiles(p, &t, Wr, br, sel, w, f.margin, f.route, dense_tiles, &route_tiles));
    const bool qsel = qproj_dense_select(&t);
    if (qsel) p.r_counts = nullptr;
    GQE_TRY(launch_gemm_pair(p, dense_tiles + route_tiles, st));
    if (qsel) {
      GQE_TRY(do_qselect(&t, x_new, Wq, sel, f.Q, st));
    } else {
      GQE_TRY(route_finish(&t, sel, f.seg_off, f.seg_tok, nullptr, f.route, st));
      GQE_TRY(do_qgather(&t, x_new, Wq, sel, f.seg_off, f.seg_tok, f.Q, st));
    }
  }
  // the cache side: append, split-K attention, merge
  DecodeParams dp;
  dp.Q = f.Q;
  dp.Kn = f.Kn;
  dp.Vn = f.Vn;
  dp.Kc = static_cast<__nv_bfloat16*>(K_cache);
  dp.Vc = static_cast<__nv_bfloat16*>(V_cache);
  dp.cache_len = cache_len;
  dp.part_ml = f.part_ml;
  dp.part_o = f.part_o;
  dp.O = f.O;
  dp.B = d->B;
  dp.T = d->T;
  dp.G = d->G;
  dp.k = d->k;
  dp.Ha = d->G * d->k + 1;
  dp.rmax = f.rmax;
  dp.nsplit = f.nsplit;
  dp.scale_log2 = 1.4426950408889634f / sqrtf(64.f);
  const long long pieces = (long long)d->B * d->G * 64 / 8 * 2;
  if (!skinny)
    GQE_TRY(launch_pdl(decode_append_kernel, dim3((unsigned)std::min<long long>(cdiv(pieces, 256), 4096)), dim3(256),
                       0, st, dp));
  GQE_TRY(launch_decode_attn_mma(dp, &dp.nsplit, st));
  GQE_TRY(launch_pdl(decode_merge_kernel, dim3((unsigned)((long long)d->B * dp.Ha)), dim3(kDecMergeThreads), 0, st, dp));
  if (skinny) {
    const int smem = sk_smem(ka_cols, false, d->B);
    GQE_TRY(set_smem(decode_out_kernel, smem));
    return launch_pdl(decode_out_kernel, dim3((unsigned)(d->D / 64) * kSkCluster), dim3(kSkinnyThreads), smem, st,
                      pp);
  }
  return do_combine(&t, f.O, w, Wo, y, f.A, st);
}

int gqa_dense_forward(const gqe_dims* d, const void* x, const void* Wq, const void* Wk, const void* Wv,
                      const void* Wo_dense, void* y, void* ws, size_t ws_bytes, void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({x, Wq, Wk, Wv, Wo_dense, y}));
  GQE_TRY(check_ws(ws, ws_bytes, gqe_workspace_bytes(d, GQE_OP_DENSE)));
  GQE_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Carver c{static_cast<uint8_t*>(ws)};
  DenseWs w = carve_dense(c, d);
  const long long N = (long long)d->B * d->T;
  const int G = d->G, M = d->M, H = G * M;
  const int wq_cols = (G * M + 1) * 64;
  const DenseSeg segs[3] = {
      {Wq, wq_cols, 0, H * 64, w.Q, (long long)H * 64, 0},
      {Wk, G * 64, 0, G * 64, w.K, (long long)G * 64, 0},
      {Wv, G * 64, 0, G * 64, w.V, (long long)G * 64, 0},
  };
  GQE_TRY(gemm_dense(x, N, d->D, segs, 3, st));
  GQE_TRY(do_attn2(d, w.Q, H, w.K, w.V, w.O, true, false, st));
  const DenseSeg so = {Wo_dense, d->D, 0, d->D, y, (long long)d->D, 0};
  return gemm_dense(w.O, N, H * 64, &so, 1, st);
}

int gqe_check_error(void* stream) {
  GQE_TRY(cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(stream))));
  int word = 0;
  GQE_TRY(cuda_status(cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int))));
  if (word != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
    return word == kDevErrTimeout ? GQE_ERR_TIMEOUT : GQE_ERR_DEVICE_CHECK;
  }
  return GQE_OK;
}

const char* gqe_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

int gqe_selftest_wait_timeout(void* stream) {
  GQE_TRY(check_device());
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_status(cudaGetLastError());
}

const char* gqe_status_string(int status) {
  switch (status) {
    case GQE_OK: return "ok";
    case GQE_ERR_INVALID_ARG: return "invalid argument (null or misaligned pointer, or bad dims)";
    case GQE_ERR_UNSUPPORTED: return "unsupported shape";
    case GQE_ERR_WORKSPACE: return "workspace too small or misaligned";
    case GQE_ERR_CUDA: return "CUDA runtime error";
    case GQE_ERR_TIMEOUT: return "device pipeline wait timed out";
    case GQE_ERR_NO_DEVICE: return "no sm_100 device is current";
    case GQE_ERR_DEVICE_CHECK: return "a device-side index check failed (access skipped)";
    default: return "unknown status";
  }
}

}  // extern "C"

// ===========================================================================
// gqe_route_noalloc: gqe_route for callers that cannot allocate device memory
// ===========================================================================
// The router's only scratch (per-chunk expert counts and their scanned bases)
// lives in this fixed array instead of a caller-provided workspace. Every GPU
// that loads the library keeps these bytes reserved until the process exits.
namespace {

constexpr size_t kNoAllocScratchBytes = 1u << 20;  // 1 MiB
__device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device. In host code the
// array's name only stands for it, so the address is looked up once per
// device with that device current, then reused.
int route_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GQE_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return GQE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return GQE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GQE_OK;
}

}  // namespace

extern "C" int gqe_route_noalloc(const gqe_dims* d, const void* x, const void* Wr, const float* br, int32_t* sel,
                                 float* w, float* margin, int32_t* seg_off, int32_t* seg_tok, int32_t* row_map,
                                 void* stream) {
  GQE_TRY(check_dims(d));
  GQE_TRY(check_ptrs({x, Wr, sel, w, seg_off, seg_tok}));
  if (br && !aligned16(br)) return GQE_ERR_INVALID_ARG;
  if (margin && !aligned16(margin)) return GQE_ERR_INVALID_ARG;
  if (row_map && !aligned16(row_map)) return GQE_ERR_INVALID_ARG;
  Carver sizing{nullptr};
  carve_route(sizing, d);
  if (sizing.off > kNoAllocScratchBytes) return GQE_ERR_WORKSPACE;
  GQE_TRY(check_device());
  void* scratch = nullptr;
  GQE_TRY(route_scratch(&scratch));
  // No buffer needs zeroing: the select kernel writes every count and the
  // scan kernel writes every base before they are read.
  Carver c{static_cast<uint8_t*>(scratch)};
  RouteWs rw = carve_route(c, d);
  return do_route(d, x, Wr, br, sel, w, margin, seg_off, seg_tok, row_map, rw, static_cast<cudaStream_t>(stream));
}
