/*
 * gqe.h -- C ABI of libgqe: the Grouped Query Experts (GQE) attention-layer
 * forward pass on NVIDIA B200 (sm_100a).
 *
 * The method ("Grouped Query Experts: Mixture-of-Experts on GQA
 * Self-Attention"; gist.science technical summary, section "Architecture and
 * routing"; animattoys.com article on the same paper, section 4 "How GQE
 * works"): inside every GQA group the M query heads form a pool of experts; a
 * per-token router activates the top-k of them; K/V projections and K/V heads
 * stay dense; every selected expert attends causally to its group's K/V; the
 * layer output is the output projection of [hard concatenation of the selected
 * experts | per-group weighted slot (router probabilities renormalised over
 * the selected set) | one always-on shared head].
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers (cudaMalloc'd or torch-owned),
 *    except where a name ends in `_host`. The caller owns every buffer and the
 *    workspace; the library never allocates or frees device memory.
 *  - Tensors are dense row-major. "bf16" = IEEE bfloat16 stored as uint16.
 *    Weights are [in, out]. Token index n = b*T + t.
 *  - Every pointer must be 16-byte aligned; D and dh multiples of 64.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *    asynchronous: they validate arguments on the host, enqueue kernels and
 *    return. Invalid arguments return an error code before any launch.
 *  - `ws`/`ws_bytes`: caller-provided device workspace of at least
 *    gqe_workspace_bytes(dims, op) bytes, 256-byte aligned. Contents on entry
 *    are ignored.
 *  - Device-side failures (a pipeline wait that exceeded its time limit) are
 *    recorded in a sticky per-device error word read by gqe_check_error().
 *
 * Supported shapes (others return GQE_ERR_UNSUPPORTED): dh == 64;
 * D % 64 == 0; 1 <= k <= M; G*M a power of two in [8, 64]; k and M in {1,2,4,8}
 * (128 must be a multiple of the rows each token contributes to one
 * attention tile); B*T < 2^31 / (G*k+1) / 64.
 */
#ifndef GQE_H_
#define GQE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer dimensions: batch, tokens per sequence, d_model, KV groups, experts
 * per group, experts selected per group, head dim. The shared head is always
 * on. */
typedef struct gqe_dims {
  int32_t B, T, D, G, M, k, dh;
} gqe_dims;

enum gqe_status {
  GQE_OK = 0,
  GQE_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad dims          */
  GQE_ERR_UNSUPPORTED = -2,  /* shape outside the supported set above      */
  GQE_ERR_WORKSPACE = -3,    /* ws too small or misaligned                  */
  GQE_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed        */
  GQE_ERR_TIMEOUT = -5,      /* a device pipeline wait hit its time limit   */
  GQE_ERR_NO_DEVICE = -6,    /* no sm_100 device current                    */
  GQE_ERR_DEVICE_CHECK = -7  /* a device-side index check failed; the
                                offending access was skipped               */
};

/* Operation selector for gqe_workspace_bytes. */
enum gqe_op {
  GQE_OP_ROUTE = 1,
  GQE_OP_QPROJ = 2,
  GQE_OP_ATTN = 3,
  GQE_OP_COMBINE = 4,
  GQE_OP_FORWARD = 5,
  GQE_OP_DENSE = 6,
  GQE_OP_FORWARD_HOST = 7,
  GQE_OP_DECODE = 8,
  GQE_OP_FORWARD_VARIANT = 9
};

/* Output construction of gqe_forward_variant. */
enum gqe_combine_mode {
  GQE_COMBINE_SLOT = 0,         /* GQE: [hard concat | renormalised slot per group | shared] */
  GQE_COMBINE_HARD = 1,         /* ablation: [hard concat | shared], no slot                 */
  GQE_COMBINE_WEIGHTED = 2,     /* ablation: [concat, each selected output scaled by its
                                   expert's in-group probability (not renormalised) |
                                   shared], no slot                                           */
  GQE_COMBINE_GLOBAL_SLOT = 3,  /* [hard concat | ONE slot: all selected outputs averaged
                                   with their in-group probabilities renormalised over
                                   all G*k selected experts | shared]                         */
  GQE_COMBINE_NO_SHARED = 4     /* ablation: [hard concat | renormalised slot per group],
                                   no shared head (neither its query nor its attention
                                   is computed)                                               */
};

/* How gqe_forward_variant computes the selected experts' queries, or'ed into
 * its `mode`. Both give the same Q (the same dot products, accumulated in the
 * same order); they differ in the work done.
 *   GQE_QPROJ_AUTO   : GQE_QPROJ_DENSE when M <= 2k, else GQE_QPROJ_GATHER
 *                      (what gqe_forward does)
 *   GQE_QPROJ_GATHER : selected heads only: the tokens of every (sequence,
 *                      group, expert) are compacted and their rows of x
 *                      gathered per expert (gqe_route + gqe_qproj)
 *   GQE_QPROJ_DENSE  : every routed head's query is projected on the tensor
 *                      cores and each token's selected rows are kept (at
 *                      most M/k times the selected heads' flops, no
 *                      compaction and no gather) */
enum gqe_qproj_path {
  GQE_QPROJ_AUTO = 0,
  GQE_QPROJ_GATHER = 0x100,
  GQE_QPROJ_DENSE = 0x200
};

/* Workspace bytes the operation needs for these dims (0 if none); returns 0
 * and nothing else for invalid dims (check with gqe_validate_dims). */
size_t gqe_workspace_bytes(const gqe_dims* d, int op);

/* GQE_OK if the dims are supported, else the error code a call would give. */
int gqe_validate_dims(const gqe_dims* d);

/*
 * gqe_route -- the per-token router and the token compaction.
 * Method: gist.science summary, "Architecture and routing", conditional
 * activation (per token, top-k experts of every group) and the renormalised
 * weighted sum (router probabilities renormalised over the selected set);
 * animattoys.com article, section 4 (router scores each expert of each group,
 * activates the k best).
 *
 *   logits[n,g,e] = sum_d x[n,d] * Wr[d, g*M+e] + br[g*M+e]    (fp32 accumulate)
 *   p = softmax over e within the group; top-k by p (exact ties -> lower e)
 *
 * In : x  [B*T, D] bf16; Wr [D, G*M] bf16; br [G*M] fp32 or NULL (zeros).
 * Out: sel     [B*T, G, k] int32  selected experts, ascending
 *      w       [B*T, G, k] fp32   p_sel / sum(p_sel), same order as sel
 *      margin  [B*T, G]    fp32   logit of k-th ranked minus (k+1)-th
 *                                 (+inf when k == M); NULL to skip
 *      seg_off [B*G*M + 1] int32  segment s = (b*G + g)*M + e starts at
 *                                 seg_off[s]; seg_off[B*G*M] = B*T*G*k
 *      seg_tok [B*T*G*k]   int32  token n of every compacted row, ascending
 *                                 within each segment
 *      row_map [B*T, G, k] int32  compacted row of (n, g, slot); NULL to skip
 * ws: gqe_workspace_bytes(d, GQE_OP_ROUTE) (per-chunk expert counts).
 */
int gqe_route(const gqe_dims* d, const void* x, const void* Wr, const float* br,
              int32_t* sel, float* w, float* margin, int32_t* seg_off,
              int32_t* seg_tok, int32_t* row_map, void* ws, size_t ws_bytes,
              void* stream);

/*
 * gqe_route_noalloc -- gqe_route without a caller workspace. (The paper has no
 * counterpart: this is a calling convenience of the library.)
 *
 * For callers that cannot allocate device memory on this path: for example
 * code embedded in a host program that owns and pre-reserves all device
 * memory, or a latency-critical loop where a cudaMalloc (which can
 * synchronise the device) is not acceptable. The router's scratch (two int32
 * arrays of B * ceil(T/128) * G*M counts) lives in a fixed 1 MiB array inside
 * the library; every GPU that loads the library keeps those bytes reserved
 * until the process exits. Arguments, outputs and results are exactly those
 * of gqe_route.
 *
 * - Returns GQE_ERR_WORKSPACE, before any launch, when the scratch would
 *   exceed 1 MiB, i.e. when 2 * B * ceil(T/128) * G*M * 4 bytes (each array
 *   rounded up to 256 bytes) is larger than 1048576.
 * - The first call on each device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is kept for the life of the process: do not use this entry
 *   point on a device after cudaDeviceReset (or any teardown of its primary
 *   context) in the same process, since the array then moves.
 * - Every call on a device shares the one array and leaves its contents
 *   behind. Nothing in it needs to start at zero (every entry is written
 *   before it is read), but calls that overlap on the GPU (different streams
 *   without ordering between them) race on it and give wrong token lists.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
int gqe_route_noalloc(const gqe_dims* d, const void* x, const void* Wr,
                      const float* br, int32_t* sel, float* w, float* margin,
                      int32_t* seg_off, int32_t* seg_tok, int32_t* row_map,
                      void* stream);

/*
 * gqe_qproj -- dense K/V projection and the query projection of the selected
 * experts only (plus the shared head), on tcgen05 tensor cores.
 * Method: gist.science summary, "Architecture and routing", dense KV path
 * (K/V projections unchanged from GQA) and sparsity on the query side only;
 * animattoys.com article, section 4 (each expert has its own query
 * projection; the group's experts read the same K/V).
 *
 * In : x [B*T, D]; Wq [D, (G*M+1)*dh] (routed head h = g*M+e, shared head
 *      last); Wk, Wv [D, G*dh]; sel/seg_off/seg_tok from gqe_route.
 * Out: Q [B*T, G*k+1, dh] bf16: Q[n, g*k+j] = x[n] Wq[:, head of sel[n,g,j]],
 *        Q[n, G*k] = x[n] Wq[:, shared];
 *      K, V [B*T, G, dh] bf16.
 * ws: none (0 bytes). Segment sizes are read on the device: no host sync.
 */
int gqe_qproj(const gqe_dims* d, const void* x, const void* Wq, const void* Wk,
              const void* Wv, const int32_t* sel, const int32_t* seg_off,
              const int32_t* seg_tok, void* Q, void* K, void* V, void* ws,
              size_t ws_bytes, void* stream);

/*
 * gqe_attn -- routed causal attention (FlashAttention-style, tcgen05 + TMEM,
 * K/V tiles streamed by TMA).
 * Method: animattoys.com article, section 4 (every selected expert computes
 * attention on its own against its group's shared K/V; the shared head is
 * always computed); gist.science summary, "Architecture and routing".
 * The shared head attends KV head 0 (the pages do not say which; this is the
 * library's fixed choice).
 *
 *   O[n, g*k+j] = sum_{s<=t} softmax_s(Q[n,g*k+j] . K[b,s,g] / sqrt(dh)) V[b,s,g]
 *   O[n, G*k]   = same with Q[n, G*k] against KV head 0
 *
 * In : Q [B*T, G*k+1, dh]; K, V [B*T, G, dh]. Out: O [B*T, G*k+1, dh] bf16.
 * Arithmetic: S and O accumulate in fp32 (TMEM), P rounded to bf16.
 */
int gqe_attn(const gqe_dims* d, const void* Q, const void* K, const void* V,
             void* O, void* ws, size_t ws_bytes, void* stream);

/*
 * gqe_combine -- output construction and output projection.
 * Method: gist.science summary, "Architecture and routing", output
 * construction (hard concatenation; renormalised weighted sum; always-on
 * shared head); animattoys.com article, section 4 (the three parts are merged
 * and passed through the final output projection).
 *
 *   A[n] = [O[n,0..G*k-1] (concat) | sum_j w[n,g,j] O[n,g*k+j] for g (slot)
 *           | O[n,G*k] (shared)]           width (G*k + G + 1)*dh
 *   y    = A Wo,   Wo [(G*k+G+1)*dh, D] bf16, y [B*T, D] bf16.
 * For k == 1 every renormalised weight is exactly 1, so the slot of group g
 * is O[n, g] and the projection reads all of A straight from O (no
 * workspace). For k > 1 A is assembled in the workspace first.
 * ws: gqe_workspace_bytes(d, GQE_OP_COMBINE) (0 when k == 1).
 */
int gqe_combine(const gqe_dims* d, const void* O, const float* w,
                const void* Wo, void* y, void* ws, size_t ws_bytes,
                void* stream);

/*
 * gqe_forward -- route -> qproj -> attn -> combine on one stream.
 * The selected queries follow GQE_QPROJ_AUTO (enum gqe_qproj_path): for
 * M <= 2k a dense product over all routed heads keeps each token's selected
 * rows, and the segment lists (seg_off, seg_tok, row_map) are not built;
 * for M > 2k the selected tokens are gathered per expert. Either way Q, and
 * so y, is the same as gqe_route + gqe_qproj + gqe_attn + gqe_combine give.
 * ws: gqe_workspace_bytes(d, GQE_OP_FORWARD); it holds every intermediate
 * (sel, w, margin, segments, Q, K, V, O, ...).
 */
int gqe_forward(const gqe_dims* d, const void* x, const void* Wq,
                const void* Wk, const void* Wv, const void* Wr,
                const float* br, const void* Wo, void* y, void* ws,
                size_t ws_bytes, void* stream);

/*
 * gqe_forward_host -- gqe_forward with the activations in HOST memory: the
 * call enqueues the copy of x_host into the workspace, the forward pass and
 * the copy of y back to y_host, all on `stream` (pin both host buffers for the
 * copies to be asynchronous). Weights are device pointers.
 * Host-buffer lifetime: the call returns once the work is enqueued. x_host
 * must stay allocated and unmodified, and y_host allocated and unread, until
 * the stream has passed the call (cudaStreamSynchronize, or an event recorded
 * after it). With pinned memory from a caching allocator, a buffer released
 * early can be handed out again and overwritten before its copy has run.
 * ws: gqe_workspace_bytes(d, GQE_OP_FORWARD_HOST).
 */
int gqe_forward_host(const gqe_dims* d, const void* x_host, const void* Wq,
                     const void* Wk, const void* Wv, const void* Wr,
                     const float* br, const void* Wo, void* y_host, void* ws,
                     size_t ws_bytes, void* stream);

/*
 * gqe_forward_variant -- gqe_forward with the output construction chosen by
 * `mode` (enum gqe_combine_mode). Method: animattoys.com article, section 6:
 * besides the full design (hard concatenation, a renormalised weighted slot
 * and the always-on shared head) the ablation trains a pure hard
 * concatenation and a concatenation weighted directly by the router's scores
 * without the renormalised slot; the gist.science summary, "Experimental
 * results", words the same ablation as removing the renormalised slot or the
 * shared head; the article's section 4 can be read as ONE weighted-average
 * slot over all selected experts. This library's readings: the variants keep
 * every part they do not name as removed, and the "router's scores" are the
 * in-group softmax probabilities of the selected experts.
 *
 * Wo rows, in A's column order (concat g-major, slot j; slots; shared):
 *     GQE_COMBINE_SLOT         (G*k + G + 1)*dh  (identical to gqe_forward)
 *     GQE_COMBINE_HARD         (G*k + 1)*dh
 *     GQE_COMBINE_WEIGHTED     (G*k + 1)*dh
 *     GQE_COMBINE_GLOBAL_SLOT  (G*k + 2)*dh
 *     GQE_COMBINE_NO_SHARED    (G*k + G)*dh
 * `mode` may also carry one enum gqe_qproj_path value (or'ed in).
 * ws: gqe_workspace_bytes(d, GQE_OP_FORWARD_VARIANT). An unknown mode returns
 * GQE_ERR_INVALID_ARG. Everything else as gqe_forward.
 */
int gqe_forward_variant(const gqe_dims* d, int mode, const void* x, const void* Wq,
                        const void* Wk, const void* Wv, const void* Wr,
                        const float* br, const void* Wo, void* y, void* ws,
                        size_t ws_bytes, void* stream);

/*
 * gqe_decode -- one generation step of the layer against a key/value cache.
 * Method: the layer of gqe_forward applied to one new token per sequence
 * (gist.science summary, "Architecture and routing"; animattoys.com
 * article, section 4); aiboss88.com wiki on grouped-query attention,
 * inference section: a decoder caches the key/value heads and reads them
 * back at every step. The pages give no decode procedure; this library's
 * reading: the new token of sequence b sits at position L_b = cache_len[b],
 * its K/V row is written there, and each of its query rows (the k selected
 * experts of every group, the shared head on KV head 0) attends positions
 * 0..L_b.
 *
 * d->B sequences, d->T = cache capacity (positions per sequence).
 * In : cache_len [B] int32 (device), 0 <= L_b < T; x_new [B, D] bf16;
 *      Wq, Wk, Wv, Wr, br, Wo as gqe_forward.
 * In/out: K_cache, V_cache [B, T, G, dh] bf16: rows < L_b are read; row L_b
 *      of each sequence is overwritten with the new token's K/V; rows past
 *      L_b are neither read nor written.
 * Out: y [B, D] bf16; sel [B, G, k] int32 and w [B, G, k] fp32 (the routing
 *      of the new tokens, as gqe_route).
 * ws : gqe_workspace_bytes(d, GQE_OP_DECODE).
 * A cache_len outside [0, T) skips that sequence's cache access and sets the
 * device check word (gqe_check_error returns GQE_ERR_DEVICE_CHECK). All
 * pointers are device pointers except d; B <= 65535. Asynchronous on
 * `stream`; capturable in a CUDA graph (no host synchronisation).
 */
int gqe_decode(const gqe_dims* d, const int32_t* cache_len, const void* x_new,
               const void* Wq, const void* Wk, const void* Wv, const void* Wr,
               const float* br, const void* Wo, void* K_cache, void* V_cache,
               void* y, int32_t* sel, float* w, void* ws, size_t ws_bytes,
               void* stream);

/*
 * gqa_dense_forward -- the all-heads GQA baseline the method is compared with
 * (gist.science summary, "Experimental results": 16 query heads over 8 KV
 * groups, all active). Head h = g*M+e attends KV group g; k is ignored.
 *   y = concat_h O_h Wo_dense,  Wq's first G*M*dh columns, Wo_dense [G*M*dh, D].
 * ws: gqe_workspace_bytes(d, GQE_OP_DENSE).
 */
int gqa_dense_forward(const gqe_dims* d, const void* x, const void* Wq,
                      const void* Wk, const void* Wv, const void* Wo_dense,
                      void* y, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then read and clear the current device's sticky
 * error word: GQE_OK, GQE_ERR_TIMEOUT, GQE_ERR_DEVICE_CHECK, or GQE_ERR_CUDA
 * if the stream itself reported an error. */
int gqe_check_error(void* stream);

/* Description of the CUDA error behind the last GQE_ERR_CUDA returned on the
 * calling host thread ("no error" if there was none). */
const char* gqe_last_cuda_error(void);

/*
 * gqe_selftest_wait_timeout -- failure-detection self-test. Enqueues on
 * `stream` one small kernel that waits on a pipeline barrier nothing will
 * ever complete, with the same bounded wait as every kernel of the library.
 * After about 2 s the wait gives up. It records a timeout in the device error
 * word and the kernel returns; it does not trap. The next gqe_check_error
 * then returns GQE_ERR_TIMEOUT, and the context stays usable. Returns
 * GQE_ERR_CUDA if the launch fails.
 */
int gqe_selftest_wait_timeout(void* stream);

/* Static description of a status code. */
const char* gqe_status_string(int status);

/* Library ABI version (major*100 + minor). */
int gqe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQE_H_ */
