// attn.cuh -- shared definitions of the attention kernel (attn2.cuh): row
// sets and the lazy-rescale threshold.
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
#pragma once

#include "sm100.cuh"

namespace gqe {

constexpr int kMaxRowSets = 72;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct AttnRowSet {
  int h0;   // first Q head of the set
  int rr;   // rows per token (1, 2, 4 or 8)
  int kvg;  // KV head the set attends
  int tm;   // which Q tensor map (box height rr)
  int ob;   // first 64-wide output block of the set in a token's output row
};

}  // namespace gqe
