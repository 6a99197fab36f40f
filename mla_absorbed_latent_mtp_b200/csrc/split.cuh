// split.cuh -- the split-L bookkeeping shared by the attend kernel, which leaves one
// unnormalised partial (O, m, l) per CTA-group segment of a sequence, and the kernels that
// merge those partials with their log-sum-exp weights (the combine, and the merge fused
// into the W_UV up-projection).
//
// The tiles of all sequences of the tile list form one list that G CTA groups split into
// equal contiguous ranges: group g takes tiles [g*T/G, (g+1)*T/G).  A sequence of the list
// is a cache sequence b (dense / paged: its Q queries share the tiles, one CTA per query in
// every group) or one (b, i) index list (indexed: one CTA per group).  The partial of group
// g for sequence s and query i sits in workspace slot (g + s) * Q + i (dense / paged) or
// g + s (indexed); the first attend CTA writes, per sequence, its first tile and tile count.
#pragma once

#include "internal.h"

namespace mla {
namespace split {

__device__ __forceinline__ int num_seqs(const AttendParams &p, int mode) {
  return mode == kModeIndexed ? p.B * p.Q : p.B;
}

__device__ __forceinline__ long long group_start(long long g, long long T, long long G) { return g * T / G; }

// The group whose tile range holds tile t: the largest g with g*T/G <= t.
__device__ __forceinline__ long long group_of(long long t, long long T, long long G) { return ((t + 1) * G - 1) / T; }

// The partials of sequence s, from the table the attend kernel wrote: `count` groups, the
// k-th being partial_group(k).  With at least as many tiles as groups (T >= G) every group
// holds tiles and the sequence's partials are those of the consecutive groups
// g_first .. g_first + count - 1; with fewer tiles than groups every group holds at most one
// tile, so the k-th partial is the group of the sequence's k-th tile (enumerating the
// groups in between would visit mostly empty ones).
struct GroupRange {
  long long g_first;  // first group (T >= G)
  long long ts;       // first tile of the sequence
  long long T, G;
  int count;          // number of partials
  __device__ __forceinline__ long long partial_group(int k) const {
    return T >= G ? g_first + k : group_of(ts + k, T, G);
  }
};

__device__ __forceinline__ GroupRange seq_group_range(const AttendParams &p, int mode, int s) {
  const int ns = num_seqs(p, mode);
  GroupRange r;
  r.G = p.groups;
  r.T = p.seq_ts[ns - 1] + p.seq_nt[ns - 1];
  r.ts = p.seq_ts[s];
  const int nt = p.seq_nt[s];
  r.g_first = 0;
  r.count = 0;
  if (nt > 0) {
    if (r.T >= r.G) {
      r.g_first = group_of(r.ts, r.T, r.G);
      r.count = (int)(group_of(r.ts + nt - 1, r.T, r.G) - r.g_first + 1);
    } else {
      r.count = nt;
    }
  }
  return r;
}

// Workspace slot of the partial of group g, tile-list sequence s, query i.
__device__ __forceinline__ long long partial_slot(const AttendParams &p, int mode, long long g, int s, int i) {
  return mode == kModeIndexed ? g + s : (g + s) * p.Q + i;
}

}  // namespace split
}  // namespace mla
