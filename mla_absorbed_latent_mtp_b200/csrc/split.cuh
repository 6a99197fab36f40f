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

// The range of groups that processed tiles of sequence s, from the table the attend kernel
// wrote: groups g_first .. g_first + nslot - 1 (nslot = 0 for a sequence without tiles).
// T is the total tile count.  A group inside the range holds no tiles of s only when there
// are fewer tiles than groups (then some groups are empty).
struct GroupRange {
  long long g_first;
  long long T;
  int nslot;
};

__device__ __forceinline__ GroupRange seq_group_range(const AttendParams &p, int mode, int s) {
  const int ns = num_seqs(p, mode);
  const long long G = p.groups;
  GroupRange r;
  r.T = p.seq_ts[ns - 1] + p.seq_nt[ns - 1];
  const long long ts = p.seq_ts[s];
  const int nt = p.seq_nt[s];
  long long g_last = -1;
  r.g_first = 0;
  if (nt > 0) {
    r.g_first = ((ts + 1) * G - 1) / r.T;
    g_last = ((ts + nt) * G - 1) / r.T;
  }
  r.nslot = (int)(g_last - r.g_first + 1);
  return r;
}

// Whether group g holds any tiles (always true when every group has tiles).
__device__ __forceinline__ bool group_live(long long g, long long T, long long G) {
  return T >= G || group_start(g, T, G) < group_start(g + 1, T, G);
}

// Workspace slot of the partial of group g, tile-list sequence s, query i.
__device__ __forceinline__ long long partial_slot(const AttendParams &p, int mode, long long g, int s, int i) {
  return mode == kModeIndexed ? g + s : (g + s) * p.Q + i;
}

}  // namespace split
}  // namespace mla
