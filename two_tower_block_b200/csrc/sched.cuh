// Work split shared by the attention kernels, the split combine and the host.
//
// A "unit" is one (sequence, KV head[, block]) problem: its S*g packed query
// rows attend to one key list.  Its key list is cut into tiles: tile 0 is the
// block's own S keys, tiles 1.. are the visible context keys, key_tile at a
// time.  All units' tiles are laid end to end (unit-major) into one global
// sequence of T tiles, and range c of C' = min(C, T) gets tiles [floor(c*T/C'),
// floor((c+1)*T/C')); ranges c >= C' are empty.  Every range therefore carries the same work up to one
// tile, whatever the length mix, and a unit is cut only where a range
// boundary falls inside it.
//
// A range's pieces of units are "segments".  A segment that covers a whole
// unit writes the final output.  Otherwise it writes a partial (O / l and its
// lse) to slot 2*c + which, where which = 0 if the segment begins at the
// range's first tile and 1 otherwise; a cut unit is then finished by the
// combine kernel.  Only a range's first and last segment can belong to a cut
// unit, so 2*C slots always suffice.
//
// A plan may instead give the boundaries as a table starts[0..C'] (starts[0] = 0,
// starts[C'] = T, strictly increasing), which the block-causal calls of the default
// kernel use to weigh each unit's fixed cost (built by the plan on the host); everything
// above holds for it unchanged.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define TT_HD __host__ __device__ __forceinline__
#else
#define TT_HD inline
#endif

namespace tt {

TT_HD long long range_start(long long T, int C, int c) { return (long long)c * T / C; }

// Ranges actually used: min(C, T), so that every used range holds at least one
// tile and the ranges touching a cut unit are consecutive and all non-empty.
TT_HD int used_ranges(long long T, int C) { return T < (long long)C ? (int)T : C; }

// Index of the range whose [start, end) contains global tile x (0 <= x < T):
// the largest c with floor(c*T/C) <= x, i.e. ceil((x+1)*C/T) - 1.
TT_HD int range_of_tile(long long T, int C, long long x) {
  return (int)(((x + 1) * (long long)C + T - 1) / T) - 1;
}

// The same two for a boundary table (null: the uniform split).
TT_HD long long range_start_tab(const long long* tab, long long T, int C, int c) {
  return tab ? tab[c] : range_start(T, C, c);
}
TT_HD int range_of_tile_tab(const long long* tab, long long T, int C, long long x) {
  if (!tab) return range_of_tile(T, C, x);
  int lo = 0, hi = C - 1;  // the largest c with tab[c] <= x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= x) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

TT_HD int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Number of tiles of a unit whose visible context has L keys.
TT_HD int unit_tiles(int L, int key_tile) { return 1 + ceil_div(L, key_tile); }

// Per-range record the attention kernel leaves for the combine: the unit that
// is cut and begins in this range (or -1), the last range touching it, and
// the slot choice of this range's piece.
struct SplitRecord {
  int unit;
  int last_range;
  int first_which;
  int pad;
};

}  // namespace tt
