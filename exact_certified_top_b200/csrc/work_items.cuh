// Work items of the certified and filter scorers: tiles of 8 consecutive
// query rows of a chunk, longest rows first, and the processing order of the
// key tiles each item sees (tile 0, which holds the first seed keys, then from
// the diagonal tile downwards).
#pragma once

#include <stdint.h>

#include "dosa_internal.h"

namespace dosa {

constexpr int kItemQueries = 8;
// The epilogue warps meet (threshold refresh) every this many key tiles of an
// item and at the end of the item's range.
constexpr int kCkptTiles = 8;

struct Geom {
  int64_t t0;        // absolute first row
  int64_t local0;    // chunk-local first row
  int nq;            // valid queries in the item
  int64_t pos_first; // position of the first query
  int n_tiles;       // key tiles 0..n_tiles-1 hold every visible key
};

__device__ __forceinline__ Geom item_geometry(int64_t row0, int64_t rows, int64_t pos0, int n_items,
                                              int item) {
  Geom g;
  const int tile = n_items - 1 - item;        // longest rows first
  g.local0 = (int64_t)tile * kItemQueries;
  g.t0 = row0 + g.local0;
  const int64_t left = rows - g.local0;
  g.nq = (int)(left < kItemQueries ? left : kItemQueries);
  g.pos_first = pos0 + g.local0;
  g.n_tiles = (int)((g.pos_first + g.nq - 1) / kKeyTile) + 1;
  return g;
}

// Key tile processed at step ti of an item with n_tiles tiles.
__device__ __forceinline__ int tile_at(int ti, int n_tiles) {
  return ti == 0 ? 0 : n_tiles - ti;
}

// What the probe pass decided for an item (certified workspace flags): the
// filter scorer finishes it, or ranked screening does (rank_screen.cu,
// rescore.cu).  Before the decisions: kItemSample marks the items probed first
// (every kProbeSampleStride-th, longest rows first), and kItemProbe the others
// once the sample showed that screening pays somewhere; otherwise they become
// kItemUnprobed (filter scorer from the warm-up's end).
enum ItemFlag : int {
  kItemFilter = 1,
  kItemRank = 2,
  kItemSample = 4,
  kItemProbe = 5,
  kItemUnprobed = 6
};
// Every kProbeSampleStride-th item is sampled; on a chunk of more items than
// kProbeSampleStride * kProbeSampleItems the stride grows so that about
// kProbeSampleItems are (enough for the decision, and the sample's set-up and
// probe cost stops growing with the chunk).  The stride is prime and not 37,
// so that the sampled items spread evenly over the persistent CTAs (CTA b
// takes items b, b + grid, ...) for a grid of 148 or any other grid that is
// not a multiple of it.
constexpr int kProbeSampleStride = 7;
constexpr int kProbeSampleItems = 256;

inline int probe_stride(int n_items) {
  static const int kPrimes[] = {7, 11, 13, 17, 19, 23, 29, 31, 41, 43, 47, 53, 59, 61,
                                67, 71, 73, 79, 83, 89, 97, 101, 103, 107, 109, 113};
  const int want = (n_items + kProbeSampleItems - 1) / kProbeSampleItems;
  for (int pr : kPrimes)
    if (pr >= want) return pr;
  return 127;
}

struct Range {
  int begin, end;   // empty when end <= begin
};

__device__ __forceinline__ Range item_steps(const StepRange& sr, const int* item_flag,
                                            const Geom& g, int item) {
  Range r;
  r.begin = sr.begin;
  r.end = g.n_tiles < sr.end ? g.n_tiles : sr.end;
  if (sr.want_flag >= 0) {
    const int f = item_flag[item];
    if (sr.alt_flag > 0 && f == sr.alt_flag) r.begin = sr.alt_begin;
    else if (f != sr.want_flag) r.end = r.begin;
  }
  return r;
}

}  // namespace dosa
