// Where a cache tile lives. A contiguous region keeps the tiles_per_seq tiles of each (sequence,
// head) together, pairs in row-major order. A paged region is a pool of pages of 64 tokens (two
// tiles) for every head, [pages][heads][2 tiles], and a caller-owned block table
// [batch][pages_per_seq] names the physical page of each 64-token page of a sequence -- the layout a
// serving system's page allocator hands out, where sequences that share a prefix can share its pages
// ("TurboQuant vs OSCAR vs EpiCache", OSCAR's fused kernels compatible with paged attention and the
// prefix cache).
#pragma once

namespace kvq {

constexpr int kStatusBadPage = 2;  // cache status bit: a block-table entry named no page of the pool

// Index of tile `tile` of (seq, head) among the region's tiles, or -1 when the block table's entry is
// not a page of the pool (the call then sets kStatusBadPage; readers use page 0 instead, writers skip).
__device__ __forceinline__ long tile_index(const int* table, int pages_per_seq, int n_pages, int tiles_per_seq,
                                          int heads, int seq, int head, int tile) {
  if (!table) return ((long)seq * heads + head) * tiles_per_seq + tile;
  const int page = __ldcg(table + (long)seq * pages_per_seq + (tile >> 1));
  if (page < 0 || page >= n_pages) return -1;
  return ((long)page * heads + head) * 2 + (tile & 1);
}

// A reader's tile: tile_index, with an invalid page replaced by page 0 (in bounds) and flagged.
__device__ __forceinline__ long tile_index_read(const int* table, int pages_per_seq, int n_pages, int tiles_per_seq,
                                               int heads, int seq, int head, int tile, int* err) {
  const long i = tile_index(table, pages_per_seq, n_pages, tiles_per_seq, heads, seq, head, tile);
  if (i >= 0) return i;
  atomicOr(err, kStatusBadPage);
  return (long)head * 2 + (tile & 1);
}

}  // namespace kvq
