// Work tables shared by the host builder (dbuf.cu) and the kernels.
#pragma once

#include <cstdint>

namespace dbuf_k {

constexpr int kAlign = 16;             // tensor starts are multiples of 16 elements
constexpr int kTile = 4096;            // elements per tile / pipeline stage
constexpr int kMaxBlk = 254;           // whole blocks per WHOLE tile (scales fit one 2 KB copy)
constexpr int64_t kZeroChunk = 65536;  // elements per ZERO tile
constexpr int64_t kPackChunk = 16384;  // elements per copy-in CTA (32 KB)

constexpr int kMaxStripTiles = 256;    // quantisation tiles per STRIP entry

enum : int32_t { TILE_WHOLE = 0, TILE_LARGE = 1, TILE_ZERO = 2, TILE_STRIP = 3 };

// One entry of the step kernel's work table.
//   WHOLE: up to kMaxBlk whole blocks of one tensor, (e0 % 16) + n <= kTile.
//   LARGE: one block longer than that, streamed in kTile chunks, twice.
//   ZERO : a padding range; its bf16 copy is set to zero.
//   STRIP: columns [c0, c0 + n) of the rows of one k-row block of a tensor
//          quantised in tiles of `magic` columns (2-D blocks): e0 = element
//          (row 0, column c0), b = row stride (cols), nblk = rows, blk0 =
//          scale index of the strip's first tile, n <= kTile.  Streamed
//          twice in chunks of whole rows (several rows per chunk when
//          cols <= kTile, else one row's n columns).
struct Tile {
    int64_t e0;    // first bucket element
    int64_t blk0;  // index of the first block (scale index)
    int64_t n;     // elements (STRIP: columns)
    int32_t b;     // block size (WHOLE), row stride (STRIP), 0 otherwise
    int32_t kind;
    int32_t nblk;  // blocks in the entry (STRIP: rows)
    uint32_t magic;  // WHOLE with b >= 2: ceil(2^32 / b), so x / b == umulhi(x, magic) for x < 2^16;
                     // STRIP: tile width in columns
};
static_assert(sizeof(Tile) == 40, "tile layout");

// One CTA of the copy-in gather.
struct PackChunk {
    int64_t src_off;  // element offset in the source tensor
    int64_t dst_off;  // element offset in the bucket
    int32_t tensor;   // caller's tensor index
    int32_t count;    // elements
};

}  // namespace dbuf_k
