// Internal definitions shared by the host plan builder and the CUDA kernels.
#pragma once
#include <stdint.h>

namespace rae {

constexpr int32_t kPlanMagic = 0x52414531;  // "RAE1"

// Kernel families chosen by the plan.
enum Kind : int32_t {
  kKindNone = 0,
  kKindDecodeSimt = 1,   // paged, <= 8 query rows per (request, KV head): CUDA cores, HBM bound
  kKindTcPaged = 2,      // paged, tcgen05 tiles of 128 query rows
  kKindTcRagged = 3,     // ragged spans, tcgen05 tiles of 128 query rows
  kKindTcPagedSwap = 4,  // paged, 9..64 query rows per unit, d = 128: keys on the MMA M side
};

// Plan image header (int32 words).
enum Hdr : int32_t {
  kHdrMagic = 0,
  kHdrKind = 1,
  kHdrNumTiles = 2,
  kHdrNumCtas = 3,
  kHdrNumMerge = 4,    // output rows merged from split partials (informational)
  kHdrBatch = 5,
  kHdrTotalQ = 6,
  kHdrBlockSize = 7,
  kHdrOffCtaPtr = 8,
  kHdrOffTiles = 9,
  kHdrSplitUnits = 10, // units whose keys were split (arrival counters used)
  kHdrOffA = 11,   // paged: qo_indptr [B+1]        ragged: cu_q [S+1]
  kHdrOffB = 12,   // paged: kv_len [B]             ragged: cu_kv [S+1]
  kHdrOffC = 13,   // paged: kv_page_indptr [B+1]   ragged: unused
  kHdrOffD = 14,   // paged: kv_page_indices [nnz]  ragged: unused
  kHdrRowsMax = 15,
  kHdrWords = 16,
};

// One work tile: query rows of one (request, KV head, query chunk) against a key range.
// Rows are ordered (token, head-in-group): row = tok * g + j.
struct Tile {
  int32_t req;        // request (paged) or span (ragged)
  int32_t kv_head;
  int32_t q0;         // first query token (global packed index)
  int32_t qn;         // query tokens in the tile
  int32_t kv0;        // first key (logical index within the request's keys)
  int32_t kv1;        // one past the last key of this tile
  int32_t part;       // -1: write out directly; else first partial row of this split
  int32_t split;      // split index within the unit (0 when unsplit)
  int32_t munit;      // split unit (index of its arrival counter); -1 when unsplit
  int32_t nsplit;     // splits of the unit (1 when unsplit)
  int32_t nkvh;       // KV heads of the unit: kv_head ... kv_head + nkvh - 1 (1 except decode)
  int32_t pad1;
};
static_assert(sizeof(Tile) == 48, "tile is 12 words");

// Work-unit block granularity in keys: the tcgen05 kernels step 128 keys at a time, the
// SIMT decode kernel 16 keys (one 16-row chunk of a page).
constexpr int32_t kTcBlockKeys = 128;
constexpr int32_t kSimtChunkKeys = 16;
constexpr int32_t kSimtMaxRows = 8;
// Most KV heads in a decode unit: one per consumer warp of the decode kernel, so that a
// 16-key chunk of a page is one contiguous run of the unit's heads (pool layout
// [pages, Hkv, P, d]).  A request's KV heads form units of this many, the last one fewer.
constexpr int32_t kSimtMaxHeads = 4;
constexpr int32_t kTcRows = 128;

// Workspace layout: [error words | slot 0 image | slot 1 image | write staging | partial O |
// partial lse | split arrival counters], every region 256-byte aligned.
constexpr int64_t kErrWordsBytes = 256;

}  // namespace rae
