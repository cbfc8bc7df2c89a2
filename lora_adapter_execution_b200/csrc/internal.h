// Host/device shared layout of a plan. Plain structs only (no CUDA types), so the
// host planner (plan.cpp, g++) and the kernels (lora_b200.cu, nvcc) agree on it.
#pragma once

#include <stdint.h>

#include <vector>

namespace lora {

constexpr int kTileM = 128;      // tokens per fused-GEMM output tile
constexpr int kAugBlock = 64;    // augmented-K columns per shrink-output block
constexpr int kAugBlockBytes = kTileM * kAugBlock * 2;  // 16 KB, one swizzled smem image
constexpr int kShrinkN = 64;     // rank columns per shrink work unit
constexpr int kUnitRows = 32;    // token rows per shrink work unit (a chunk's rows are split)
constexpr int kPieceTokens = 1024;  // tokens per piece of a segment in the backward's per-adapter contractions

// One 128-token output tile of the sorted order.
struct TileDesc {
  int32_t row0;    // first sorted position
  int32_t rows;    // valid rows (<= 128)
  int32_t chunk0;  // first ChunkDesc of this tile
  int32_t nchunk;  // adapters touching the tile
  int32_t kaug;    // augmented K = sum of the chunks' 2*kc (multiple of 32)
  int32_t contig;  // original index of row 0 if the tile's tokens are consecutive originals, else -1
  int64_t uofs;    // byte offset of the tile's s*U image in the plan scratch
  int32_t aug0;    // first AugBlockDesc of the tile (one per 64 augmented columns)
  int32_t pad_;
};

// One adapter K block of a tile (64 augmented columns, up to 4 MMA K steps of 16):
// the distinct 16-row slices of B_pool it reads and which slice each K step uses.
// Precomputed by the planner so the GEMM's copy-issuing thread only reads it.
struct AugBlockDesc {
  int32_t prow[4];  // first B_pool row of slot 0..nslot-1 (0 past nslot)
  int32_t info;     // nslot | slot of K step q at bits 4 + 2q | steps << 12
  int32_t valid;    // rows of slot u that belong to its adapter, 5 bits at bit 5u (1..16):
                    // the rest of the 16-row slice is another adapter's rows and is
                    // zeroed in shared memory before the MMA reads it
  int32_t pad_[2];
};

// One adapter's run of rows inside one tile: its K slice of the augmented contraction.
struct ChunkDesc {
  int32_t adapter;
  int32_t pool_row;  // off_a: first row of the adapter in A_pool / B_pool
  int32_t rank;      // r_a
  int32_t kc;        // r_a rounded up to 16 (MMA K step)
  int32_t kofs;      // first augmented-K column of the chunk within its tile (hi part;
                     // the lo part starts at kofs + kc)
  int32_t lo, hi;    // tile-local rows [lo, hi) owned by the adapter
  int32_t tile;
};

// Shrink work unit: rank columns [n0, n0+nn) of one chunk, over the chunk's
// tile-local rows [r0, r1) (at most kUnitRows: small units keep more stages of
// the shrink's ring in flight). The fields after zero_fill repeat what the unit's
// chunk and tile hold, so the shrink reads its whole geometry in one access.
struct alignas(16) UnitDesc {
  int32_t chunk;
  int32_t n0;
  int32_t nn;
  int32_t last;       // 1 if this is the chunk's last rank piece (it also zero-fills U_save up to r_max)
  int32_t r0, r1;     // tile-local rows
  int32_t zero_fill;  // 1: the unit also writes the zeros of its image columns in the
                      // tile rows outside the chunk (one row piece per chunk does)
  int32_t row0;       // sorted position of row r0 (tile row0 + r0)
  int32_t contig;     // original index of row r0 if the tile's tokens are consecutive, else -1
  int32_t frow;       // first A_pool row of the piece (the adapter's pool_row + n0)
  int32_t nvalid;     // columns of the piece that are real ranks
  int32_t tile;
  int32_t clo, chi;   // the chunk's tile-local rows
  int32_t kcol;       // augmented-K column of the piece's hi part (chunk kofs + n0)
  int32_t kc;         // the chunk's rank rounded up to 16 (hi-to-lo column distance)
  int32_t adapter;
  int32_t pad_;
  int64_t uofs;       // byte offset of the tile's s*U image in the plan scratch
};

// A piece of one segment (consecutive sorted tokens of one adapter) for the
// multi-adapter backward's contractions dA_a, dB_a: at most kPieceTokens tokens.
// A segment of one piece writes its adapter's gradient rows itself; the pieces
// of a longer segment write partial sums (partial_row = first row of this
// piece's r_a rows in the partial buffer) that a reduction adds in piece order.
struct alignas(16) PieceDesc {
  int32_t start, len;   // sorted positions
  int32_t in_row;       // row of the piece's first token in X / dY: its sorted position when the
                        // plan gathers (the backward reads sorted copies), else its original
                        // index (the piece is then a run of consecutive original tokens)
  int32_t adapter, rank, pool_row;
  int32_t seg_pieces;   // pieces of the segment (1: direct write)
  int32_t first_piece;  // index of the segment's first piece
  int32_t partial_row;  // -1 when seg_pieces == 1
  int32_t pad_[3];
};

// One term of a fused adapter switch: adapter rows [pool_row, pool_row + rank)
// of every layer's pools, weighted by coef, as augmented columns
// [kofs, kofs + 2*kc) of every tile (hi part, then lo part).
struct alignas(16) SwitchTerm {
  int32_t pool_row;
  int32_t rank;
  int32_t kc;    // rank rounded up to 16
  int32_t kofs;
  float coef;
  int32_t pad_[3];
};

struct HostPlan {
  int64_t T = 0, d_in = 0, d_out = 0;
  int32_t n_adapters = 0;
  std::vector<int32_t> perm;     // sorted position -> original token
  std::vector<int32_t> seg;      // n_seg x 3: adapter, start, length
  std::vector<int64_t> offsets;  // n_adapters + 1
  std::vector<TileDesc> tiles;
  std::vector<ChunkDesc> chunks;
  std::vector<UnitDesc> units;
  std::vector<AugBlockDesc> augblocks;
  std::vector<int32_t> mt_order;  // m-tiles by decreasing adapter work (stable)
  std::vector<PieceDesc> pieces;  // the backward's per-segment pieces, segment by segment
  int64_t partial_rows = 0;       // rows of the partial buffer (pieces of multi-piece segments)
  int32_t r_max = 0;
  int64_t sum_r_used = 0, sum_r_tokens = 0, aug_k_total = 0;
  int64_t scratch_bytes = 0;
  int64_t xs_offset = -1;  // byte offset of the sorted copy of X in the scratch (-1: not needed)
  int32_t max_chunk_rows = 0;
};

// The adapter K blocks of one tile whose chunks (consecutive, kofs ascending,
// each 2*kc augmented columns: hi part then lo part) span kaug columns.
void append_aug_blocks(const ChunkDesc *chunks, int32_t nchunk, int32_t kaug, std::vector<AugBlockDesc> &out);

// Returns LORA_OK or a LORA_ERR_* code; fills `hp` on success.
int build_host_plan(const int32_t *ids, int64_t T, const int32_t *ranks, int32_t n_adapters,
                    int64_t d_in, int64_t d_out, HostPlan &hp);

}  // namespace lora
