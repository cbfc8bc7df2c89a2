// Host planner: group a batch's tokens by adapter and lay out the fused GEMM's
// augmented-K work.
//
// Grouping requests by adapter so the base GEMM runs batched while each
// adapter's xAB is computed for its own tokens without padding follows the
// batching section (批处理) of "S-LoRA：一个GPU运行数千大模型成为可能"; the
// rank-exact pool offsets follow its Unified Paging section (a rank-R weight
// occupies R vectors). Building the grouping once per batch and reusing it in
// every layer follows the decide-once framework (整体框架) of "AdaFuse:
// Accelerating Dynamic Adapter Inference via Token-Level Pre-Gating and Fused
// Kernel Optimization".
#include <algorithm>

#include "../../include/lora.h"
#include "internal.h"

namespace lora {

void append_aug_blocks(const ChunkDesc *chunks, int32_t nchunk, int32_t kaug, std::vector<AugBlockDesc> &out) {
  // for each 16-wide K step its B_pool rows (the hi and lo steps of a chunk read
  // the same rows); distinct row slices get slots
  int32_t c = 0;
  for (int32_t k0 = 0; k0 < kaug; k0 += kAugBlock) {
    AugBlockDesc ab{};
    const int32_t steps = std::min<int32_t>(4, (kaug - k0) / 16);
    int32_t nslot = 0, map = 0;
    for (int32_t q = 0; q < steps; ++q) {
      const int32_t kq = k0 + q * 16;
      while (c + 1 < nchunk && kq >= chunks[c].kofs + 2 * chunks[c].kc) ++c;
      const ChunkDesc &cd = chunks[c];
      int32_t o = kq - cd.kofs;
      if (o >= cd.kc) o -= cd.kc;
      const int32_t prow = cd.pool_row + o;
      int32_t sl = 0;
      while (sl < nslot && ab.prow[sl] != prow) ++sl;
      if (sl == nslot) {
        ab.valid |= std::min<int32_t>(16, cd.rank - o) << (5 * nslot);
        ab.prow[nslot++] = prow;
      }
      map |= sl << (2 * q);
    }
    ab.info = nslot | (map << 4) | (steps << 12);
    out.push_back(ab);
  }
}

// Empty every table of the plan but keep its storage: a rebuild for the next
// batch then allocates nothing once the tables have reached their sizes.
static void reset_plan(HostPlan &hp) {
  hp.perm.clear();
  hp.seg.clear();
  hp.offsets.clear();
  hp.tiles.clear();
  hp.chunks.clear();
  hp.units.clear();
  hp.augblocks.clear();
  hp.mt_order.clear();
  hp.pieces.clear();
  hp.partial_rows = 0;
  hp.r_max = 0;
  hp.sum_r_used = hp.sum_r_tokens = hp.aug_k_total = 0;
  hp.scratch_bytes = 0;
  hp.xs_offset = -1;
  hp.max_chunk_rows = 0;
}

int build_host_plan(const int32_t *ids, int64_t T, const int32_t *ranks, int32_t n_adapters,
                    int64_t d_in, int64_t d_out, HostPlan &hp) {
  if (!ids || !ranks || T <= 0 || n_adapters <= 0 || d_in < 8 || d_out < 8 || (d_in % 8) ||
      (d_out % 8))
    return LORA_ERR_ARG;
  if (T > (int64_t)1 << 30 || d_in > (int64_t)1 << 30 || d_out > (int64_t)1 << 30)
    return LORA_ERR_ARG;
  for (int32_t a = 0; a < n_adapters; ++a)
    if (ranks[a] < 1 || ranks[a] > LORA_MAX_RANK) return LORA_ERR_RANK;
  {
    // one unsigned compare per id (negative ids wrap above n_adapters), no early exit
    uint32_t bad = 0;
    for (int64_t t = 0; t < T; ++t) bad |= static_cast<uint32_t>(ids[t]) >= static_cast<uint32_t>(n_adapters);
    if (bad) return LORA_ERR_ID;
  }

  reset_plan(hp);
  hp.T = T;
  hp.d_in = d_in;
  hp.d_out = d_out;
  hp.n_adapters = n_adapters;

  hp.offsets.assign(n_adapters + 1, 0);
  for (int32_t a = 0; a < n_adapters; ++a) hp.offsets[a + 1] = hp.offsets[a] + ranks[a];
  if (hp.offsets[n_adapters] >= ((int64_t)1 << 31) - 256) return LORA_ERR_ARG;

  // Stable counting sort by adapter id (T < 2^30: positions fit int32). Both
  // passes walk runs of equal ids with the run's counter in a register: a
  // batch of whole requests has long runs, where one increment per token in
  // memory would wait on the previous one.
  static thread_local std::vector<int32_t> count, cursor;
  count.assign(n_adapters + 1, 0);
  for (int64_t t = 0; t < T;) {
    const int32_t a = ids[t];
    int64_t e = t + 1;
    while (e < T && ids[e] == a) ++e;
    count[a + 1] += static_cast<int32_t>(e - t);
    t = e;
  }
  for (int32_t a = 0; a < n_adapters; ++a) count[a + 1] += count[a];  // count[a] = start of a
  cursor.assign(count.begin(), count.end() - 1);
  hp.perm.resize(T);
  int32_t *perm = hp.perm.data();
  int32_t *cur = cursor.data();
  for (int64_t t = 0; t < T;) {
    const int32_t a = ids[t];
    int32_t c = cur[a];
    do perm[c++] = static_cast<int32_t>(t++);
    while (t < T && ids[t] == a);
    cur[a] = c;
  }

  // Segments, ascending adapter id, adapters without tokens skipped.
  hp.seg.reserve(3 * static_cast<size_t>(std::min<int64_t>(n_adapters, T)));
  for (int32_t a = 0; a < n_adapters; ++a) {
    int64_t len = count[a + 1] - count[a];
    if (len == 0) continue;
    hp.seg.push_back(a);
    hp.seg.push_back((int32_t)count[a]);
    hp.seg.push_back((int32_t)len);
    hp.r_max = std::max(hp.r_max, ranks[a]);
    hp.sum_r_used += ranks[a];
    hp.sum_r_tokens += (int64_t)ranks[a] * len;
  }
  const int32_t n_seg = (int32_t)(hp.seg.size() / 3);

  // Tiles of 128 sorted positions; each adapter run inside a tile is a chunk
  // whose K slice is twice the adapter's rank rounded up to the 16-wide MMA
  // step: s*U enters the MMA as bf16 hi + lo parts against the same B rows,
  // so the adapter term keeps ~16 mantissa bits whatever the scale.
  const int64_t n_tiles = (T + kTileM - 1) / kTileM;
  hp.tiles.reserve(n_tiles);
  hp.chunks.reserve(n_tiles + n_seg);  // a chunk per segment, plus one per tile boundary a segment crosses
  int32_t s = 0;  // current segment
  int64_t uofs = 0;
  for (int64_t m = 0; m < n_tiles; ++m) {
    TileDesc td{};
    td.row0 = (int32_t)(m * kTileM);
    td.rows = (int32_t)std::min<int64_t>(kTileM, T - m * kTileM);
    td.chunk0 = (int32_t)hp.chunks.size();
    int32_t kofs = 0;
    const int64_t r_end = td.row0 + td.rows;
    while (s < n_seg && hp.seg[3 * s + 1] < r_end) {
      const int32_t a = hp.seg[3 * s + 0];
      const int64_t s_beg = hp.seg[3 * s + 1];
      const int64_t s_end = s_beg + hp.seg[3 * s + 2];
      ChunkDesc cd{};
      cd.adapter = a;
      cd.pool_row = (int32_t)hp.offsets[a];
      cd.rank = ranks[a];
      cd.kc = (ranks[a] + 15) / 16 * 16;
      cd.kofs = kofs;
      cd.lo = (int32_t)(std::max<int64_t>(s_beg, td.row0) - td.row0);
      cd.hi = (int32_t)(std::min<int64_t>(s_end, r_end) - td.row0);
      cd.tile = (int32_t)m;
      kofs += 2 * cd.kc;  // bf16 hi part, then the bf16 lo part of s*U
      hp.max_chunk_rows = std::max(hp.max_chunk_rows, cd.hi - cd.lo);
      hp.chunks.push_back(cd);
      if (s_end <= r_end) ++s;  // segment finished inside this tile
      else break;               // segment continues into the next tile
    }
    td.nchunk = (int32_t)hp.chunks.size() - td.chunk0;
    td.kaug = kofs;
    // the tile's adapter K blocks
    td.aug0 = (int32_t)hp.augblocks.size();
    append_aug_blocks(hp.chunks.data() + td.chunk0, td.nchunk, td.kaug, hp.augblocks);
    // consecutive originals?
    bool contig = true;
    for (int32_t i = 1; i < td.rows && contig; ++i)
      contig = hp.perm[td.row0 + i] == hp.perm[td.row0] + i;
    td.contig = contig ? hp.perm[td.row0] : -1;
    td.uofs = uofs;
    uofs += (int64_t)((td.kaug + kAugBlock - 1) / kAugBlock) * kAugBlockBytes;
    hp.aug_k_total += td.kaug;
    hp.tiles.push_back(td);
  }
  // Tiles whose tokens are not consecutive originals read X through a sorted
  // copy that the row gather writes into the scratch before the shrink runs.
  bool any_gathered = false;
  for (const TileDesc &td : hp.tiles) any_gathered |= td.contig < 0;
  if (any_gathered) {
    hp.xs_offset = (uofs + 255) / 256 * 256;
    uofs = hp.xs_offset + T * d_in * 2;
  }
  hp.scratch_bytes = uofs;

  // Visiting order of m-tiles for the persistent GEMM: most augmented K first, so
  // the heavy tiles (many small adapters) start early instead of ending last.
  hp.mt_order.resize(hp.tiles.size());
  for (size_t m = 0; m < hp.tiles.size(); ++m) hp.mt_order[m] = (int32_t)m;
  std::stable_sort(hp.mt_order.begin(), hp.mt_order.end(),
                   [&](int32_t a, int32_t b) { return hp.tiles[a].kaug > hp.tiles[b].kaug; });

  // Shrink units: each chunk's rank columns in pieces of at most 64. When chunk
  // sizes are uneven (the largest has at least 4x the rows of the median, as
  // with a few popular adapters among many rare ones), chunk rows are also cut
  // into pieces of at most kUnitRows, so the big chunks do not set the length of
  // the whole kernel; even chunks stay whole (fewer re-reads of A).
  int32_t piece_rows = kTileM;
  if (!hp.chunks.empty()) {
    std::vector<int32_t> rows;
    rows.reserve(hp.chunks.size());
    for (const ChunkDesc &cd : hp.chunks) rows.push_back(cd.hi - cd.lo);
    const int32_t max_rows = *std::max_element(rows.begin(), rows.end());
    std::nth_element(rows.begin(), rows.begin() + rows.size() / 2, rows.end());
    const int32_t median = std::max(1, rows[rows.size() / 2]);
    if (max_rows >= 4 * median) piece_rows = kUnitRows;
  }
  for (int32_t c = 0; c < (int32_t)hp.chunks.size(); ++c) {
    const ChunkDesc &cd = hp.chunks[c];
    for (int32_t r0 = cd.lo; r0 < cd.hi; r0 += piece_rows) {
      for (int32_t n0 = 0; n0 < cd.kc; n0 += kShrinkN) {
        UnitDesc u{};
        u.chunk = c;
        u.n0 = n0;
        u.nn = std::min(kShrinkN, cd.kc - n0);
        u.last = (n0 + kShrinkN >= cd.kc) ? 1 : 0;
        u.r0 = r0;
        u.r1 = std::min(cd.hi, r0 + piece_rows);
        u.zero_fill = r0 == cd.lo ? 1 : 0;
        const TileDesc &td = hp.tiles[cd.tile];
        u.row0 = td.row0 + r0;
        u.contig = td.contig >= 0 ? td.contig + r0 : -1;
        u.frow = cd.pool_row + n0;
        u.nvalid = std::max(0, std::min(u.nn, cd.rank - n0));
        u.tile = cd.tile;
        u.clo = cd.lo;
        u.chi = cd.hi;
        u.kcol = cd.kofs + n0;
        u.kc = cd.kc;
        u.adapter = cd.adapter;
        u.uofs = td.uofs;
        hp.units.push_back(u);
      }
    }
  }
  // The backward's per-adapter contractions: each segment in pieces of at most
  // kPieceTokens sorted tokens, partial sums only for segments of several
  // pieces. Without a sorted copy of X the backward reads original rows, so a
  // piece is then also cut where the original index does not continue.
  for (int32_t sidx = 0; sidx < n_seg; ++sidx) {
    const int32_t a = hp.seg[3 * sidx], start = hp.seg[3 * sidx + 1], len = hp.seg[3 * sidx + 2];
    const int32_t first = (int32_t)hp.pieces.size();
    for (int32_t i = start; i < start + len;) {
      int32_t n = std::min<int32_t>(kPieceTokens, start + len - i);
      if (!any_gathered)
        for (int32_t j = 1; j < n; ++j)
          if (hp.perm[i + j] != hp.perm[i] + j) { n = j; break; }
      PieceDesc pd{};
      pd.start = i;
      pd.len = n;
      pd.in_row = any_gathered ? i : hp.perm[i];
      pd.adapter = a;
      pd.rank = ranks[a];
      pd.pool_row = (int32_t)hp.offsets[a];
      pd.first_piece = first;
      hp.pieces.push_back(pd);
      i += n;
    }
    const int32_t np = (int32_t)hp.pieces.size() - first;
    for (int32_t q = first; q < first + np; ++q) {
      hp.pieces[q].seg_pieces = np;
      hp.pieces[q].partial_row = np > 1 ? (int32_t)hp.partial_rows : -1;
      if (np > 1) hp.partial_rows += ranks[a];
    }
  }

  // Launch order, longest first: one CTA (or cluster) takes one unit, and
  // blocks start in index order as earlier ones finish, so the units with the
  // most rows and rank columns per 64-column block go in the first wave and
  // the short ones fill the tail. Units write disjoint parts of the image and
  // of U_save, so their order is free. The key (rows rounded up to 16, plus
  // the piece width) is at most kTileM + kShrinkN: a stable bucket sort by
  // decreasing key.
  {
    constexpr int kKeys = kTileM + kShrinkN + 1;
    // bucket of a unit: kKeys - 1 - key, so the largest key comes first (the
    // clamp only guards the arrays: rows <= kTileM and nn <= kShrinkN hold)
    auto bucket = [](const UnitDesc &u) {
      const int key = ((u.r1 - u.r0 + 15) / 16) * 16 + u.nn;
      return kKeys - 1 - std::min(std::max(key, 0), kKeys - 1);
    };
    int32_t start[kKeys + 1] = {};  // start[b + 1] counts bucket b, then the prefix sums
    for (const UnitDesc &u : hp.units) ++start[bucket(u) + 1];
    for (int k = 0; k < kKeys; ++k) start[k + 1] += start[k];
    static thread_local std::vector<UnitDesc> sorted;
    sorted.resize(hp.units.size());
    for (const UnitDesc &u : hp.units) sorted[start[bucket(u)]++] = u;
    hp.units.swap(sorted);
  }
  return LORA_OK;
}

}  // namespace lora
