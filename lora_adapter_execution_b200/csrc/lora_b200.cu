// C ABI of the multi-adapter LoRA linear layer (include/lora.h): plan lifecycle,
// argument validation, TMA descriptor encoding and kernel launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <limits>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>
#include <new>

#include "gemm.cuh"
#include "skinny.cuh"
#include "switch.cuh"
#include "tsqr.cuh"
#include "compress.cuh"

using namespace lora;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::atomic<bool> init{false};  // set once, after the fields below (release)
  int status = LORA_OK;
  int num_sms = 0;
  // the fused forward's cooperative launch: most CTAs resident at once in
  // clusters of S = 1, 2, 4 (index S)
  int fz_max_ctas[5] = {0, 0, 0, 0, 0};
};
DeviceState g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool qr_kernel_attributes();  // qr_api.inc

int device_state(DeviceState **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LORA_ERR_CUDA;
  DeviceState &d = g_dev[dev];
  if (!d.init.load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!d.init.load(std::memory_order_relaxed)) {
      int major = 0, minor = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        d.status = LORA_ERR_CUDA;
      } else if (major != 10 || minor != 0) {
        d.status = LORA_ERR_UNSUPPORTED;
      } else {
        d.status = LORA_OK;
        if (!g_encode) {
          cudaDriverEntryPointQueryResult q;
          void *fn = nullptr;
          if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
              q != cudaDriverEntryPointSuccess || !fn)
            d.status = LORA_ERR_CUDA;
          else
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
        }
        if (d.status == LORA_OK) {
          bool ok = true;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<false, kEpiStore>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<true, kEpiBwdLora>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBwd) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<false, kEpiMergeAdd>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<true, kEpiStore>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<false, kEpiStore, true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_gemm_kernel<true, kEpiBwdMulti>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_shrink_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sk_smem(4)) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_shrink_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     sk_smem(2)) == cudaSuccess;
          ok &= cudaFuncSetAttribute(lora_tcontract_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     tc_smem(kTcMaxR)) == cudaSuccess;
          ok &= qr_kernel_attributes();
          if (!ok) d.status = LORA_ERR_CUDA;
          for (int S = 1; ok && S <= 4; S *= 2) {
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3(static_cast<unsigned>(S));
            cfg.blockDim = dim3(kGemmThreads);
            cfg.dynamicSmemBytes = kGemmSmem;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = S;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, lora_gemm_kernel<false, kEpiStore, true>, &cfg) ==
                cudaSuccess)
              d.fz_max_ctas[S] = std::min(clusters * S, d.num_sms);
            else
              cudaGetLastError();  // no extra shrink CTAs then
          }
        }
      }
      d.init.store(true, std::memory_order_release);
    }
  }
  *out = &d;
  return d.status;
}

// 2-D bf16 tensor map over a row-major [rows x cols] matrix.
bool make_map(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, uint32_t box_cols,
              uint32_t box_rows, CUtensorMapSwizzle swz) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D fp32 tensor map over a row-major [rows x cols] matrix, no swizzle.
bool make_map_f32(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, uint32_t box_cols,
                  uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view {64, rows, cols / 64} of a row-major bf16 [rows x cols] matrix
// (cols % 64 == 0): one box {64, box_rows, blocks} copies `blocks` consecutive
// 64-column blocks of `box_rows` rows, each block stored as [box_rows][64].
bool make_map_blocks(CUtensorMap *m, const void *base, int64_t cols, int64_t rows, uint32_t box_rows,
                     uint32_t blocks) {
  cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(cols / 64)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * 2, 128};
  cuuint32_t box[3] = {64, box_rows, blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// m-tiles per group of the GEMM tile order: a group's 128-row blocks of A take
// about 16 MB, so they stay in L2 while its n-tiles run (on 8192 x 4096 x 11008
// this cut DRAM reads of the base GEMM from 853 MB to 428 MB; on 16384 x 4096 x
// 4096 from 1.9 GB to 283 MB).
int default_group_m(int n_mt, int64_t K) {
  const int64_t per_mtile = static_cast<int64_t>(kBM) * K * 2;
  const int64_t g = (16ll << 20) / per_mtile;
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g, n_mt)));
}

// Cluster size of the shrink (CTAs that split one unit's contraction): the
// choice in 1..4 with the least work on the critical path, counting whole waves
// of ctas_per_sm CTAs per SM (a second, mostly empty wave costs a full one) and,
// per CTA, its 64-column blocks plus a fixed cost of its setup and tail (about
// 2.8 us in per-CTA timelines, some 32 blocks' worth at ~0.09 us per block).
int shrink_split(int n_units, int64_t K, int num_sms, int ctas_per_sm, int64_t *cost_out = nullptr) {
  const int64_t kb = (K + kSkBK - 1) / kSkBK;
  const int64_t slots = static_cast<int64_t>(ctas_per_sm) * num_sms;
  int best = 1;
  int64_t best_cost = -1;
  for (int ks = 1; ks <= 4 && ks <= kb; ++ks) {
    const int64_t waves = (static_cast<int64_t>(n_units) * ks + slots - 1) / slots;
    const int64_t cost = waves * ((kb + ks - 1) / ks + 32);
    if (best_cost < 0 || cost < best_cost) {
      best = ks;
      best_cost = cost;
    }
  }
  if (cost_out) *cost_out = best_cost;
  return best;
}

// The shrink build for a launch: the small-piece build (three CTAs per SM, a
// smaller ring) when every piece allows it and it leaves no more stages on the
// critical path than the two-per-SM build. On a tie its third CTA per SM still
// pays: with the units launched longest first, the last wave holds only short
// units (590 units of at most 32 rows and rank columns: 59.4 -> 55.3 us).
int shrink_build(int n_units, int64_t K, int num_sms, int max_nn, int *ks_out) {
  int64_t cost_big = 0, cost_small = 0;
  const int ks_big = shrink_split(n_units, K, num_sms, sk_ctas_per_sm(4), &cost_big);
  if (max_nn <= 32) {
    const int ks_small = shrink_split(n_units, K, num_sms, sk_ctas_per_sm(2), &cost_small);
    if (cost_small <= cost_big) {
      *ks_out = ks_small;
      return 2;
    }
  }
  *ks_out = ks_big;
  return 4;
}

int launch_status() { return cudaGetLastError() == cudaSuccess ? LORA_OK : LORA_ERR_CUDA; }

// Forward GEMM launch: persistent CTAs when there are enough output tiles to
// fill the GPU; otherwise clusters of S CTAs split the K loop of each tile
// (S a power of two, S * tiles <= SMs, S <= number of K blocks).
int fwd_ksplit(int n_tiles, int KB, int num_sms) {
  int S = 1;
  while (S < 4 && 2 * S * n_tiles <= num_sms && 2 * S <= KB) S *= 2;  // S in {1, 2, 4}
  return S;
}

// Tiles of the persistent fused GEMM per CTA: in the kernel's visiting order,
// each tile goes to the CTA with the least estimated work so far (greedy list
// scheduling). A tile costs its base K blocks plus 1.3x its adapter K blocks
// (per-CTA timings: an adapter block takes about 1.3 times a base block). With
// equal costs this is the round robin the kernel would do by itself; with the
// uneven adapter work of many small adapters per tile it evens out the CTAs'
// loads. Output: off[grid + 1] then the tile indices, CTA by CTA, or nothing
// when the round robin is about as even.
void build_schedule(const HostPlan &hp, int grid, int group_m, std::vector<int32_t> &out) {
  const int n_mt = static_cast<int>(hp.tiles.size());
  const int n_nt = static_cast<int>((hp.d_out + kBN - 1) / kBN);
  const int KB = static_cast<int>((hp.d_in + kBK - 1) / kBK);
  const int n_tiles = n_mt * n_nt;
  out.clear();
  if (grid <= 0 || grid > 65535 || n_tiles <= 0) return;
  // per m-tile cost; the visiting order of tile_mn walked group by group (n
  // index outer, m index inner inside a group), so no division per tile
  std::vector<int64_t> mcost(n_mt);
  for (int mt = 0; mt < n_mt; ++mt) mcost[mt] = 10 * KB + 13 * ((hp.tiles[mt].kaug + kAugBlock - 1) / kAugBlock);
  // the round robin's loads first: when even a perfect split of whole tiles
  // (at least the mean, the largest tile, and ceil(tiles / CTAs) of the
  // cheapest tiles on one CTA) could not beat its heaviest CTA by 2 % the
  // greedy pass is skipped (nearly uniform tiles: fine-tuning, prefill)
  std::vector<int64_t> rr(grid, 0);
  int64_t total = 0, cmax = 0, cmin = std::numeric_limits<int64_t>::max();
  {
    int brr = 0;
    for (int m0 = 0; m0 < n_mt; m0 += group_m) {
      const int gm = std::min(group_m, n_mt - m0);
      for (int nt = 0; nt < n_nt; ++nt)
        for (int r = 0; r < gm; ++r) {
          const int mi = m0 + r;
          const int64_t c = mcost[hp.mt_order.empty() ? mi : hp.mt_order[mi]];
          rr[brr] += c;
          total += c;
          cmax = std::max(cmax, c);
          cmin = std::min(cmin, c);
          if (++brr == grid) brr = 0;
        }
    }
  }
  const int64_t rr_max = *std::max_element(rr.begin(), rr.end());
  const int64_t bound =
      std::max({cmax, (total + grid - 1) / grid, static_cast<int64_t>((n_tiles + grid - 1) / grid) * cmin});
  if (bound * 100 > rr_max * 98) return;
  // the loads as a binary min-heap of (work << 16 | CTA): ties go to the lowest CTA
  std::vector<uint64_t> heap(grid);
  for (int b = 0; b < grid; ++b) heap[b] = static_cast<uint64_t>(b);
  std::vector<int32_t> owner(n_tiles);
  int t = 0;
  for (int m0 = 0; m0 < n_mt; m0 += group_m) {
    const int gm = std::min(group_m, n_mt - m0);
    for (int nt = 0; nt < n_nt; ++nt)
      for (int r = 0; r < gm; ++r, ++t) {
        const int mi = m0 + r;
        const int64_t c = mcost[hp.mt_order.empty() ? mi : hp.mt_order[mi]];
        // the least loaded CTA takes tile t; its load grows: sift the top down
        const uint64_t top = heap[0];
        owner[t] = static_cast<int32_t>(top & 0xFFFFu);
        const uint64_t v = top + (static_cast<uint64_t>(c) << 16);
        int h = 0;
        while (true) {
          const int l = 2 * h + 1;
          if (l >= grid) break;
          const int m = (l + 1 < grid && heap[l + 1] < heap[l]) ? l + 1 : l;
          if (heap[m] >= v) break;
          heap[h] = heap[m];
          h = m;
        }
        heap[h] = v;
      }
  }
  // keep it only where it shortens the heaviest CTA by more than 2 % against the
  // round robin (whose tile order keeps more operands shared through L2)
  int64_t greedy_max = 0;
  for (uint64_t v : heap) greedy_max = std::max<int64_t>(greedy_max, static_cast<int64_t>(v >> 16));
  if (greedy_max * 100 > rr_max * 98) return;
  out.assign(grid + 1 + n_tiles, 0);
  for (int u = 0; u < n_tiles; ++u) ++out[owner[u] + 1];
  for (int b = 0; b < grid; ++b) out[b + 1] += out[b];
  std::vector<int32_t> pos(out.begin(), out.begin() + grid);
  for (int u = 0; u < n_tiles; ++u) out[grid + 1 + pos[owner[u]]++] = u;
}

int launch_fwd_gemm(DeviceState *ds, GemmParams gp, const CUtensorMap &a, const CUtensorMap &b,
                    const CUtensorMap &bl, lora_stream_t stream) {
  const int n_tiles = gp.n_mt * gp.n_nt;
  const int KB = (gp.K + kBK - 1) / kBK;
  gp.group_m = default_group_m(gp.n_mt, gp.K);
  const int S = fwd_ksplit(n_tiles, KB, ds->num_sms);
  gp.ksplit = S;
  if (S > 1) gp.sched_off = gp.sched_tiles = nullptr;  // one tile per cluster
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(S == 1 ? std::min(ds->num_sms, n_tiles) : n_tiles * S));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = stream;
  // programmatic serialization: the GEMM's setup overlaps the end of the
  // kernel before it (the shrink), whose results it waits for in pdl_wait
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S == 1 ? 1 : 2;
  if (cudaLaunchKernelEx(&cfg, lora_gemm_kernel<false, kEpiStore>, a, b, bl, a, a, a, gp) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

}  // namespace

struct lora_plan {
  HostPlan hp;
  HostPlan spare;  // the table set a rebuild fills before it swaps it in (storage kept across batches)
  void *dev = nullptr;       // perm | tiles | chunks | units
  uint8_t *scratch = nullptr;
  const int32_t *d_perm = nullptr;
  const TileDesc *d_tiles = nullptr;
  const ChunkDesc *d_chunks = nullptr;
  const UnitDesc *d_units = nullptr;
  const int32_t *d_mt_order = nullptr;
  const AugBlockDesc *d_augblocks = nullptr;
  const PieceDesc *d_pieces = nullptr;
  std::vector<int32_t> sched;           // the fused GEMM's per-CTA tiles (build_schedule), if persistent
  const int32_t *d_sched = nullptr;     // off[grid + 1] | tiles
  // the fused forward's launch (lora_linear_fwd_fused): its grid, the shrink
  // units of each CTA (off[grid + 1] | units), units per m-tile, and its counters
  // (per m-tile, then the row-copy count), zeroed before each launch
  int fz_grid = 0;
  int fz_gemm_ctas = 0;  // the first fz_gemm_ctas CTAs run GEMM tiles, the others only shrink units
  std::vector<int32_t> fz_tab;          // off[grid + 1] | units | need[n_mt]
  const int32_t *d_fz_off = nullptr, *d_fz_units = nullptr, *d_fz_need = nullptr;
  int32_t *d_fz_cnt = nullptr;
  // the multi-adapter backward's contraction: its pieces dealt into contiguous
  // ranges of about equal stage counts, one range per grid row (off[P + 1])
  std::vector<int32_t> ranges;
  const int32_t *d_ranges = nullptr;
  void *stage[2] = {nullptr, nullptr};  // pinned host staging of the tables, used in turn
  size_t stage_cap[2] = {0, 0};
  cudaEvent_t stage_ev[2] = {nullptr, nullptr};  // the last copy out of each staging buffer
  int stage_next = 0;
  int xws_S = 0;          // split of the fused GEMM whose exchange workspace the scratch holds (0: none)
  size_t xws_offset = 0;  // its byte offset in the scratch
  size_t dev_cap = 0, scratch_cap = 0;  // allocated bytes (a rebuild reuses them when they fit)
  int device = 0;
};

namespace {
// A plan's tables and scratch live on the device that was current when it was
// built; calls on any other device are rejected.
bool on_plan_device(const lora_plan *pl) {
  int d = -1;
  return cudaGetDevice(&d) == cudaSuccess && d == pl->device;
}

// The shrink over the plan's units (one CTA cluster per unit): In rows by mIn
// (box {64, 16}), factor rows by mF (box {64, 16}), sp.K the contraction length;
// the caller fills the rest of sp (scale, mask, outputs). Launched with
// programmatic stream serialization.
int launch_unit_shrink(DeviceState *ds, const lora_plan *plan, const CUtensorMap &mIn, const CUtensorMap &mF,
                       const CUtensorMap &mBits, ShrinkParams sp, lora_stream_t stream) {
  const HostPlan &hp = plan->hp;
  sp.mode = 0;
  sp.T = static_cast<int32_t>(hp.T);
  const int n_units = static_cast<int>(hp.units.size());
  // the build (and cluster size) with the fewest stages on the critical path
  int max_nn = 0;
  for (const UnitDesc &u : hp.units) max_nn = std::max(max_nn, static_cast<int>(u.nn));
  int ks = 1;
  const int max_nb16 = shrink_build(n_units, sp.K, ds->num_sms, max_nn, &ks);
  int64_t slice = (sp.K + ks - 1) / ks;
  slice = (slice + kSkBK - 1) / kSkBK * kSkBK;
  sp.ksplit = ks;
  sp.kslice = static_cast<int32_t>(slice);
  sp.units = plan->d_units;
  sp.chunks = plan->d_chunks;
  sp.tiles = plan->d_tiles;
  sp.perm = plan->d_perm;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(n_units * ks));
  cfg.blockDim = dim3(kSkThreads);
  cfg.dynamicSmemBytes = sk_smem(max_nb16);
  cfg.stream = stream;
  // programmatic serialization: the shrink's setup (barriers, its plan entry)
  // overlaps the end of the kernel before it; it waits in pdl_wait before
  // touching its inputs or any output
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, max_nb16 <= 2 ? lora_shrink_kernel<2> : lora_shrink_kernel<4>, mIn, mF, mBits,
                         sp) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}
}  // namespace

extern "C" {

const char *lora_status_string(int code) {
  switch (code) {
    case LORA_OK: return "ok";
    case LORA_ERR_ARG: return "invalid argument";
    case LORA_ERR_ID: return "adapter id out of range";
    case LORA_ERR_RANK: return "rank out of range";
    case LORA_ERR_CUDA: return "CUDA error";
    case LORA_ERR_DEVICE: return "device status word set (bounds or wait timeout)";
    case LORA_ERR_UNSUPPORTED: return "device is not sm_100";
    case LORA_ERR_NOMEM: return "out of memory";
    case LORA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace {
// Device side of a plan: (re)allocate its table block and scratch when they are
// smaller than the plan needs (kept otherwise, so a rebuilt plan reuses them),
// then upload the tables. Returns LORA_OK or an error; on error the plan keeps
// no device memory.
// sync: wait until the tables are on the device before returning.
int upload_plan(lora_plan *pl, lora_stream_t stream, bool sync) {
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  cudaGetDevice(&pl->device);
  const HostPlan &hp = pl->hp;
  auto up = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
  const size_t b_perm = up(sizeof(int32_t) * hp.perm.size());
  const size_t b_tiles = up(sizeof(TileDesc) * hp.tiles.size());
  const size_t b_chunks = up(sizeof(ChunkDesc) * hp.chunks.size());
  const size_t b_units = up(sizeof(UnitDesc) * hp.units.size());
  const size_t b_order = up(sizeof(int32_t) * hp.mt_order.size());
  const size_t b_aug = up(sizeof(AugBlockDesc) * hp.augblocks.size());
  const size_t b_pieces = up(sizeof(PieceDesc) * hp.pieces.size());
  // the persistent fused GEMM's tile schedule (its grid and tile order as launched)
  pl->sched.clear();
  {
    const int n_mt = static_cast<int>(hp.tiles.size());
    const int n_tiles = n_mt * static_cast<int>((hp.d_out + kBN - 1) / kBN);
    const int KB = static_cast<int>((hp.d_in + kBK - 1) / kBK);
    if (n_tiles > 0 && fwd_ksplit(n_tiles, KB, ds->num_sms) == 1)
      build_schedule(hp, std::min(ds->num_sms, n_tiles), default_group_m(n_mt, hp.d_in), pl->sched);
  }
  const size_t b_sched = up(sizeof(int32_t) * pl->sched.size());
  // the fused forward: units dealt to the launch's CTAs in the plan's order
  // (longest first), round robin; units per m-tile
  pl->fz_tab.clear();
  pl->fz_grid = 0;
  {
    const int n_mt = static_cast<int>(hp.tiles.size());
    const int n_tiles = n_mt * static_cast<int>((hp.d_out + kBN - 1) / kBN);
    const int KB = static_cast<int>((hp.d_in + kBK - 1) / kBK);
    if (n_tiles > 0) {
      const int S = fwd_ksplit(n_tiles, KB, ds->num_sms);
      const int Gg = S == 1 ? std::min(ds->num_sms, n_tiles) : n_tiles * S;
      const int nu = static_cast<int>(hp.units.size());
      // CTAs the GEMM leaves free (whole clusters, within what can be resident
      // at once) take the units, so the GEMM CTAs start their K loops at once;
      // with no room every CTA runs units first
      int Gx = std::max(0, std::min(ds->fz_max_ctas[S] - Gg, (nu + S - 1) / S * S));
      Gx = Gx / S * S;
      const int G = Gg + Gx;
      // the unit-only CTAs take the units when there are enough of them for
      // about two each; otherwise every CTA takes units, the unit-only ones first
      const bool only = Gx > 0 && 2 * Gx >= nu;
      const int nw = only ? Gx : G;  // the CTAs that take units
      pl->fz_grid = G;
      pl->fz_gemm_ctas = Gg;
      pl->fz_tab.assign(G + 1 + nu + n_mt, 0);
      // dealing position w of CTA b: the unit-only CTAs come first in the
      // rotation, so with every CTA taking units they get the extra ones
      auto pos = [&](int b) { return only ? b - Gg : (b >= Gg ? b - Gg : b + Gx); };
      for (int b = 0; b < G; ++b) {
        const int w = pos(b);
        pl->fz_tab[b + 1] = pl->fz_tab[b] + ((w >= 0 && w < nw) ? (nu - w + nw - 1) / nw : 0);
      }
      for (int b = 0; b < G; ++b) {
        const int w = pos(b);
        if (w < 0 || w >= nw) continue;
        for (int u = w, j = pl->fz_tab[b]; u < nu; u += nw, ++j) pl->fz_tab[G + 1 + j] = u;
      }
      for (int u = 0; u < nu; ++u) ++pl->fz_tab[G + 1 + nu + hp.units[u].tile];
    }
  }
  const size_t b_fz = up(sizeof(int32_t) * pl->fz_tab.size());
  // about two CTAs per SM over the wider of the two contractions' column blocks
  pl->ranges.clear();
  {
    const int np = static_cast<int>(hp.pieces.size());
    const int64_t cols = (std::max(hp.d_in, hp.d_out) + kTcCols - 1) / kTcCols;
    const int P = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(std::max(np, 1), (2 * ds->num_sms + cols / 2) / std::max<int64_t>(1, cols))));
    int64_t total = 0;
    for (const PieceDesc &pd : hp.pieces) total += (pd.len + kTcTok - 1) / kTcTok;
    pl->ranges.assign(P + 1, np);
    pl->ranges[0] = 0;
    int64_t cum = 0;
    int k = 1;
    for (int i = 0; i < np && k < P; ++i) {
      cum += (hp.pieces[i].len + kTcTok - 1) / kTcTok;
      while (k < P && cum * P >= total * k) pl->ranges[k++] = i + 1;
    }
  }
  const size_t b_rng = up(sizeof(int32_t) * pl->ranges.size());
  const size_t b_fzc = up(sizeof(int32_t) * (hp.tiles.size() + 1));
  const size_t total = b_perm + b_tiles + b_chunks + b_units + b_order + b_aug + b_pieces + b_sched + b_fz + b_fzc +
                       b_rng;
  auto release = [&]() {
    if (pl->dev) cudaFree(pl->dev);
    if (pl->scratch) cudaFree(pl->scratch);
    pl->dev = nullptr;
    pl->scratch = nullptr;
    pl->dev_cap = 0;
    pl->scratch_cap = 0;
  };
  if (total > pl->dev_cap) {
    if (pl->dev) cudaFree(pl->dev);
    pl->dev = nullptr;
    pl->dev_cap = 0;
    if (cudaMalloc(&pl->dev, total) != cudaSuccess) {
      cudaGetLastError();
      release();
      return LORA_ERR_NOMEM;
    }
    pl->dev_cap = total;
  }
  // a split-K fused GEMM exchanges its partial sums through a workspace behind
  // the scratch's images (and sorted X): [tiles][S][S] slots of xslot_bytes(S)
  pl->xws_S = 0;
  pl->xws_offset = 0;
  size_t scratch_total = static_cast<size_t>(hp.scratch_bytes);
  {
    const int n_tiles = static_cast<int>(hp.tiles.size()) * static_cast<int>((hp.d_out + kBN - 1) / kBN);
    const int KB = static_cast<int>((hp.d_in + kBK - 1) / kBK);
    const int S = n_tiles > 0 ? fwd_ksplit(n_tiles, KB, ds->num_sms) : 1;
    if (S > 1) {
      pl->xws_S = S;
      pl->xws_offset = up(scratch_total);
      scratch_total = pl->xws_offset + static_cast<size_t>(n_tiles) * S * S * xslot_bytes(S);
    }
  }
  if (scratch_total > pl->scratch_cap) {
    if (pl->scratch) cudaFree(pl->scratch);
    pl->scratch = nullptr;
    pl->scratch_cap = 0;
    if (cudaMalloc(reinterpret_cast<void **>(&pl->scratch), scratch_total) != cudaSuccess) {
      cudaGetLastError();
      release();
      return LORA_ERR_NOMEM;
    }
    pl->scratch_cap = scratch_total;
  }
  uint8_t *base = static_cast<uint8_t *>(pl->dev);
  pl->d_perm = reinterpret_cast<const int32_t *>(base);
  pl->d_tiles = reinterpret_cast<const TileDesc *>(base + b_perm);
  pl->d_chunks = reinterpret_cast<const ChunkDesc *>(base + b_perm + b_tiles);
  pl->d_units = reinterpret_cast<const UnitDesc *>(base + b_perm + b_tiles + b_chunks);
  pl->d_mt_order = reinterpret_cast<const int32_t *>(base + b_perm + b_tiles + b_chunks + b_units);
  pl->d_augblocks =
      reinterpret_cast<const AugBlockDesc *>(base + b_perm + b_tiles + b_chunks + b_units + b_order);
  uint8_t *pieces_dst = base + b_perm + b_tiles + b_chunks + b_units + b_order + b_aug;
  pl->d_pieces = reinterpret_cast<const PieceDesc *>(pieces_dst);
  uint8_t *sched_dst = pieces_dst + b_pieces;
  pl->d_sched = pl->sched.empty() ? nullptr : reinterpret_cast<const int32_t *>(sched_dst);
  uint8_t *fz_dst = sched_dst + b_sched;
  {
    const int G = pl->fz_grid, nu = static_cast<int>(hp.units.size());
    const int32_t *f = reinterpret_cast<const int32_t *>(fz_dst);
    pl->d_fz_off = f;
    pl->d_fz_units = f + G + 1;
    pl->d_fz_need = f + G + 1 + nu;
    pl->d_fz_cnt = reinterpret_cast<int32_t *>(fz_dst + b_fz);
  }
  uint8_t *rng_dst = fz_dst + b_fz + b_fzc;
  pl->d_ranges = reinterpret_cast<const int32_t *>(rng_dst);
  // The tables go to the device in one copy from one of the plan's two pinned
  // staging buffers, laid out as the device buffer. A staging buffer is refilled
  // only after its previous copy has completed (its event), so consecutive
  // rebuilds need no stream synchronisation.
  bool ok = true;
  const int k = pl->stage_next;
  if (pl->stage_ev[k]) ok &= cudaEventSynchronize(pl->stage_ev[k]) == cudaSuccess;
  else ok &= cudaEventCreateWithFlags(&pl->stage_ev[k], cudaEventDisableTiming) == cudaSuccess;
  if (ok && total > pl->stage_cap[k]) {
    if (pl->stage[k]) cudaFreeHost(pl->stage[k]);
    pl->stage[k] = nullptr;
    pl->stage_cap[k] = 0;
    if (cudaHostAlloc(&pl->stage[k], total, cudaHostAllocDefault) != cudaSuccess) {
      cudaGetLastError();
      release();
      return LORA_ERR_NOMEM;
    }
    pl->stage_cap[k] = total;
  }
  if (ok) {
    uint8_t *h = static_cast<uint8_t *>(pl->stage[k]);
    auto put = [&](size_t off, const void *src, size_t bytes) {
      if (bytes) std::memcpy(h + off, src, bytes);
    };
    put(0, hp.perm.data(), sizeof(int32_t) * hp.perm.size());
    put(b_perm, hp.tiles.data(), sizeof(TileDesc) * hp.tiles.size());
    put(b_perm + b_tiles, hp.chunks.data(), sizeof(ChunkDesc) * hp.chunks.size());
    put(b_perm + b_tiles + b_chunks, hp.units.data(), sizeof(UnitDesc) * hp.units.size());
    put(b_perm + b_tiles + b_chunks + b_units, hp.mt_order.data(), sizeof(int32_t) * hp.mt_order.size());
    put(b_perm + b_tiles + b_chunks + b_units + b_order, hp.augblocks.data(),
        sizeof(AugBlockDesc) * hp.augblocks.size());
    put(static_cast<size_t>(pieces_dst - base), hp.pieces.data(), sizeof(PieceDesc) * hp.pieces.size());
    put(static_cast<size_t>(sched_dst - base), pl->sched.data(), sizeof(int32_t) * pl->sched.size());
    put(static_cast<size_t>(fz_dst - base), pl->fz_tab.data(), sizeof(int32_t) * pl->fz_tab.size());
    put(static_cast<size_t>(rng_dst - base), pl->ranges.data(), sizeof(int32_t) * pl->ranges.size());
    ok &= cudaMemcpyAsync(base, h, total, cudaMemcpyHostToDevice, stream) == cudaSuccess;
    ok &= cudaEventRecord(pl->stage_ev[k], stream) == cudaSuccess;
    pl->stage_next = k ^ 1;
  }
  if (ok && sync) ok &= cudaStreamSynchronize(stream) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    release();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}
}  // namespace

extern "C" {

int lora_plan_build(const int32_t *ids_host, int64_t T, const int32_t *ranks_host, int32_t n_adapters,
                    int64_t d_in, int64_t d_out, lora_stream_t stream, lora_plan_t *out) {
  if (!out) return LORA_ERR_ARG;
  lora_plan *pl = new (std::nothrow) lora_plan();
  if (!pl) return LORA_ERR_NOMEM;
  int rc = build_host_plan(ids_host, T, ranks_host, n_adapters, d_in, d_out, pl->hp);
  if (rc == LORA_OK) rc = upload_plan(pl, stream, true);
  if (rc != LORA_OK) {
    lora_plan_destroy(pl);  // also frees the staging buffers and events an upload made
    return rc;
  }
  *out = pl;
  return LORA_OK;
}

int lora_plan_rebuild(lora_plan_t plan, const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                      int32_t n_adapters, int64_t d_in, int64_t d_out, lora_stream_t stream) {
  if (!plan || !plan->dev || !on_plan_device(plan)) return LORA_ERR_ARG;
  // the new tables go into the spare set (the previous batch's storage, reused)
  int rc = build_host_plan(ids_host, T, ranks_host, n_adapters, d_in, d_out, plan->spare);
  if (rc != LORA_OK) return rc;  // the plan is unchanged
  std::swap(plan->hp, plan->spare);
  return upload_plan(plan, stream, false);
}

int lora_plan_build_host(const int32_t *ids_host, int64_t T, const int32_t *ranks_host, int32_t n_adapters,
                         int64_t d_in, int64_t d_out, lora_plan_t *out) {
  if (!out) return LORA_ERR_ARG;
  lora_plan *pl = new (std::nothrow) lora_plan();
  if (!pl) return LORA_ERR_NOMEM;
  const int rc = build_host_plan(ids_host, T, ranks_host, n_adapters, d_in, d_out, pl->hp);
  if (rc != LORA_OK) {
    delete pl;
    return rc;
  }
  *out = pl;
  return LORA_OK;
}

int lora_plan_get(lora_plan_t plan, int32_t *perm_host, int32_t *seg_host, int32_t *n_seg) {
  if (!plan) return LORA_ERR_ARG;
  const HostPlan &hp = plan->hp;
  if (perm_host) std::memcpy(perm_host, hp.perm.data(), sizeof(int32_t) * hp.perm.size());
  if (seg_host) std::memcpy(seg_host, hp.seg.data(), sizeof(int32_t) * hp.seg.size());
  if (n_seg) *n_seg = static_cast<int32_t>(hp.seg.size() / 3);
  return LORA_OK;
}

int lora_plan_info(lora_plan_t plan, lora_plan_info_t *info) {
  if (!plan || !info) return LORA_ERR_ARG;
  const HostPlan &hp = plan->hp;
  info->T = hp.T;
  info->d_in = hp.d_in;
  info->d_out = hp.d_out;
  info->n_adapters = hp.n_adapters;
  info->n_segments = static_cast<int32_t>(hp.seg.size() / 3);
  info->n_tiles = static_cast<int32_t>(hp.tiles.size());
  info->r_max = hp.r_max;
  info->sum_r_used = hp.sum_r_used;
  info->sum_r_tokens = hp.sum_r_tokens;
  info->aug_k_total = hp.aug_k_total;
  info->scratch_bytes = hp.scratch_bytes;
  info->gathers_x = hp.xs_offset >= 0 ? 1 : 0;
  return LORA_OK;
}

void lora_plan_destroy(lora_plan_t plan) {
  if (!plan) return;
  for (int k = 0; k < 2; ++k) {
    if (plan->stage_ev[k]) {
      cudaEventSynchronize(plan->stage_ev[k]);  // its copy may still read the staging buffer
      cudaEventDestroy(plan->stage_ev[k]);
    }
    if (plan->stage[k]) cudaFreeHost(plan->stage[k]);
  }
  if (plan->dev) cudaFree(plan->dev);
  if (plan->scratch) cudaFree(plan->scratch);
  delete plan;
}

int lora_linear_shrink(lora_plan_t plan, const uint16_t *X, const uint16_t *A_pool, const float *scale,
                       double p_drop, uint64_t seed, float *U_save, const uint32_t *keep_bits,
                       lora_stream_t stream) {
  if (!plan || !plan->dev || !X || !A_pool || !scale) return LORA_ERR_ARG;
  if (!on_plan_device(plan)) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(A_pool)) return LORA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(keep_bits) & 3u) return LORA_ERR_ARG;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  const HostPlan &hp = plan->hp;
  const int64_t R = hp.offsets[hp.n_adapters];
  CUtensorMap mX16, mA16;
  uint16_t *Xs = hp.xs_offset >= 0 ? reinterpret_cast<uint16_t *>(plan->scratch + hp.xs_offset) : nullptr;
  bool ok = true;
  ok &= make_map(&mX16, Xs ? Xs : X, hp.d_in, hp.T, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mA16, A_pool, hp.d_in, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return LORA_ERR_ARG;
  ShrinkParams sp{};
  sp.mode = 0;
  sp.K = static_cast<int32_t>(hp.d_in);
  sp.scale = scale;
  sp.thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  sp.keep_bits = sp.thr ? keep_bits : nullptr;  // no mask without dropout
  sp.wpr = (hp.d_in + 31) / 32;
  // units of consecutive tokens copy their keep bits with each stage when the
  // bit array's rows are 16-byte multiples (d_in % 128 == 0)
  CUtensorMap mBits16 = mX16;
  if (sp.keep_bits && sp.wpr % 4 == 0) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(sp.wpr), static_cast<cuuint64_t>(hp.T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(sp.wpr) * 4};
    cuuint32_t box[2] = {4, 16};
    cuuint32_t estr[2] = {1, 1};
    sp.bits_tma = g_encode(&mBits16, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(sp.keep_bits), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    if (!sp.bits_tma) mBits16 = mX16;
  }
  sp.seed = seed;
  sp.inv_keep = p_drop > 0.0 ? static_cast<float>(1.0 / (1.0 - p_drop)) : 1.0f;
  sp.uimg = plan->scratch;
  sp.x_sorted = Xs ? 1 : 0;
  sp.U_save = U_save;
  sp.r_max = hp.r_max;
  if (Xs) {
    // sorted copy of X first (the shrink and the fused GEMM read token tiles from it)
    const int64_t pieces = hp.T * (hp.d_in / 8);
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((pieces + 255) / 256, 8 * ds->num_sms));
    lora_gather_rows_kernel<<<blocks, 256, 0, stream>>>(X, plan->d_perm, Xs, hp.T, hp.d_in);
    if (cudaGetLastError() != cudaSuccess) return LORA_ERR_CUDA;
  }
  return launch_unit_shrink(ds, plan, mX16, mA16, mBits16, sp, stream);
}

int lora_fused_gemm(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *B_pool, uint16_t *Y,
                    lora_stream_t stream) {
  if (!plan || !plan->dev || !X || !W || !B_pool || !Y) return LORA_ERR_ARG;
  if (!on_plan_device(plan)) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(B_pool) || !aligned16(Y)) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  const HostPlan &hp = plan->hp;
  const int64_t R = hp.offsets[hp.n_adapters];
  CUtensorMap mX128, mW, mBl;
  const bool sorted = hp.xs_offset >= 0;
  const void *Asrc = sorted ? static_cast<const void *>(plan->scratch + hp.xs_offset) : static_cast<const void *>(X);
  bool ok = true;
  ok &= make_map(&mX128, Asrc, hp.d_in, hp.T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  const bool b3d = hp.d_out % 64 == 0;
  ok &= b3d ? make_map_blocks(&mW, W, hp.d_out, hp.d_in, 64, kBN / 64)
            : make_map(&mW, W, hp.d_out, hp.d_in, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= b3d ? make_map_blocks(&mBl, B_pool, hp.d_out, R, 16, kBN / 64)
            : make_map(&mBl, B_pool, hp.d_out, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return LORA_ERR_ARG;
  GemmParams gp{};
  gp.b3d = b3d ? 1 : 0;
  gp.w3d = b3d ? 1 : 0;
  gp.T = static_cast<int32_t>(hp.T);
  gp.K = static_cast<int32_t>(hp.d_in);
  gp.N = static_cast<int32_t>(hp.d_out);
  gp.n_mt = static_cast<int32_t>(hp.tiles.size());
  gp.n_nt = static_cast<int32_t>((hp.d_out + kBN - 1) / kBN);
  gp.tiles = plan->d_tiles;
  gp.chunks = plan->d_chunks;
  gp.perm = plan->d_perm;
  gp.uimg = plan->scratch;
  gp.mt_order = plan->d_mt_order;
  gp.augblocks = plan->d_augblocks;
  {
    const int KB = (gp.K + kBK - 1) / kBK;
    if (plan->xws_S > 1 && fwd_ksplit(gp.n_mt * gp.n_nt, KB, ds->num_sms) == plan->xws_S)
      gp.xws = plan->scratch + plan->xws_offset;
  }
  if (plan->d_sched) {
    // the lists were made for the persistent grid of the plan's device; they
    // apply only to a launch of that same grid
    const int n_tiles = gp.n_mt * gp.n_nt;
    const int grid = static_cast<int>(plan->sched.size()) - n_tiles - 1;
    if (grid == std::min(ds->num_sms, n_tiles)) {
      gp.sched_off = plan->d_sched;
      gp.sched_tiles = plan->d_sched + grid + 1;
    }
  }
  gp.a_sorted = sorted ? 1 : 0;
  gp.out = reinterpret_cast<__nv_bfloat16 *>(Y);
  return launch_fwd_gemm(ds, gp, mX128, mW, mBl, stream);
}

int lora_linear_fwd(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                    const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed, uint16_t *Y,
                    float *U_save, const uint32_t *keep_bits, lora_stream_t stream) {
  if (!plan || !plan->dev || !X || !W || !A_pool || !B_pool || !scale || !Y) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(A_pool) || !aligned16(B_pool) || !aligned16(Y))
    return LORA_ERR_ARG;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  const int rc = lora_linear_shrink(plan, X, A_pool, scale, p_drop, seed, U_save, keep_bits, stream);
  if (rc != LORA_OK) return rc;
  return lora_fused_gemm(plan, X, W, B_pool, Y, stream);
}

int lora_linear_fwd_host(lora_plan_t plan, const int32_t *ids_host, int64_t T, const int32_t *ranks_host,
                         int32_t n_adapters, const uint16_t *X_host, uint16_t *X_dev, const uint16_t *W,
                         const uint16_t *A_pool, const uint16_t *B_pool, const float *scale, double p_drop,
                         uint64_t seed, uint16_t *Y_dev, uint16_t *Y_host, float *U_save, const uint32_t *keep_bits,
                         lora_stream_t stream) {
  // every argument is checked before anything is queued
  if (!plan || !plan->dev || !ids_host || !ranks_host || !X_host || !X_dev || !Y_dev || !Y_host) return LORA_ERR_ARG;
  if (!W || !A_pool || !B_pool || !scale) return LORA_ERR_ARG;
  if (!aligned16(X_dev) || !aligned16(W) || !aligned16(A_pool) || !aligned16(B_pool) || !aligned16(Y_dev))
    return LORA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(keep_bits) & 3u) return LORA_ERR_ARG;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  const int64_t d_in = plan->hp.d_in, d_out = plan->hp.d_out;
  int rc = lora_plan_rebuild(plan, ids_host, T, ranks_host, n_adapters, d_in, d_out, stream);
  if (rc != LORA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(X_dev, X_host, static_cast<size_t>(T * d_in) * 2, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  rc = lora_linear_fwd(plan, X_dev, W, A_pool, B_pool, scale, p_drop, seed, Y_dev, U_save, keep_bits, stream);
  if (rc != LORA_OK) return rc;
  if (cudaMemcpyAsync(Y_host, Y_dev, static_cast<size_t>(T * d_out) * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

int lora_linear_fwd_fused(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                          const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed, uint16_t *Y,
                          float *U_save, const uint32_t *keep_bits, lora_stream_t stream) {
  if (!plan || !plan->dev || !X || !W || !A_pool || !B_pool || !scale || !Y) return LORA_ERR_ARG;
  if (!on_plan_device(plan)) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(A_pool) || !aligned16(B_pool) || !aligned16(Y)) return LORA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(keep_bits) & 3u) return LORA_ERR_ARG;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  const HostPlan &hp = plan->hp;
  const int64_t R = hp.offsets[hp.n_adapters];
  const bool sorted = hp.xs_offset >= 0;
  uint16_t *Xs = sorted ? reinterpret_cast<uint16_t *>(plan->scratch + hp.xs_offset) : nullptr;
  const void *Asrc = sorted ? static_cast<const void *>(Xs) : static_cast<const void *>(X);
  // the GEMM's maps (as lora_fused_gemm) and the shrink's (as lora_linear_shrink)
  CUtensorMap mX128, mW, mBl, mX16, mA16;
  const bool b3d = hp.d_out % 64 == 0;
  bool ok = make_map(&mX128, Asrc, hp.d_in, hp.T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= b3d ? make_map_blocks(&mW, W, hp.d_out, hp.d_in, 64, kBN / 64)
            : make_map(&mW, W, hp.d_out, hp.d_in, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= b3d ? make_map_blocks(&mBl, B_pool, hp.d_out, R, 16, kBN / 64)
            : make_map(&mBl, B_pool, hp.d_out, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mX16, Asrc, hp.d_in, hp.T, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mA16, A_pool, hp.d_in, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return LORA_ERR_ARG;
  ShrinkParams sp{};
  sp.mode = 0;
  sp.T = static_cast<int32_t>(hp.T);
  sp.K = static_cast<int32_t>(hp.d_in);
  sp.ksplit = 1;  // one CTA per unit
  sp.kslice = static_cast<int32_t>((hp.d_in + kSkBK - 1) / kSkBK * kSkBK);
  sp.units = plan->d_units;
  sp.chunks = plan->d_chunks;
  sp.tiles = plan->d_tiles;
  sp.perm = plan->d_perm;
  sp.scale = scale;
  sp.thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  sp.keep_bits = sp.thr ? keep_bits : nullptr;
  sp.wpr = (hp.d_in + 31) / 32;
  CUtensorMap mBits16 = mX16;
  if (sp.keep_bits && sp.wpr % 4 == 0) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(sp.wpr), static_cast<cuuint64_t>(hp.T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(sp.wpr) * 4};
    cuuint32_t box[2] = {4, 16};
    cuuint32_t estr[2] = {1, 1};
    sp.bits_tma = g_encode(&mBits16, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(sp.keep_bits), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    if (!sp.bits_tma) mBits16 = mX16;
  }
  sp.seed = seed;
  sp.inv_keep = p_drop > 0.0 ? static_cast<float>(1.0 / (1.0 - p_drop)) : 1.0f;
  sp.uimg = plan->scratch;
  sp.x_sorted = sorted ? 1 : 0;
  sp.U_save = U_save;
  sp.r_max = hp.r_max;

  GemmParams gp{};
  gp.b3d = b3d ? 1 : 0;
  gp.w3d = b3d ? 1 : 0;
  gp.T = static_cast<int32_t>(hp.T);
  gp.K = static_cast<int32_t>(hp.d_in);
  gp.N = static_cast<int32_t>(hp.d_out);
  gp.n_mt = static_cast<int32_t>(hp.tiles.size());
  gp.n_nt = static_cast<int32_t>((hp.d_out + kBN - 1) / kBN);
  gp.tiles = plan->d_tiles;
  gp.chunks = plan->d_chunks;
  gp.perm = plan->d_perm;
  gp.uimg = plan->scratch;
  gp.mt_order = plan->d_mt_order;
  gp.augblocks = plan->d_augblocks;
  gp.a_sorted = sorted ? 1 : 0;
  gp.out = reinterpret_cast<__nv_bfloat16 *>(Y);
  const int n_tiles = gp.n_mt * gp.n_nt;
  const int KB = (gp.K + kBK - 1) / kBK;
  gp.group_m = default_group_m(gp.n_mt, gp.K);
  const int S = fwd_ksplit(n_tiles, KB, ds->num_sms);
  gp.ksplit = S;
  const int Gg = S == 1 ? std::min(ds->num_sms, n_tiles) : n_tiles * S;
  if (Gg != plan->fz_gemm_ctas) return LORA_ERR_ARG;  // the unit lists were dealt for this grid
  const int G = plan->fz_grid;
  gp.gemm_ctas = Gg;
  if (S > 1 && plan->xws_S == S) gp.xws = plan->scratch + plan->xws_offset;
  if (S == 1 && plan->d_sched && static_cast<int>(plan->sched.size()) - n_tiles - 1 == Gg) {
    gp.sched_off = plan->d_sched;
    gp.sched_tiles = plan->d_sched + G + 1;
  }
  gp.fz_unit_off = plan->d_fz_off;
  gp.fz_units = plan->d_fz_units;
  gp.fz_tile_need = plan->d_fz_need;
  gp.fz_tile_cnt = plan->d_fz_cnt;
  gp.fz_grid_cnt = plan->d_fz_cnt + hp.tiles.size();
  gp.fz_X = X;
  gp.fz_Xs = Xs;
  gp.fz_sp = sp;
  if (cudaMemsetAsync(plan->d_fz_cnt, 0, sizeof(int32_t) * (hp.tiles.size() + 1), stream) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  // cooperative: every CTA is resident at once, so the waits for other CTAs'
  // row copies and shrink units end
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = kGemmSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = S == 1 ? 1 : 2;
  if (cudaLaunchKernelEx(&cfg, lora_gemm_kernel<false, kEpiStore, true>, mX128, mW, mBl, mX16, mA16, mBits16, gp) !=
      cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  return LORA_OK;
}

int lora_base_gemm(const uint16_t *X, const uint16_t *W, uint16_t *Y, int64_t T, int64_t d_in, int64_t d_out,
                   lora_stream_t stream) {
  if (!X || !W || !Y || T <= 0 || d_in < 8 || d_out < 8 || (d_in % 8) || (d_out % 8)) return LORA_ERR_ARG;
  if (T > (int64_t)1 << 30 || d_in > (int64_t)1 << 30 || d_out > (int64_t)1 << 30) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(Y)) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  CUtensorMap mX128, mW;
  const bool w3d = d_out % 64 == 0;
  bool ok = make_map(&mX128, X, d_in, T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
            (w3d ? make_map_blocks(&mW, W, d_out, d_in, 64, kBN / 64)
                 : make_map(&mW, W, d_out, d_in, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B));
  if (!ok) return LORA_ERR_ARG;
  GemmParams gp{};
  gp.w3d = w3d ? 1 : 0;
  gp.T = static_cast<int32_t>(T);
  gp.K = static_cast<int32_t>(d_in);
  gp.N = static_cast<int32_t>(d_out);
  gp.n_mt = static_cast<int32_t>((T + kBM - 1) / kBM);
  gp.n_nt = static_cast<int32_t>((d_out + kBN - 1) / kBN);
  gp.a_sorted = 0;
  gp.out = reinterpret_cast<__nv_bfloat16 *>(Y);
  return launch_fwd_gemm(ds, gp, mX128, mW, mW, stream);
}

// Workspace layout: dU f32 [T, rp] | (r % 16 != 0: U f32 [T, rp]) | dB partial
// [S, r, d_out] | dA partial [S, r, d_in], rp = r rounded up to 16 (the token
// contraction reads whole 16-rank groups; the padding columns are zero).
// Token splits of the backward contractions: about two CTAs per SM of a B200
// (148 SMs) over the wider of the two column ranges, at least 64 tokens each.
static int64_t bwd_splits(int64_t T, int64_t d_in, int64_t d_out) {
  const int64_t cols = (std::max(d_in, d_out) + kTcCols - 1) / kTcCols;
  int64_t s = (2 * 148 + cols / 2) / cols;
  s = std::min<int64_t>(s, (T + kTcTok - 1) / kTcTok);
  return std::max<int64_t>(1, std::min<int64_t>(s, 16));
}

namespace {
struct BwdLayout {
  int64_t S, rp;
  int64_t off_dU, off_U, off_pdB, off_pdA, total;  // off_U < 0: U_save is read directly
};
BwdLayout bwd_layout(int64_t T, int64_t d_in, int64_t d_out, int32_t r) {
  auto up = [](int64_t b) { return (b + 255) & ~static_cast<int64_t>(255); };
  BwdLayout L{};
  L.S = bwd_splits(T, d_in, d_out);
  L.rp = (r + 15) / 16 * 16;
  L.off_dU = 0;
  int64_t o = up(T * L.rp * 4);
  L.off_U = -1;
  if (r % 16 != 0) {
    L.off_U = o;
    o += up(T * L.rp * 4);
  }
  L.off_pdB = o;
  o += up(L.S * r * d_out * 4);
  L.off_pdA = o;
  o += up(L.S * r * d_in * 4);
  L.total = o;
  return L;
}
}  // namespace

size_t lora_linear_bwd_workspace_size(int64_t T, int64_t d_in, int64_t d_out, int32_t r) {
  if (T <= 0 || d_in <= 0 || d_out <= 0 || r <= 0 || r > LORA_MAX_RANK) return 0;
  return static_cast<size_t>(bwd_layout(T, d_in, d_out, r).total);
}

int lora_linear_bwd(const uint16_t *X, const uint16_t *W, const uint16_t *A, const uint16_t *B, float scale,
                    double p_drop, uint64_t seed, const float *U_save, const uint16_t *dY, uint16_t *dX,
                    float *dA, float *dB, int64_t T, int64_t d_in, int64_t d_out, int32_t r, void *workspace,
                    size_t workspace_bytes, const uint32_t *keep_bits, lora_stream_t stream) {
  if (!X || !W || !A || !B || !U_save || !dY || !dX || !dA || !dB) return LORA_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(keep_bits) & 3u) return LORA_ERR_ARG;
  if (T <= 0 || d_in < 8 || d_out < 8 || (d_in % 8) || (d_out % 8)) return LORA_ERR_ARG;
  if (T > (int64_t)1 << 30 || d_in > (int64_t)1 << 30 || d_out > (int64_t)1 << 30) return LORA_ERR_ARG;
  if (r < 1 || r > LORA_MAX_RANK) return LORA_ERR_RANK;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  // U_save rows are r fp32 apart; a tensor map needs 16-byte row strides, so
  // U_save itself is read only when r % 16 == 0 (else its padded copy)
  if (!aligned16(X) || !aligned16(W) || !aligned16(A) || !aligned16(B) || !aligned16(dY) || !aligned16(dX) ||
      (reinterpret_cast<uintptr_t>(U_save) & 3u) || (reinterpret_cast<uintptr_t>(dA) & 3u) ||
      (reinterpret_cast<uintptr_t>(dB) & 3u) || (r % 16 == 0 && !aligned16(U_save)))
    return LORA_ERR_ARG;
  const BwdLayout Lw = bwd_layout(T, d_in, d_out, r);
  if (!workspace || workspace_bytes < static_cast<size_t>(Lw.total) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return LORA_ERR_WORKSPACE;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;

  const int64_t S = Lw.S;
  const int rp = static_cast<int>(Lw.rp);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  float *dU = reinterpret_cast<float *>(ws + Lw.off_dU);
  float *Ug = Lw.off_U >= 0 ? reinterpret_cast<float *>(ws + Lw.off_U) : const_cast<float *>(U_save);
  float *pdB = reinterpret_cast<float *>(ws + Lw.off_pdB);
  float *pdA = reinterpret_cast<float *>(ws + Lw.off_pdA);

  const uint64_t thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  const float inv_keep = p_drop > 0.0 ? static_cast<float>(1.0 / (1.0 - p_drop)) : 1.0f;

  CUtensorMap mdY16, mB16, mdY128, mWt, mdY64, mX64;
  bool ok = true;
  ok &= make_map(&mdY16, dY, d_out, T, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mB16, B, d_out, r, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mdY128, dY, d_out, T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mWt, W, d_out, d_in, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mdY64, dY, d_out, T, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  ok &= make_map(&mX64, X, d_in, T, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return LORA_ERR_ARG;

  // K3a: dU = s * dY * B^T (fp32, rows padded to rp with zeros)
  {
    ShrinkParams sp{};
    sp.mode = 1;
    sp.T = static_cast<int32_t>(T);
    sp.K = static_cast<int32_t>(d_out);
    sp.r = r;
    sp.npieces = (rp + kShrinkN - 1) / kShrinkN;
    sp.scale1 = scale;
    sp.x_sorted = 0;
    sp.dU = dU;
    const int n_units = static_cast<int>((T + kTileM - 1) / kTileM) * sp.npieces;
    int ks = 1;
    const int max_nb16 = shrink_build(n_units, d_out, ds->num_sms, std::min(kShrinkN, rp), &ks);
    int64_t slice = (d_out + ks - 1) / ks;
    slice = (slice + kSkBK - 1) / kSkBK * kSkBK;
    sp.ksplit = ks;
    sp.kslice = static_cast<int32_t>(slice);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(n_units * ks));
    cfg.blockDim = dim3(kSkThreads);
    cfg.dynamicSmemBytes = sk_smem(max_nb16);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, max_nb16 <= 2 ? lora_shrink_kernel<2> : lora_shrink_kernel<4>, mdY16, mB16, mdY16,
                           sp) != cudaSuccess) {
      cudaGetLastError();
      return LORA_ERR_CUDA;
    }
  }
  if (Lw.off_U >= 0) {
    // U_save with its rows padded to rp columns, for the dB contraction's tensor map
    const int64_t n = T * rp;
    lora_pad_cols_kernel<<<static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 16 * ds->num_sms)), 256, 0,
                           stream>>>(U_save, r, Ug, rp, T);
  }
  // K3b: dX = dY * W^T + D ⊙ (dU * A^T)
  {
    GemmParams gp{};
    gp.T = static_cast<int32_t>(T);
    gp.K = static_cast<int32_t>(d_out);
    gp.N = static_cast<int32_t>(d_in);
    gp.n_mt = static_cast<int32_t>((T + kBM - 1) / kBM);
    gp.n_nt = static_cast<int32_t>((d_in + kBN - 1) / kBN);
    gp.a_sorted = 0;
    gp.out = reinterpret_cast<__nv_bfloat16 *>(dX);
    gp.dU = dU;
    gp.A = A;
    gp.r = r;
    gp.du_stride = rp;
    gp.seed = seed;
    gp.thr = thr;
    gp.keep_bits = thr ? keep_bits : nullptr;
    gp.wpr = (d_in + 31) / 32;
    gp.inv_keep = inv_keep;
    gp.ksplit = 1;
    gp.group_m = default_group_m(gp.n_mt, gp.K);
    const int grid = std::min(ds->num_sms, gp.n_mt * gp.n_nt);
    lora_gemm_kernel<true, kEpiBwdLora><<<grid, kGemmThreads, kGemmSmemBwd, stream>>>(mdY128, mWt, mWt, mWt, mWt, mWt, gp);
    if (cudaGetLastError() != cudaSuccess) return LORA_ERR_CUDA;
  }
  // K3c: dB = s * U^T * dY and dA = (D ⊙ X)^T * dU, split over tokens, then
  // reduced; one launch of each contraction per group of up to 64 ranks
  {
    const int64_t tsplit = ((T + S - 1) / S + kTcTok - 1) / kTcTok * kTcTok;
    // keep bits in the dA contraction need a 16-byte row stride (d_in % 128 == 0);
    // otherwise it re-derives the mask from the generator
    bool use_bits = thr != 0 && keep_bits != nullptr && ((d_in + 31) / 32) % 4 == 0;
    CUtensorMap mBits = mX64;  // unused unless the dA contraction reads keep bits
    if (use_bits) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>((d_in + 31) / 32), static_cast<cuuint64_t>(T)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>((d_in + 31) / 32) * 4};
      cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcCols / 32), static_cast<cuuint32_t>(kTcTok)};
      cuuint32_t estr[2] = {1, 1};
      if (g_encode(&mBits, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(keep_bits), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        use_bits = false;
    }
    const int64_t ustride = Lw.off_U >= 0 ? rp : r;  // r % 16 == 0 when U_save is read directly
    for (int k0 = 0; k0 < r; k0 += kTcMaxR) {
      const int w = std::min(kTcMaxR, rp - k0);  // a multiple of 16
      CUtensorMap mU, mdU;
      if (!make_map_f32(&mU, Ug, ustride, T, w, 64) || !make_map_f32(&mdU, dU, rp, T, w, 64)) return LORA_ERR_ARG;
      TcParams tp{};
      tp.T = static_cast<int32_t>(T);
      tp.r = w;
      tp.r_valid = std::min(w, r - k0);
      tp.k0 = k0;
      tp.r_total = r;
      tp.splits = static_cast<int32_t>(S);
      tp.tsplit = static_cast<int32_t>(tsplit);
      tp.N = static_cast<int32_t>(d_out);
      tp.thr = 0;
      tp.keep_bits = nullptr;
      tp.partial = pdB;
      dim3 grid_b(static_cast<unsigned>((d_out + kTcCols - 1) / kTcCols), static_cast<unsigned>(S));
      const int smem_b = tc_smem(w);
      lora_tcontract_kernel<<<grid_b, kTcThreads, smem_b, stream>>>(mdY64, mU, mBits, mU, mU, mU, tp);
      tp.N = static_cast<int32_t>(d_in);
      tp.thr = thr;
      tp.seed = seed;
      // with keep bits, each stage's bits come through the copy engine with its tile
      tp.keep_bits = use_bits ? keep_bits : nullptr;
      const int smem_a = tc_smem(w);
      tp.wpr = (d_in + 31) / 32;
      tp.partial = pdA;
      dim3 grid_a(static_cast<unsigned>((d_in + kTcCols - 1) / kTcCols), static_cast<unsigned>(S));
      lora_tcontract_kernel<<<grid_a, kTcThreads, smem_a, stream>>>(mX64, mdU, mBits, mdU, mdU, mdU, tp);
    }
    const int64_t nb = static_cast<int64_t>(r) * d_out;
    const int64_t na = static_cast<int64_t>(r) * d_in;
    lora_reduce_splits_kernel<<<static_cast<unsigned>(std::min<int64_t>((nb + 255) / 256, 4096)), 256, 0, stream>>>(
        pdB, static_cast<int>(S), nb, scale, dB);
    lora_reduce_splits_kernel<<<static_cast<unsigned>(std::min<int64_t>((na + 255) / 256, 4096)), 256, 0, stream>>>(
        pdA, static_cast<int>(S), na, inv_keep, dA);
  }
  return launch_status();
}


// Workspace of lora_linear_bwd_multi, in this order (each part 256-byte aligned):
// s·dU images (the plan's image layout) | sorted X, sorted dY, sorted keep bits
// (when the plan gathers) | G = dY·B_a^T and U, both [T, rp] fp32 in sorted
// order (rp = r_max rounded up to 16) | dA, dB partial rows of multi-piece
// segments.
namespace {
struct BwdMultiLayout {
  int64_t img, xs, dys, bits, g, u, pda, pdb, total;
};
BwdMultiLayout bwd_multi_layout(const HostPlan &hp) {
  auto up = [](int64_t b) { return (b + 255) & ~static_cast<int64_t>(255); };
  const bool gathers = hp.xs_offset >= 0;
  const int64_t rp = (hp.r_max + 15) / 16 * 16;
  const int64_t wpr = (hp.d_in + 31) / 32;
  BwdMultiLayout L{};
  int64_t o = 0;
  L.img = o;
  o += up(gathers ? hp.xs_offset : hp.scratch_bytes);
  L.xs = gathers ? o : -1;
  if (gathers) o += up(hp.T * hp.d_in * 2);
  L.dys = gathers ? o : -1;
  if (gathers) o += up(hp.T * hp.d_out * 2);
  L.bits = gathers ? o : -1;
  if (gathers) o += up(hp.T * wpr * 4);
  L.g = o;
  o += up(hp.T * rp * 4);
  L.u = o;
  o += up(hp.T * rp * 4);
  L.pda = o;
  o += up(hp.partial_rows * hp.d_in * 4);
  L.pdb = o;
  o += up(hp.partial_rows * hp.d_out * 4);
  L.total = o;
  return L;
}
}  // namespace

size_t lora_linear_bwd_multi_workspace_size(lora_plan_t plan) {
  if (!plan) return 0;
  return static_cast<size_t>(bwd_multi_layout(plan->hp).total);
}

int lora_linear_bwd_multi(lora_plan_t plan, const uint16_t *X, const uint16_t *W, const uint16_t *A_pool,
                          const uint16_t *B_pool, const float *scale, double p_drop, uint64_t seed,
                          const float *U_save, const uint16_t *dY, uint16_t *dX, float *dA_pool, float *dB_pool,
                          void *workspace, size_t workspace_bytes, const uint32_t *keep_bits, lora_stream_t stream) {
  if (!plan || !plan->dev || !X || !W || !A_pool || !B_pool || !scale || !U_save || !dY || !dX || !dA_pool ||
      !dB_pool)
    return LORA_ERR_ARG;
  if (!on_plan_device(plan)) return LORA_ERR_ARG;
  if (!aligned16(X) || !aligned16(W) || !aligned16(A_pool) || !aligned16(B_pool) || !aligned16(dY) ||
      !aligned16(dX) || (reinterpret_cast<uintptr_t>(U_save) & 3u) || (reinterpret_cast<uintptr_t>(dA_pool) & 3u) ||
      (reinterpret_cast<uintptr_t>(dB_pool) & 3u) || (reinterpret_cast<uintptr_t>(keep_bits) & 3u))
    return LORA_ERR_ARG;
  if (!(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  const HostPlan &hp = plan->hp;
  if (hp.pieces.size() > 65535) return LORA_ERR_ARG;  // one grid row of the reduction per piece
  const BwdMultiLayout Lw = bwd_multi_layout(hp);
  if (!workspace || workspace_bytes < static_cast<size_t>(Lw.total) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return LORA_ERR_WORKSPACE;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;

  const int64_t T = hp.T, d_in = hp.d_in, d_out = hp.d_out;
  const int64_t R = hp.offsets[hp.n_adapters];
  const int rp = (hp.r_max + 15) / 16 * 16;
  const int64_t wpr = (d_in + 31) / 32;
  const bool gathers = hp.xs_offset >= 0;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *img = ws + Lw.img;
  const uint16_t *Xr = gathers ? reinterpret_cast<const uint16_t *>(ws + Lw.xs) : X;
  const uint16_t *dYr = gathers ? reinterpret_cast<const uint16_t *>(ws + Lw.dys) : dY;
  float *G = reinterpret_cast<float *>(ws + Lw.g);
  float *Us = reinterpret_cast<float *>(ws + Lw.u);
  float *pdA = reinterpret_cast<float *>(ws + Lw.pda);
  float *pdB = reinterpret_cast<float *>(ws + Lw.pdb);
  const uint64_t thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  const float inv_keep = p_drop > 0.0 ? static_cast<float>(1.0 / (1.0 - p_drop)) : 1.0f;
  const uint32_t *bits = thr ? keep_bits : nullptr;
  // keep bits for the dA contraction: rows in the order of its In rows (sorted
  // when the plan gathers), staged through TMA when rows are 16-byte multiples
  const bool bits_tc = bits && wpr % 4 == 0;
  const uint32_t *bits_in = gathers && bits_tc ? reinterpret_cast<const uint32_t *>(ws + Lw.bits) : bits;

  auto grid_for = [&](int64_t n) {
    return static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 16 * ds->num_sms));
  };
  // sorted copies of X, dY (and the keep bits) when the plan's tiles are not runs
  if (gathers) {
    lora_gather_rows_kernel<<<grid_for(T * (d_in / 8)), 256, 0, stream>>>(X, plan->d_perm,
                                                                         const_cast<uint16_t *>(Xr), T, d_in);
    lora_gather_rows_kernel<<<grid_for(T * (d_out / 8)), 256, 0, stream>>>(dY, plan->d_perm,
                                                                          const_cast<uint16_t *>(dYr), T, d_out);
    if (bits_tc)
      lora_gather_rows_kernel<<<grid_for(T * wpr / 4), 256, 0, stream>>>(
          reinterpret_cast<const uint16_t *>(bits), plan->d_perm,
          reinterpret_cast<uint16_t *>(const_cast<uint32_t *>(bits_in)), T, 2 * wpr);
  }
  // U in sorted order, rows padded to rp
  lora_gather_pad_kernel<<<grid_for(T * rp), 256, 0, stream>>>(U_save, hp.r_max, plan->d_perm, Us, rp, T);
  if (cudaGetLastError() != cudaSuccess) return LORA_ERR_CUDA;

  // dU: the plan's shrink units over dY against B_pool: s_a·dU images (hi/lo,
  // the dX GEMM's adapter operand) and G = dY·B_a^T in sorted order
  {
    CUtensorMap mdY16, mB16;
    if (!make_map(&mdY16, dYr, d_out, T, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mB16, B_pool, d_out, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B))
      return LORA_ERR_ARG;
    ShrinkParams sp{};
    sp.K = static_cast<int32_t>(d_out);
    sp.scale = scale;
    sp.inv_keep = 1.0f;
    sp.uimg = img;
    sp.x_sorted = gathers ? 1 : 0;
    sp.U_save = G;
    sp.r_max = rp;
    sp.u_sorted = 1;
    rc = launch_unit_shrink(ds, plan, mdY16, mB16, mdY16, sp, stream);
    if (rc != LORA_OK) return rc;
  }
  // dX = dY·W^T + D ⊙ (s_a·dU·A_a^T): the fused GEMM over the plan's tiles, W^T a
  // K-major operand, the adapter blocks A_pool rows (into a second accumulator,
  // masked in the epilogue, when there is dropout)
  {
    CUtensorMap mdY128, mWt, mAl;
    const bool b3d = d_in % 64 == 0;
    bool ok = make_map(&mdY128, dYr, d_out, T, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mWt, W, d_out, d_in, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B) &&
              (b3d ? make_map_blocks(&mAl, A_pool, d_in, R, 16, kBN / 64)
                   : make_map(&mAl, A_pool, d_in, R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B));
    if (!ok) return LORA_ERR_ARG;
    GemmParams gp{};
    gp.b3d = b3d ? 1 : 0;
    gp.T = static_cast<int32_t>(T);
    gp.K = static_cast<int32_t>(d_out);
    gp.N = static_cast<int32_t>(d_in);
    gp.n_mt = static_cast<int32_t>(hp.tiles.size());
    gp.n_nt = static_cast<int32_t>((d_in + kBN - 1) / kBN);
    gp.tiles = plan->d_tiles;
    gp.chunks = plan->d_chunks;
    gp.perm = plan->d_perm;
    gp.uimg = img;
    gp.mt_order = plan->d_mt_order;
    gp.augblocks = plan->d_augblocks;
    gp.a_sorted = gathers ? 1 : 0;
    gp.out = reinterpret_cast<__nv_bfloat16 *>(dX);
    gp.seed = seed;
    gp.thr = thr;
    gp.keep_bits = bits;
    gp.wpr = wpr;
    gp.inv_keep = inv_keep;
    gp.ksplit = 1;
    gp.group_m = default_group_m(gp.n_mt, gp.K);
    const int n_tiles = gp.n_mt * gp.n_nt;
    const int grid = std::min(ds->num_sms, n_tiles);
    if (plan->d_sched && d_in == d_out && static_cast<int>(plan->sched.size()) - n_tiles - 1 == grid &&
        default_group_m(gp.n_mt, d_in) == gp.group_m) {
      gp.sched_off = plan->d_sched;  // the forward's per-CTA tile lists fit this grid and tile order
      gp.sched_tiles = plan->d_sched + grid + 1;
    }
    if (thr)
      lora_gemm_kernel<true, kEpiBwdMulti><<<grid, kGemmThreads, kGemmSmem, stream>>>(mdY128, mWt, mAl, mAl, mAl, mAl, gp);
    else
      lora_gemm_kernel<true, kEpiStore><<<grid, kGemmThreads, kGemmSmem, stream>>>(mdY128, mWt, mAl, mAl, mAl, mAl, gp);
    if (cudaGetLastError() != cudaSuccess) return LORA_ERR_CUDA;
  }
  // dB_a = s_a·U^T·dY and dA_a = s_a·(D ⊙ X)^T·G over each segment's pieces, then
  // the multi-piece segments' partial sums
  {
    CUtensorMap mIn64b, mIn64a, mBits = {};
    if (!make_map(&mIn64b, dYr, d_out, T, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mIn64a, Xr, d_in, T, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return LORA_ERR_ARG;
    CUtensorMap mU[4], mG[4];
    for (int w = 0; w < 4; ++w)
      if (!make_map_f32(&mU[w], Us, rp, T, 16 * (w + 1), 64) || !make_map_f32(&mG[w], G, rp, T, 16 * (w + 1), 64))
        return LORA_ERR_ARG;
    bool use_bits = bits_tc;
    mBits = mIn64a;
    if (use_bits) {
      cuuint64_t dims[2] = {static_cast<cuuint64_t>(wpr), static_cast<cuuint64_t>(T)};
      cuuint64_t strides[1] = {static_cast<cuuint64_t>(wpr) * 4};
      cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcCols / 32), static_cast<cuuint32_t>(kTcTok)};
      cuuint32_t estr[2] = {1, 1};
      if (g_encode(&mBits, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(bits_in), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        use_bits = false;
    }
    const unsigned n_pieces = static_cast<unsigned>(hp.pieces.size());
    const unsigned n_ranges = static_cast<unsigned>(plan->ranges.size() - 1);
    const unsigned groups = static_cast<unsigned>((rp + kTcMaxR - 1) / kTcMaxR);
    const int smem = tc_smem(std::min(rp, kTcMaxR));  // the widest rank group of any piece
    TcParams tp{};
    tp.T = static_cast<int32_t>(T);
    tp.pieces = plan->d_pieces;
    tp.range_off = plan->d_ranges;
    tp.rp = rp;
    tp.scale = scale;
    // dB: In = dY, G = U, no mask
    tp.N = static_cast<int32_t>(d_out);
    tp.factor = 1.0f;
    tp.out = dB_pool;
    tp.partial = pdB;
    dim3 grid_b(static_cast<unsigned>((d_out + kTcCols - 1) / kTcCols), n_ranges, groups);
    lora_tcontract_kernel<<<grid_b, kTcThreads, smem, stream>>>(mIn64b, mU[3], mBits, mU[0], mU[1], mU[2], tp);
    // dA: In = X with the dropout mask, G = dY·B^T; the mask's 1/(1 - p) and s_a
    // scale the sums
    tp.N = static_cast<int32_t>(d_in);
    tp.thr = thr;
    tp.seed = seed;
    tp.keep_bits = use_bits ? bits_in : nullptr;
    tp.wpr = wpr;
    tp.perm = gathers ? plan->d_perm : nullptr;
    tp.factor = inv_keep;
    tp.out = dA_pool;
    tp.partial = pdA;
    dim3 grid_a(static_cast<unsigned>((d_in + kTcCols - 1) / kTcCols), n_ranges, groups);
    lora_tcontract_kernel<<<grid_a, kTcThreads, smem, stream>>>(mIn64a, mG[3], mBits, mG[0], mG[1], mG[2], tp);
    if (hp.partial_rows > 0) {
      const unsigned gb = static_cast<unsigned>(std::min<int64_t>((hp.r_max * d_out + 255) / 256, 256));
      const unsigned ga = static_cast<unsigned>(std::min<int64_t>((hp.r_max * d_in + 255) / 256, 256));
      lora_reduce_pieces_kernel<<<dim3(gb, n_pieces), 256, 0, stream>>>(plan->d_pieces, pdB, d_out, scale, 1.0f,
                                                                        dB_pool);
      lora_reduce_pieces_kernel<<<dim3(ga, n_pieces), 256, 0, stream>>>(plan->d_pieces, pdA, d_in, scale, inv_keep,
                                                                        dA_pool);
    }
  }
  return launch_status();
}

}  // extern "C"

// Scratch of lora_linear_bwd_static: one array per device, shared by every
// call; host code must not use its name as an address (that is a host-side
// stand-in), so the device address is looked up once per device below.
static __device__ __align__(256) uint8_t g_bwd_static_scratch[LORA_BWD_STATIC_SCRATCH_BYTES];
// its device address per device, published once (release) and read lock-free (acquire)
static std::atomic<void *> g_bwd_static_ptr[kMaxDevices];

extern "C" {

int lora_linear_bwd_static(const uint16_t *X, const uint16_t *W, const uint16_t *A, const uint16_t *B,
                           float scale, double p_drop, uint64_t seed, const float *U_save, const uint16_t *dY,
                           uint16_t *dX, float *dA, float *dB, int64_t T, int64_t d_in, int64_t d_out, int32_t r,
                           const uint32_t *keep_bits, lora_stream_t stream) {
  // The size check comes first and touches no pointer: an oversized request is
  // rejected before any argument is read or any CUDA call is made.
  const size_t need = lora_linear_bwd_workspace_size(T, d_in, d_out, r);
  if (need > LORA_BWD_STATIC_SCRATCH_BYTES) return LORA_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LORA_ERR_CUDA;
  void *scratch = g_bwd_static_ptr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    std::lock_guard<std::mutex> lk(g_mu);
    scratch = g_bwd_static_ptr[dev].load(std::memory_order_relaxed);
    if (!scratch) {
      if (cudaGetSymbolAddress(&scratch, g_bwd_static_scratch) != cudaSuccess || !scratch) {
        cudaGetLastError();
        return LORA_ERR_CUDA;
      }
      g_bwd_static_ptr[dev].store(scratch, std::memory_order_release);
    }
  }
  return lora_linear_bwd(X, W, A, B, scale, p_drop, seed, U_save, dY, dX, dA, dB, T, d_in, d_out, r, scratch,
                         LORA_BWD_STATIC_SCRATCH_BYTES, keep_bits, stream);
}

int lora_dropout_mask(uint64_t seed, double p_drop, int64_t T, int64_t d_in, uint8_t *mask_dev,
                      lora_stream_t stream) {
  if (!mask_dev || T <= 0 || d_in <= 0 || !(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK && rc != LORA_ERR_UNSUPPORTED) return rc;
  const uint64_t thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  const int64_t n = T * d_in;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 65535));
  lora_mask_kernel<<<blocks, 256, 0, stream>>>(seed, thr, T, d_in, mask_dev);
  return launch_status();
}

int lora_dropout_keep_bits(uint64_t seed, double p_drop, int64_t T, int64_t d_in, uint32_t *bits_dev,
                           lora_stream_t stream) {
  if (!bits_dev || T <= 0 || d_in <= 0 || !(p_drop >= 0.0 && p_drop < 1.0)) return LORA_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(bits_dev) & 3u) != 0) return LORA_ERR_ARG;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  const uint64_t thr = p_drop > 0.0 ? static_cast<uint64_t>(ldexp(p_drop, 64)) : 0ull;
  const int64_t wpr = (d_in + 31) / 32;
  const int64_t n = T * wpr;
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 16 * ds->num_sms));
  lora_keep_bits_kernel<<<blocks, 256, 0, stream>>>(seed, thr, T, d_in, wpr, bits_dev);
  return launch_status();
}

uint64_t lora_dropout_seed_for_rows(uint64_t seed, int64_t t0, int64_t d_in) {
  if (t0 < 0 || d_in < 1) return seed;
  return seed + static_cast<uint64_t>(t0) * static_cast<uint64_t>(d_in) * 0x9E3779B97F4A7C15ull;
}

int lora_selftest_bounded_wait(uint32_t limit_us, int *waited_ok_dev, lora_stream_t stream) {
  if (!waited_ok_dev || limit_us < 1 || limit_us > 1000000) return LORA_ERR_ARG;
  lora_wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_us) * 1000ull, waited_ok_dev);
  return launch_status();
}

int lora_device_status(lora_stream_t stream, uint32_t *status_host) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return LORA_ERR_CUDA;
  const uint32_t zero = 0;
  if (v && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return LORA_ERR_CUDA;
  if (status_host) *status_host = v;
  return v ? LORA_ERR_DEVICE : LORA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ fused adapter switch
struct lora_switch {
  int64_t L = 0, d_in = 0, d_out = 0;
  std::vector<int32_t> ranks;
  std::vector<int64_t> off;  // n_adapters + 1
  int32_t max_terms = 0;
  int32_t max_kaug = 0;      // max_terms * 2 * (largest rank rounded up to 16)
  int32_t mt_per_layer = 0;
  int64_t n_tiles = 0;       // L * mt_per_layer
  int64_t img_bytes = 0;     // one tile's images
  uint8_t *img = nullptr;    // n_tiles * img_bytes
  void *dev = nullptr;       // terms | adapter blocks
  size_t dev_bytes = 0;
  void *stage[2] = {nullptr, nullptr};
  cudaEvent_t stage_ev[2] = {nullptr, nullptr};
  int stage_next = 0;
  int device = 0;
};

extern "C" {

void lora_switch_destroy(lora_switch_t sw) {
  if (!sw) return;
  for (int k = 0; k < 2; ++k) {
    if (sw->stage_ev[k]) {
      cudaEventSynchronize(sw->stage_ev[k]);
      cudaEventDestroy(sw->stage_ev[k]);
    }
    if (sw->stage[k]) cudaFreeHost(sw->stage[k]);
  }
  if (sw->dev) cudaFree(sw->dev);
  if (sw->img) cudaFree(sw->img);
  delete sw;
}

int lora_switch_create(const int32_t *ranks_host, int32_t n_adapters, int64_t L, int64_t d_in, int64_t d_out,
                       int32_t max_terms, lora_switch_t *out) {
  if (!out || !ranks_host || n_adapters < 1 || L < 1 || d_in < 8 || d_out < 8 || (d_in % 8) || (d_out % 8))
    return LORA_ERR_ARG;
  if (max_terms < 1 || max_terms > LORA_SWITCH_MAX_TERMS) return LORA_ERR_ARG;
  if (L * d_in > ((int64_t)1 << 30) || d_out > ((int64_t)1 << 30)) return LORA_ERR_ARG;
  int32_t rmax = 0;
  for (int32_t a = 0; a < n_adapters; ++a) {
    if (ranks_host[a] < 1 || ranks_host[a] > LORA_MAX_RANK) return LORA_ERR_RANK;
    rmax = std::max(rmax, ranks_host[a]);
  }
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  lora_switch *sw = new (std::nothrow) lora_switch();
  if (!sw) return LORA_ERR_NOMEM;
  sw->L = L;
  sw->d_in = d_in;
  sw->d_out = d_out;
  sw->ranks.assign(ranks_host, ranks_host + n_adapters);
  sw->off.assign(n_adapters + 1, 0);
  for (int32_t a = 0; a < n_adapters; ++a) sw->off[a + 1] = sw->off[a] + ranks_host[a];
  if (L * sw->off[n_adapters] >= ((int64_t)1 << 31) - 256) {
    delete sw;
    return LORA_ERR_ARG;
  }
  sw->max_terms = max_terms;
  sw->max_kaug = max_terms * 2 * ((rmax + 15) / 16 * 16);
  sw->mt_per_layer = static_cast<int32_t>((d_in + kTileM - 1) / kTileM);
  sw->n_tiles = L * sw->mt_per_layer;
  sw->img_bytes = static_cast<int64_t>((sw->max_kaug + kAugBlock - 1) / kAugBlock) * kAugBlockBytes;
  const size_t nblk_max = static_cast<size_t>((sw->max_kaug + kAugBlock - 1) / kAugBlock);
  sw->dev_bytes = ((sizeof(SwitchTerm) * max_terms + 255) & ~static_cast<size_t>(255)) + sizeof(AugBlockDesc) * nblk_max;
  cudaGetDevice(&sw->device);
  bool ok = cudaMalloc(reinterpret_cast<void **>(&sw->img), static_cast<size_t>(sw->n_tiles * sw->img_bytes)) ==
            cudaSuccess;
  ok = ok && cudaMalloc(&sw->dev, sw->dev_bytes) == cudaSuccess;
  for (int k = 0; k < 2 && ok; ++k) {
    ok &= cudaHostAlloc(&sw->stage[k], sw->dev_bytes, cudaHostAllocDefault) == cudaSuccess;
    ok = ok && cudaEventCreateWithFlags(&sw->stage_ev[k], cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    cudaGetLastError();
    lora_switch_destroy(sw);
    return LORA_ERR_NOMEM;
  }
  *out = sw;
  return LORA_OK;
}

int lora_switch_apply(lora_switch_t sw, uint16_t *W, const uint16_t *A_pool, const uint16_t *B_pool,
                      const int32_t *term_adapter_host, const float *term_coef_host, int32_t n_terms,
                      lora_stream_t stream) {
  if (!sw || !W || !A_pool || !B_pool || !term_adapter_host || !term_coef_host) return LORA_ERR_ARG;
  if (n_terms < 1 || n_terms > sw->max_terms) return LORA_ERR_ARG;
  if (!aligned16(W) || !aligned16(A_pool) || !aligned16(B_pool)) return LORA_ERR_ARG;
  {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d != sw->device) return LORA_ERR_ARG;
  }
  const int32_t n_adapters = static_cast<int32_t>(sw->ranks.size());
  for (int32_t j = 0; j < n_terms; ++j)
    if (term_adapter_host[j] < 0 || term_adapter_host[j] >= n_adapters) return LORA_ERR_ID;
  DeviceState *ds = nullptr;
  int rc = device_state(&ds);
  if (rc != LORA_OK) return rc;
  // the terms' augmented columns (hi part, then lo part, per term) and the
  // adapter blocks that read their B rows, the same for every tile
  std::vector<SwitchTerm> terms(n_terms);
  std::vector<ChunkDesc> chunks(n_terms);
  int32_t kofs = 0;
  for (int32_t j = 0; j < n_terms; ++j) {
    const int32_t a = term_adapter_host[j];
    SwitchTerm &t = terms[j];
    t = SwitchTerm{};
    t.pool_row = static_cast<int32_t>(sw->off[a]);
    t.rank = sw->ranks[a];
    t.kc = (t.rank + 15) / 16 * 16;
    t.kofs = kofs;
    t.coef = term_coef_host[j];
    ChunkDesc &c = chunks[j];
    c = ChunkDesc{};
    c.adapter = a;
    c.pool_row = t.pool_row;
    c.rank = t.rank;
    c.kc = t.kc;
    c.kofs = kofs;
    kofs += 2 * t.kc;
  }
  const int32_t kaug = kofs;
  std::vector<AugBlockDesc> aug;
  append_aug_blocks(chunks.data(), n_terms, kaug, aug);
  const size_t b_terms = (sizeof(SwitchTerm) * sw->max_terms + 255) & ~static_cast<size_t>(255);
  const size_t total = b_terms + sizeof(AugBlockDesc) * aug.size();
  // one copy from one of two pinned staging buffers (refilled once its last
  // copy has completed), stream-ordered before the kernels that read it
  const int k = sw->stage_next;
  if (cudaEventSynchronize(sw->stage_ev[k]) != cudaSuccess) return LORA_ERR_CUDA;
  uint8_t *h = static_cast<uint8_t *>(sw->stage[k]);
  std::memcpy(h, terms.data(), sizeof(SwitchTerm) * n_terms);
  std::memcpy(h + b_terms, aug.data(), sizeof(AugBlockDesc) * aug.size());
  uint8_t *dbase = static_cast<uint8_t *>(sw->dev);
  if (cudaMemcpyAsync(dbase, h, total, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaEventRecord(sw->stage_ev[k], stream) != cudaSuccess) {
    cudaGetLastError();
    return LORA_ERR_CUDA;
  }
  sw->stage_next = k ^ 1;
  const int64_t R = sw->off[n_adapters];
  // DOWN: c·A of every term, as the tiles' swizzled images
  {
    const int64_t n = sw->n_tiles * (kaug / 8) * kTileM;
    const unsigned blocks = static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 32 * ds->num_sms));
    lora_switch_images_kernel<<<blocks, 256, 0, stream>>>(A_pool, reinterpret_cast<const SwitchTerm *>(dbase),
                                                          n_terms, R, sw->d_in, sw->mt_per_layer, sw->n_tiles, kaug,
                                                          sw->img_bytes, sw->img);
    if (cudaGetLastError() != cudaSuccess) return LORA_ERR_CUDA;
  }
  // W += DOWN·UP on the tensor cores, every layer in one persistent launch
  CUtensorMap mBl, mW;
  const bool b3d = sw->d_out % 64 == 0;
  bool ok = b3d ? make_map_blocks(&mBl, B_pool, sw->d_out, sw->L * R, 16, kBN / 64)
                : make_map(&mBl, B_pool, sw->d_out, sw->L * R, 64, 16, CU_TENSOR_MAP_SWIZZLE_128B);
  // the weights as 128-row x 64-column boxes: each tile's W blocks
  ok = ok && make_map(&mW, W, sw->d_out, sw->L * sw->d_in, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return LORA_ERR_ARG;
  GemmParams gp{};
  gp.b3d = b3d ? 1 : 0;
  gp.T = static_cast<int32_t>(sw->L * sw->d_in);
  gp.K = 0;
  gp.N = static_cast<int32_t>(sw->d_out);
  gp.n_mt = static_cast<int32_t>(sw->n_tiles);
  gp.n_nt = static_cast<int32_t>((sw->d_out + kBN - 1) / kBN);
  gp.uimg = sw->img;
  gp.augblocks = reinterpret_cast<const AugBlockDesc *>(dbase + b_terms);
  gp.out = reinterpret_cast<__nv_bfloat16 *>(W);
  gp.group_m = 1;
  gp.ksplit = 1;
  gp.merge_kaug = kaug;
  gp.mt_per_layer = sw->mt_per_layer;
  gp.merge_rows = static_cast<int32_t>(sw->d_in);
  gp.layer_brows = static_cast<int32_t>(R);
  gp.merge_img_bytes = sw->img_bytes;
  const int64_t n_tiles = static_cast<int64_t>(gp.n_mt) * gp.n_nt;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(ds->num_sms, n_tiles));
  // no base K blocks: the A map carries the weights' W blocks, the W map is unused
  lora_gemm_kernel<false, kEpiMergeAdd><<<grid, kGemmThreads, kGemmSmem, stream>>>(mW, mBl, mBl, mBl, mBl, mBl, gp);
  return launch_status();
}

}  // extern "C"

// The batched tall-skinny QR and post-hoc compression entry points (and their
// kernels' launch attributes, qr_kernel_attributes).
#include "qr_api.inc"
