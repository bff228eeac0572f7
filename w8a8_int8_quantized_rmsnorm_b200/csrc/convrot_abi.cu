// libconvrot.so: the C ABI declared in include/convrot.h.
//
// Host side only: argument validation, TMA tensor-map encoding, launch
// configuration and the work schedule of the GEMM.  All arithmetic of the
// method runs in the kernels of rowquant.cuh and gemm.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/convrot.h"
#include "actquant.cuh"
#include "gemm.cuh"
#include "gemm2sm.cuh"
#include "rowquant.cuh"
#include "selftest.cuh"

using namespace convrot;

namespace {

// ------------------------------------------------------------------ helpers
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

cudaStream_t as_cuda(convrot_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

struct DeviceInfo {
  int device = -1;
  int sms = 0;
};

DeviceInfo current_device() {
  static std::atomic<int> cached_sms[64];
  DeviceInfo d;
  if (cudaGetDevice(&d.device) != cudaSuccess || d.device < 0 || d.device >= 64) {
    d.device = -1;
    return d;
  }
  int v = cached_sms[d.device].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d.device) != cudaSuccess) v = 0;
    cached_sms[d.device].store(v, std::memory_order_relaxed);
  }
  d.sms = v;
  return d;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A 2-D row-major tensor [rows, cols] of elements of `esize` bytes, box
// [box_rows, box_cols], with or without the 128-byte swizzle.  Encoded maps
// are kept in a small per-thread cache keyed by everything they encode, so a
// steady stream of calls on the same buffers encodes nothing.
struct MapKey {
  const void* base;
  uint64_t rows, cols;
  uint32_t box_rows, box_cols;
  int dtype, esize, swizzle;
  bool operator==(const MapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && box_rows == o.box_rows &&
           box_cols == o.box_cols && dtype == o.dtype && esize == o.esize && swizzle == o.swizzle;
  }
};

bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, int esize,
              CUtensorMapDataType dtype, uint32_t box_rows, uint32_t box_cols, bool swizzle128) {
  constexpr int kCache = 32;
  struct Entry {
    MapKey key;
    CUtensorMap map;
    bool valid;
  };
  thread_local Entry cache[kCache] = {};
  thread_local int next = 0;
  const MapKey key{base, rows, cols, box_rows, box_cols, static_cast<int>(dtype), esize,
                   swizzle128 ? 1 : 0};
  for (int i = 0; i < kCache; ++i) {
    if (cache[i].valid && cache[i].key == key) {
      *map = cache[i].map;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE,
         swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  Entry& e = cache[next];
  next = (next + 1) % kCache;
  e.key = key;
  e.map = *map;
  e.valid = true;
  return true;
}

bool make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_rows, uint32_t box_bytes, bool swizzle128) {
  return make_map(map, base, rows, row_bytes, 1, CU_TENSOR_MAP_DATA_TYPE_UINT8, box_rows,
                  box_bytes, swizzle128);
}

// An N-d tiled map (N <= 3) of elements of `esize` bytes with the given
// dimensions (innermost first), byte strides of dimensions 1..N-1, box and
// swizzle mode; cached per thread like make_map.
bool make_map_nd(CUtensorMap* map, const void* base, int rank, CUtensorMapDataType dtype,
                 int esize, const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  struct Key {
    const void* base;
    int rank, dtype, esize, swz;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    bool operator==(const Key& o) const {
      return std::memcmp(this, &o, sizeof(Key)) == 0;
    }
  };
  struct Entry {
    Key key;
    CUtensorMap map;
    bool valid;
  };
  constexpr int kCache = 16;
  thread_local Entry cache[kCache] = {};
  thread_local int next = 0;
  Key key;
  std::memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = rank;
  key.dtype = static_cast<int>(dtype);
  key.esize = esize;
  key.swz = static_cast<int>(swizzle);
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides[i];
  }
  for (int i = 0; i < kCache; ++i) {
    if (cache[i].valid && cache[i].key == key) {
      *map = cache[i].map;
      return true;
    }
  }
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 3) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    if (i + 1 < rank) st[i] = strides[i];
  }
  const CUresult r = fn(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st,
                        bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  Entry& e = cache[next];
  next = (next + 1) % kCache;
  e.key = key;
  e.map = *map;
  e.valid = true;
  return true;
}

convrot_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA;
}

// Number of device timeouts convrot_device_status has reported.  A kernel that
// gave up on a bounded wait may have left partial sums and tile counters in
// its split-tile workspace; the library's own fixed workspace is cleared again
// before its next use when this count has moved.
std::atomic<unsigned> g_timeouts_reported{0};

// ------------------------------------------------------------------ rowquant
struct RowPlan {
  int team, rows_per_cta, passes;
  bool resident;
};

RowPlan plan_rows(int K) {
  const int groups = (K + 255) / 256;
  const int lanes = 4 * groups;  // four threads per virtual 256-group
  RowPlan p;
  if (lanes <= 32) {
    int t = 4;
    while (t < lanes) t <<= 1;
    p.team = t;
    p.passes = 1;
  } else if (lanes <= 256) {
    p.team = (lanes + 31) / 32 * 32;
    p.passes = 1;
  } else {
    p.team = 256;
    p.passes = (lanes + 255) / 256;
  }
  p.rows_per_cta = std::max(1, 256 / p.team);
  p.resident = p.passes == 1;
  return p;
}

// Launches a hot-path kernel with programmatic dependent launch (its set-up
// may overlap the tail of the previous kernel on the stream; the kernel waits
// for that kernel before touching memory) and, if cluster > 1, in clusters.
template <typename... KArgs, typename... Args>
convrot_status launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...) != cudaSuccess) return CONVROT_ERR_CUDA;
  return launch_status();
}

template <int GRP, int PRE, int QK, bool RES>
convrot_status launch_rowquant_t(const RowQuantArgs& a, int threads, cudaStream_t st) {
  auto k = rowquant_kernel<GRP, PRE, QK, RES>;
  const DeviceInfo d = current_device();
  // occupancy per (device, block size in warps), computed once
  static std::atomic<int> occ[64][33];
  const int slot = std::min(32, (threads + 31) / 32);
  int per_sm = d.device >= 0 ? occ[d.device][slot].load(std::memory_order_relaxed) : 0;
  if (per_sm == 0) {
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, threads, 0) != cudaSuccess)
      return CONVROT_ERR_CUDA;
    if (d.device >= 0) occ[d.device][slot].store(per_sm, std::memory_order_relaxed);
  }
  const int row_blocks = (a.rows + a.rows_per_cta - 1) / a.rows_per_cta;
  const int grid = std::max(1, std::min(row_blocks, std::max(1, per_sm) * std::max(1, d.sms)));
  return launch_pdl(k, dim3(grid), dim3(threads), 0, st, 1, a);
}

template <int GRP, int PRE, int QK>
convrot_status launch_rowquant_grp(const RowQuantArgs& a, const RowPlan& p, cudaStream_t st) {
  const int threads = p.team * p.rows_per_cta;
  return p.resident ? launch_rowquant_t<GRP, PRE, QK, true>(a, threads, st)
                    : launch_rowquant_t<GRP, PRE, QK, false>(a, threads, st);
}

// group: 256, 16 or 0 (no rotation)
template <int PRE, int QK>
convrot_status launch_rowquant_pre(RowQuantArgs& a, int group, cudaStream_t st) {
  const RowPlan p = plan_rows(a.K);
  a.team = p.team;
  a.rows_per_cta = p.rows_per_cta;
  a.passes = p.passes;
  if (group == 256) return launch_rowquant_grp<256, PRE, QK>(a, p, st);
  if (group == 16) return launch_rowquant_grp<16, PRE, QK>(a, p, st);
  return launch_rowquant_grp<0, PRE, QK>(a, p, st);
}

// TMA-fed activation kernel: one CTA per SM, a ring of stages of `rows`
// token rows each, teams of eight threads per 256-element group.  The rows
// are staged as [rows][K / 64][64] boxes and the norm weight as [K / 32][32]
// lines, both with the 128-byte swizzle.
template <int GRP, bool NORM, bool WIDE, int NW>
convrot_status launch_actquant_w(const ActArgs& a, const float* norm_w, cudaStream_t st) {
  auto k = actquant_kernel<GRP, NORM, WIDE, NW>;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return CONVROT_ERR_CUDA;
  CUtensorMap mx, mw;
  const uint64_t xdims[3] = {64, static_cast<uint64_t>(a.K / 64), static_cast<uint64_t>(a.M)};
  const uint64_t xstr[2] = {128, static_cast<uint64_t>(a.K) * 2};
  const uint32_t xbox[3] = {64, static_cast<uint32_t>(a.K / 64), static_cast<uint32_t>(a.group_rows)};
  if (!make_map_nd(&mx, a.x, 3, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, xdims, xstr, xbox,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return CONVROT_ERR_CUDA;
  if (NORM) {
    const uint64_t wdims[2] = {32, static_cast<uint64_t>(a.K / 32)};
    const uint64_t wstr[1] = {128};
    const uint32_t wbox[2] = {32, static_cast<uint32_t>(a.w_box_lines)};
    if (!make_map_nd(&mw, norm_w, 2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, wdims, wstr, wbox,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return CONVROT_ERR_CUDA;
  } else {
    std::memset(&mw, 0, sizeof(mw));
  }
  const int groups = a.rows / a.group_rows;
  const int dyn = 1024 + a.wsm_bytes + a.xpose_bytes + groups * a.stages * a.slot_stride;
  static std::atomic<bool> configured[64];
  if (!configured[d.device].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, AQ_SMEM_BUDGET) !=
        cudaSuccess)
      return CONVROT_ERR_CUDA;
    configured[d.device].store(true, std::memory_order_release);
  }
  const int units = (a.M + a.rows - 1) / a.rows;
  const int grid = std::max(1, std::min(units, d.sms));
  return launch_pdl(k, dim3(grid), dim3(a.team * a.rows), dyn, st, 1, mx, mw, a);
}

// teams of whole warps (K >= 1024) reduce with redux and a fixed shuffle
// tree; a CTA of 32 warps (64 registers per thread) where the plan filled
// more than 24 warps, otherwise 24 (80 registers)
template <int GRP, bool NORM>
convrot_status launch_actquant_t(const ActArgs& a, const float* norm_w, cudaStream_t st) {
  const bool w32 = a.team * a.rows > 32 * 24;
  if (a.team < 32) return launch_actquant_w<GRP, NORM, false, 24>(a, norm_w, st);
  return w32 ? launch_actquant_w<GRP, NORM, true, 32>(a, norm_w, st)
             : launch_actquant_w<GRP, NORM, true, 24>(a, norm_w, st);
}

// Team and stage plan of the activation kernel: eight threads per (virtual)
// 256-element group, padded to a power of two below a warp or to whole warps;
// as many rows per stage as fit in AQ_MAX_CWARPS consumer warps, but no more
// than needed to give every SM a row first.  Returns false when K is not a
// multiple of 64 (the staged lines), the row is wider than AQ_MAX_TEAM_WARPS
// warps or the ring would hold fewer than two stages (the caller then uses
// rowquant_kernel).
bool plan_actquant(int M, int K, int group, bool norm, int sms, ActArgs& a) {
  if (K % 64) return false;
  const int lanes = 8 * ((K + 255) / 256);
  int team;
  if (lanes <= 32) {
    team = 8;
    while (team < lanes) team <<= 1;
  } else {
    team = (lanes + 31) / 32 * 32;
  }
  if (team > 32 * AQ_MAX_TEAM_WARPS) return false;
  const int team_warps = std::max(1, team / 32);
  // 32 warps per CTA (64 registers) for whole-warp teams whose width divides
  // 32 warps; 24 warps (80 registers) otherwise
  const int cta_warps = (team >= 32 && 32 % team_warps == 0) ? 32 : 24;
  const int max_rows = team >= 32 ? cta_warps / team_warps : cta_warps * (32 / team);
  const int per_sm = (M + std::max(1, sms) - 1) / std::max(1, sms);
  int rows = std::max(1, std::min(max_rows, per_sm));
  if (team < 32) rows = (rows * team + 31) / 32 * 32 / team;  // whole consumer warps
  if (team > 32 && rows > AQ_MAX_SLOTS) rows = AQ_MAX_SLOTS;  // one named barrier per row slot
  if (rows > 256) return false;                               // TMA box dimension
  const int cwarps = rows * team / 32;
  a.team = team;
  a.rows = rows;
  const int wlines = K / 32;
  a.w_copies = norm ? (wlines + 255) / 256 : 0;
  a.w_box_lines = norm ? (wlines + a.w_copies - 1) / a.w_copies : 0;
  a.wsm_bytes = norm ? (a.w_copies * a.w_box_lines * 128 + 1023) / 1024 * 1024 : 0;
  a.xpose_bytes = group == 256 ? cwarps * AQ_XPOSE_WARP_BYTES : 0;
  // staging groups: one per team of whole warps, one per warp of narrow teams
  a.group_rows = team >= 32 ? 1 : 32 / team;
  const int groups = rows / a.group_rows;
  if (groups > AQ_MAX_RINGS) return false;
  a.slot_stride = (a.group_rows * K * 2 + 1023) / 1024 * 1024;
  a.stages = std::min(AQ_MAX_STAGES, (AQ_SMEM_BUDGET - 1024 - a.wsm_bytes - a.xpose_bytes) /
                                         (groups * a.slot_stride));
  return a.stages >= 2;
}

convrot_status check_group(int group, int K, int multiple) {
  if (group != 0 && group != 16 && group != 256) return CONVROT_ERR_UNSUPPORTED;
  if (K <= 0 || K > CONVROT_MAX_K) return CONVROT_ERR_SHAPE;
  if (K % multiple) return CONVROT_ERR_SHAPE;
  if (group == 256 && K % 256) return CONVROT_ERR_SHAPE;
  return CONVROT_OK;
}

// ------------------------------------------------------------------ GEMM plan
constexpr size_t kCounterBytes = 4096;

// Cost of stream-K's fix-up (partial-tile reductions at L2 and the finalising
// read-back) in stage-times, measured against plain waves on B200: small
// partial tiles (the token-tile of the swap kernel up to 64 wide, <= 32 KB per
// CTA) cost about six stages; 128- and 256-wide tiles (64-128 KB per CTA) so
// much more that plain waves won on every such shape measured.
int fixup_stages(bool swap, int bn) { return (swap && bn <= 64) ? 6 : 24; }

struct GemmPlan {
  bool swap;
  bool pair;   // CTA-pair kernel (256-row tiles); grid/units below count pairs
  bool split;  // pair kernel in split-K clusters of two pairs; grid counts clusters
  int bn;
  int tilesA, tilesB, num_tiles, num_kb;
  int grid;
  int dp_tiles, sk_iters, sk_q, sk_r;
  size_t ws_slot_bytes, ws_count_bytes;
};

int pick_bn_swap(int M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  return 128;
}

// `units` is the number of co-resident work units: SMs for the single-CTA
// kernel, CTA pairs (clusters of two) for the pair kernel.
// `clusters4` is the number of co-resident four-CTA clusters of the split
// pair kernel (0 if unavailable).
// wbf: the weight-only path (bf16 activations, int8 weights expanded to bf16
// in tensor memory, fp32 accumulators): swapped roles at every M (weights as
// the MMA's A operand, token tiles of up to 128 as B), K atoms of 64
// elements; stream-K only where every split tile has at most two parts (each
// unit's share is at least a whole tile), so that the fp32 sum of the parts
// does not depend on their order.
GemmPlan plan_gemm(int M, int N, int K, int sms, int pairs, bool w4, int clusters4,
                   bool wbf = false) {
  GemmPlan p{};
  p.swap = M <= 128 || wbf;
  p.pair = !p.swap && pairs > 0 && !wbf;
  p.bn = p.swap ? pick_bn_swap(M) : 256;
  const int rowsA = p.swap ? N : M;
  const int rowsB = p.swap ? M : N;
  const int tileA = p.pair ? 256 : GEMM_BM;
  p.tilesA = (rowsA + tileA - 1) / tileA;
  p.tilesB = (rowsB + p.bn - 1) / p.bn;
  p.num_tiles = p.tilesA * p.tilesB;
  const int stage_k = wbf ? (GEMM_BK / 2) * wbf_katoms(p.bn)
                          : GEMM_BK * gemm_katoms(w4, p.pair, p.swap);
  p.num_kb = (K + stage_k - 1) / stage_k;
  // One wave of 256 x 256 tiles that fits the co-resident clusters: each tile
  // is split in two K halves over two CTA pairs whose partial sums meet in
  // shared memory (no stream-K workspace, no L2 round trip).
  if (p.pair && !w4 && !wbf && clusters4 > 0 && p.num_kb >= 2 && p.num_tiles <= clusters4) {
    p.split = true;
    p.grid = p.num_tiles;
    p.dp_tiles = 0;
    p.sk_iters = p.sk_q = p.sk_r = 0;
    p.ws_slot_bytes = p.ws_count_bytes = 0;
    return p;
  }
  const long long total = static_cast<long long>(p.num_tiles) * p.num_kb;
  const int units = p.pair ? pairs : sms;
  // at most 2 * units tiles are split (each with one counter per CTA of the
  // unit), so the fixed counter region always fits
  const int max_grid = static_cast<int>(kCounterBytes / 4 / 4);
  p.grid = static_cast<int>(std::min<long long>(std::min(std::max(1, units), max_grid), total));
  const int waves = p.num_tiles / p.grid;
  p.dp_tiles = waves >= 2 ? (waves - 1) * p.grid : 0;
  int sk_tiles = p.num_tiles - p.dp_tiles;
  // Stream-K evens out the last waves but pays for its split tiles (partial
  // reductions and the finalising read-back, fixup_stages() stage-times).
  // In stage units per unit: whole waves, against the data-parallel waves plus
  // the evened-out remainder plus the fix-up.  Ties go to plain waves.
  const long long t_dp = static_cast<long long>((p.num_tiles + p.grid - 1) / p.grid) * p.num_kb;
  const long long sk_total = static_cast<long long>(sk_tiles) * p.num_kb;
  const long long t_sk = static_cast<long long>(p.dp_tiles / p.grid) * p.num_kb +
                         (sk_total + p.grid - 1) / p.grid + fixup_stages(p.swap, p.bn);
  const bool two_parts = sk_tiles * p.num_kb / p.grid >= p.num_kb;
  if ((wbf && !two_parts) || t_dp <= t_sk) {
    p.dp_tiles = p.num_tiles;
    sk_tiles = 0;
  }
  p.sk_iters = sk_tiles * p.num_kb;
  p.sk_q = p.sk_iters / p.grid;
  p.sk_r = p.sk_iters % p.grid;
  // a stream-K region whose iterations split evenly into whole tiles needs no workspace
  const bool whole = p.sk_r == 0 && p.sk_q % p.num_kb == 0;
  // one int32 accumulator tile (and one counter) per split tile and CTA
  const int ctas_per_unit = p.pair ? 2 : 1;
  p.ws_slot_bytes =
      whole ? 0 : static_cast<size_t>(sk_tiles) * ctas_per_unit * GEMM_BM * p.bn * 4;
  p.ws_count_bytes = whole ? 0 : static_cast<size_t>(sk_tiles) * ctas_per_unit * 4;
  return p;
}

// Co-resident clusters of two CTAs of the pair kernel (once per device).
template <bool W4, int EPI>
int pair_units(int device) {
  static std::atomic<int> cached[64];
  if (device < 0 || device >= 64) return 0;
  int v = cached[device].load(std::memory_order_relaxed);
  if (v != 0) return v;
  using SM = Gemm2Smem<W4>;
  auto k = gemm2sm_kernel<W4, EPI>;
  const int avail = 227 * 1024 - 1024 - SM::total(0);
  const int stages = std::max(2, std::min(GEMM_MAX_STAGES, avail / SM::STAGE));
  const int smem = SM::total(stages) + 1024;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return -1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(W4 ? 448 : 320, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, k, &cfg) != cudaSuccess || clusters <= 0) {
    cudaGetLastError();
    clusters = -1;  // pair kernel unavailable: fall back to single-CTA tiles
  }
  cached[device].store(clusters, std::memory_order_relaxed);
  return clusters;
}

// Co-resident clusters of four CTAs of the split pair kernel (once per device).
template <int EPI>
int split_units(int device) {
  static std::atomic<int> cached[64];
  if (device < 0 || device >= 64) return 0;
  int v = cached[device].load(std::memory_order_relaxed);
  if (v != 0) return v;
  using SM = Gemm2Smem<false>;
  auto k = gemm2sm_kernel<false, EPI, true>;
  const int avail = 227 * 1024 - 1024 - SM::total(0);
  const int stages = std::max(2, std::min(GEMM_MAX_STAGES, avail / SM::STAGE));
  const int smem = SM::total(stages) + 1024;
  int clusters = 0;
  if (stages * SM::STAGE >= 2 * SPLIT_RECV_BYTES &&  // receive area + send staging
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(4, 1, 1);
    cfg.blockDim = dim3(320, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 4;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&clusters, k, &cfg) != cudaSuccess) clusters = 0;
  }
  cudaGetLastError();
  if (clusters <= 0) clusters = -1;  // split mode unavailable
  cached[device].store(clusters, std::memory_order_relaxed);
  return clusters;
}

// `epi` is the epilogue mode (EPI_BF16, EPI_S32 or EPI_SWIGLU).
int split_units_for(bool w4, int epi, int device) {
  if (w4 || epi == EPI_SWIGLU) return 0;  // the split-K cluster mode is int8 and plain only
  const int c = epi == EPI_S32 ? split_units<EPI_S32>(device) : split_units<EPI_BF16>(device);
  return c > 0 ? c : 0;
}

int pair_units_for(bool w4, int epi, int device) {
  if (w4) {
    if (epi == EPI_SWIGLU) return pair_units<true, EPI_SWIGLU>(device);
    return epi == EPI_S32 ? pair_units<true, EPI_S32>(device) : pair_units<true, EPI_BF16>(device);
  }
  if (epi == EPI_SWIGLU) return pair_units<false, EPI_SWIGLU>(device);
  return epi == EPI_S32 ? pair_units<false, EPI_S32>(device) : pair_units<false, EPI_BF16>(device);
}

GemmPlan plan_for(int M, int N, int K, bool w4, int epi, const DeviceInfo& d) {
  return plan_gemm(M, N, K, d.sms, pair_units_for(w4, epi, d.device), w4,
                   split_units_for(w4, epi, d.device));
}

// `units` counts CTA pairs, or (SPLIT) clusters of two pairs.
template <bool W4, int EPI, bool SPLIT = false>
convrot_status launch_gemm_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& my,
                                GemmArgs a, int units, cudaStream_t st) {
  using SM = Gemm2Smem<W4>;
  auto k = gemm2sm_kernel<W4, EPI, SPLIT>;
  const int avail = 227 * 1024 - 1024 - SM::total(0);
  const int stages = std::max(2, std::min(GEMM_MAX_STAGES, avail / SM::STAGE));
  a.stages = stages;
  const int smem = SM::total(stages) + 1024;
  const int cluster = SPLIT ? 4 : 2;
  return launch_pdl(k, dim3(cluster * units), dim3(W4 ? 448 : 320), smem, st, cluster, ma, mb, my, a);
}

// Rasterisation group of the pair kernel: as many A tiles (256 rows x K
// bytes) as fit ~40 MB, so that a group's activations stay in L2 while the
// weight tiles stream past and each weight tile is read from DRAM once per
// group (8192 x 24576 x 4096: a group of 32 instead of 8 cut the GEMM from
// 622 to 602 us, measured; fewer DRAM bytes, a higher clock under the power
// cap).
int pair_group(int K, int tilesA) {
  const long long g = (40LL << 20) / (256LL * std::max(1, K));
  return static_cast<int>(std::max(1LL, std::min<long long>(tilesA, g)));
}

// Workspace layout: a fixed region of tile counters at offset 0, then one
// int32 accumulator tile per split tile and CTA.  Every successful call leaves
// the whole buffer zero (the finalising CTA re-zeroes its accumulator and
// counter), so one zero-filled buffer serves calls of any shape.
size_t ws_bytes(const GemmPlan& p) {
  if (p.ws_slot_bytes == 0) return 0;
  return kCounterBytes + p.ws_slot_bytes;
}

template <int BN, bool SWAP, bool W4, int EPI, bool WBF = false>
convrot_status launch_gemm_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& my,
                             GemmArgs a, int grid, cudaStream_t st) {
  using SM = GemmSmem<BN, W4 || WBF, SWAP, WBF ? wbf_katoms(BN) : 0, WBF>;
  auto k = gemm_kernel<BN, SWAP, W4, EPI, WBF>;
  // as many stages as fit next to the epilogue staging and the barriers in
  // 227 KB; at least ~116 KB so that a second CTA never shares the SM's TMEM
  const int avail = 227 * 1024 - 1024 - SM::total(0);
  int stages = std::min(GEMM_MAX_STAGES, avail / SM::STAGE);
  stages = std::max(2, stages);
  a.stages = stages;
  const int smem = std::max(SM::total(stages) + 1024, 116 * 1024);
  static std::atomic<bool> configured[64];  // per instantiation and device
  const DeviceInfo d = current_device();
  if (d.device < 0) return CONVROT_ERR_CUDA;
  if (!configured[d.device].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return CONVROT_ERR_CUDA;
    configured[d.device].store(true, std::memory_order_release);
  }
  constexpr int threads = (W4 || WBF) ? 320 : 192;
  return launch_pdl(k, dim3(grid), dim3(threads), smem, st, 1, ma, mb, my, a);
}

template <int EPI>
convrot_status launch_wbf(int bn, const CUtensorMap& ma, const CUtensorMap& mb,
                          const CUtensorMap& my, const GemmArgs& a, int grid, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_gemm_t<16, true, false, EPI, true>(ma, mb, my, a, grid, st);
    case 32: return launch_gemm_t<32, true, false, EPI, true>(ma, mb, my, a, grid, st);
    case 64: return launch_gemm_t<64, true, false, EPI, true>(ma, mb, my, a, grid, st);
    default: return launch_gemm_t<128, true, false, EPI, true>(ma, mb, my, a, grid, st);
  }
}

// Weight-only path: Xr bf16 [M, K] (rotated activations), Wq int8 [N, K];
// out bf16 Y = (Xr Wq^T) * s_row, or raw fp32 accumulators (f32_out).
convrot_status run_gemm_wbf(const void* Xr, const int8_t* Wq, const float* s_row, int M, int N,
                            int K, void* out, bool f32_out, void* workspace, size_t workspace_bytes,
                            cudaStream_t st) {
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return CONVROT_ERR_CUDA;
  const GemmPlan p = plan_gemm(M, N, K, d.sms, 0, false, 0, true);
  const size_t need = ws_bytes(p);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return CONVROT_ERR_WORKSPACE;
  if (need > 0 && !aligned(workspace, 256)) return CONVROT_ERR_ALIGN;
  const int bn = p.bn;
  CUtensorMap mx, mw, my;
  std::memset(&my, 0, sizeof(my));
  // swapped roles: token atoms of 64 elements (128 bytes of a bf16 row,
  // swizzled like the int8 atoms); the weights land as boxes of 128 rows x
  // 128 bytes (two atoms) with the 128-byte swizzle and are expanded into
  // tensor memory
  if (!make_map(&mx, Xr, M, K, 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, bn, GEMM_BK / 2, true))
    return CONVROT_ERR_CUDA;
  if (!make_map_u8(&mw, Wq, N, K, GEMM_BM, GEMM_BK, true)) return CONVROT_ERR_CUDA;
  // the output as chunks of up to 32 tokens x 128 columns, unswizzled
  const uint32_t cw = bn < 32 ? bn : 32;
  const bool ok = f32_out ? make_map(&my, out, M, N, 4, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, cw, 128, false)
                          : make_map(&my, out, M, N, 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cw, 128, false);
  if (!ok) return CONVROT_ERR_CUDA;
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.rowsA = N;
  a.rowsB = M;
  a.tilesA = p.tilesA;
  a.tilesB = p.tilesB;
  a.group_a = GEMM_GROUP_A;
  a.num_tiles = p.num_tiles;
  a.num_kb = p.num_kb;
  a.dp_tiles = p.dp_tiles;
  a.sk_iters = p.sk_iters;
  a.sk_q = p.sk_q;
  a.sk_r = p.sk_r;
  a.ws_counts = need ? static_cast<unsigned*>(workspace) : nullptr;
  a.ws_acc = need ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + kCounterBytes)
                  : nullptr;
  a.s_tok = nullptr;
  a.s_row = s_row;
  a.srow_vec = (s_row != nullptr && aligned(s_row, 16)) ? 1 : 0;
  a.out = out;
  return f32_out ? launch_wbf<EPI_S32>(bn, mw, mx, my, a, p.grid, st)
                 : launch_wbf<EPI_BF16>(bn, mw, mx, my, a, p.grid, st);
}

template <bool SWAP, bool W4, int EPI>
convrot_status launch_gemm_bn(int bn, const CUtensorMap& ma, const CUtensorMap& mb,
                              const CUtensorMap& my, const GemmArgs& a, int grid,
                              cudaStream_t st) {
  if (!SWAP) return launch_gemm_t<256, false, W4, EPI>(ma, mb, my, a, grid, st);
  switch (bn) {
    case 16: return launch_gemm_t<16, true, W4, EPI>(ma, mb, my, a, grid, st);
    case 32: return launch_gemm_t<32, true, W4, EPI>(ma, mb, my, a, grid, st);
    case 64: return launch_gemm_t<64, true, W4, EPI>(ma, mb, my, a, grid, st);
    default: return launch_gemm_t<128, true, W4, EPI>(ma, mb, my, a, grid, st);
  }
}

template <bool SWAP, bool W4>
convrot_status launch_gemm_epi(int epi, int bn, const CUtensorMap& ma, const CUtensorMap& mb,
                               const CUtensorMap& my, const GemmArgs& a, int grid, cudaStream_t st) {
  if (epi == EPI_S32) return launch_gemm_bn<SWAP, W4, EPI_S32>(bn, ma, mb, my, a, grid, st);
  if (epi == EPI_SWIGLU) return launch_gemm_bn<SWAP, W4, EPI_SWIGLU>(bn, ma, mb, my, a, grid, st);
  return launch_gemm_bn<SWAP, W4, EPI_BF16>(bn, ma, mb, my, a, grid, st);
}

template <bool W4>
convrot_status launch_pair_epi(int epi, const CUtensorMap& ma, const CUtensorMap& mb,
                               const CUtensorMap& my, const GemmArgs& a, int units, cudaStream_t st) {
  if (epi == EPI_S32) return launch_gemm_pair<W4, EPI_S32>(ma, mb, my, a, units, st);
  if (epi == EPI_SWIGLU) return launch_gemm_pair<W4, EPI_SWIGLU>(ma, mb, my, a, units, st);
  return launch_gemm_pair<W4, EPI_BF16>(ma, mb, my, a, units, st);
}

// epi = EPI_BF16 (Y bf16 [M, N]), EPI_S32 (acc int32 [M, N]) or EPI_SWIGLU
// (H bf16 [M, N / 2] from interleaved gate/up weight rows).
convrot_status run_gemm(const int8_t* Xq, const void* Wq, bool w4, const float* s_tok,
                        const float* s_row, int M, int N, int K, void* out, int epi,
                        void* workspace, size_t workspace_bytes, cudaStream_t st) {
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return CONVROT_ERR_CUDA;
  const bool s32_out = epi == EPI_S32;
  const GemmPlan p = plan_for(M, N, K, w4, epi, d);
  const size_t need = ws_bytes(p);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return CONVROT_ERR_WORKSPACE;
  if (need > 0 && !aligned(workspace, 256)) return CONVROT_ERR_ALIGN;

  const int bn = p.bn;
  CUtensorMap mx, mw;
  // activations: int8 [M, K]; weights: int8 [N, K] or packed [N, K/2].  Each
  // CTA of a pair loads 128 rows of each operand.
  const uint32_t x_box_rows = p.swap ? bn : GEMM_BM;
  const uint32_t w_box_rows = (p.swap || p.pair) ? GEMM_BM : bn;
  if (!make_map_u8(&mx, Xq, M, K, x_box_rows, GEMM_BK, true)) return CONVROT_ERR_CUDA;
  if (w4) {
    if (!make_map_u8(&mw, Wq, N, K / 2, w_box_rows, GEMM_BK / 2, false)) return CONVROT_ERR_CUDA;
  } else {
    if (!make_map_u8(&mw, Wq, N, K, w_box_rows, GEMM_BK, true)) return CONVROT_ERR_CUDA;
  }

  // output map for the epilogues' TMA stores
  CUtensorMap my;
  std::memset(&my, 0, sizeof(my));
  // the SwiGLU epilogue writes N / 2 columns: 64 per staged row, or 64 per
  // 128-row tile of the swapped roles
  const uint64_t out_cols = epi == EPI_SWIGLU ? N / 2 : N;
  if (!p.swap) {
    const bool ok = s32_out ? make_map(&my, out, M, N, 4, CU_TENSOR_MAP_DATA_TYPE_INT32, 32, 32, true)
                            : make_map(&my, out, M, out_cols, 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 32, 64, true);
    if (!ok) return CONVROT_ERR_CUDA;
  } else {
    // swapped roles: chunks of up to 32 tokens x 128 output columns, unswizzled
    const uint32_t cw = bn < 32 ? bn : 32;
    const uint32_t box_cols = epi == EPI_SWIGLU ? 64 : 128;
    const bool ok = s32_out ? make_map(&my, out, M, N, 4, CU_TENSOR_MAP_DATA_TYPE_INT32, cw, 128, false)
                            : make_map(&my, out, M, out_cols, 2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cw, box_cols, false);
    if (!ok) return CONVROT_ERR_CUDA;
  }

  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.rowsA = p.swap ? N : M;
  a.rowsB = p.swap ? M : N;
  a.tilesA = p.tilesA;
  a.tilesB = p.tilesB;
  a.group_a = p.pair ? pair_group(K, p.tilesA) : GEMM_GROUP_A;
  a.num_tiles = p.num_tiles;
  a.num_kb = p.num_kb;
  a.dp_tiles = p.dp_tiles;
  a.sk_iters = p.sk_iters;
  a.sk_q = p.sk_q;
  a.sk_r = p.sk_r;
  a.s_tok = s_tok;
  a.s_row = s_row;
  a.srow_vec = (s_row != nullptr && aligned(s_row, 16)) ? 1 : 0;
  a.out = out;
  a.ws_counts = need ? static_cast<unsigned*>(workspace) : nullptr;
  a.ws_acc = need ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + kCounterBytes)
                  : nullptr;
  const CUtensorMap& ma = p.swap ? mw : mx;
  const CUtensorMap& mb = p.swap ? mx : mw;
  if (p.split)  // never for EPI_SWIGLU (split_units_for gives no clusters)
    return s32_out ? launch_gemm_pair<false, EPI_S32, true>(ma, mb, my, a, p.grid, st)
                   : launch_gemm_pair<false, EPI_BF16, true>(ma, mb, my, a, p.grid, st);
  if (p.pair)
    return w4 ? launch_pair_epi<true>(epi, ma, mb, my, a, p.grid, st)
              : launch_pair_epi<false>(epi, ma, mb, my, a, p.grid, st);
  if (w4)
    return p.swap ? launch_gemm_epi<true, true>(epi, bn, ma, mb, my, a, p.grid, st)
                  : launch_gemm_epi<false, true>(epi, bn, ma, mb, my, a, p.grid, st);
  return p.swap ? launch_gemm_epi<true, false>(epi, bn, ma, mb, my, a, p.grid, st)
                : launch_gemm_epi<false, false>(epi, bn, ma, mb, my, a, p.grid, st);
}

convrot_status check_gemm_shape(int M, int N, int K, bool w4) {
  if (M < 0 || N < 0 || K <= 0 || K > CONVROT_MAX_K) return CONVROT_ERR_SHAPE;
  if (K % (w4 ? 32 : 16)) return CONVROT_ERR_SHAPE;
  if (N % 8) return CONVROT_ERR_SHAPE;
  return CONVROT_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int convrot_version(void) { return (1 << 16) | 0; }

const char* convrot_status_string(convrot_status st) {
  switch (st) {
    case CONVROT_OK: return "CONVROT_OK";
    case CONVROT_ERR_NULL: return "CONVROT_ERR_NULL: a required pointer is NULL";
    case CONVROT_ERR_SHAPE: return "CONVROT_ERR_SHAPE: unsupported or inconsistent size";
    case CONVROT_ERR_ALIGN: return "CONVROT_ERR_ALIGN: pointer not aligned as required";
    case CONVROT_ERR_UNSUPPORTED: return "CONVROT_ERR_UNSUPPORTED: unsupported option";
    case CONVROT_ERR_CUDA: return "CONVROT_ERR_CUDA: a CUDA call failed";
    case CONVROT_ERR_DEVICE_TIMEOUT: return "CONVROT_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    case CONVROT_ERR_WORKSPACE: return "CONVROT_ERR_WORKSPACE: workspace missing or too small";
  }
  return "CONVROT_ERR_UNKNOWN";
}

convrot_status convrot_device_status(convrot_stream_t stream, uint32_t* detail) {
  if (cudaStreamSynchronize(as_cuda(stream)) != cudaSuccess) return CONVROT_ERR_CUDA;
  unsigned v = 0;
  const unsigned zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  if (detail) *detail = v;
  if (v) g_timeouts_reported.fetch_add(1u, std::memory_order_relaxed);
  return v ? CONVROT_ERR_DEVICE_TIMEOUT : CONVROT_OK;
}

convrot_status convrot_selftest_wait_timeout(uint32_t limit_cycles, convrot_stream_t stream) {
  if (limit_cycles < 1000u || limit_cycles > 100000000u) return CONVROT_ERR_SHAPE;
  selftest_wait_timeout_kernel<<<1, 32, 0, as_cuda(stream)>>>(static_cast<long long>(limit_cycles));
  return launch_status();
}

convrot_status convrot_quantize_weight(const void* W, int N, int K, int group,
                                       const float* col_scale, int8_t* Wq, float* s_row,
                                       convrot_stream_t stream) {
  if (N < 0) return CONVROT_ERR_SHAPE;
  const convrot_status g = check_group(group, K, 16);
  if (g != CONVROT_OK) return g;
  if (N == 0) return CONVROT_OK;
  if (!W || !Wq || !s_row) return CONVROT_ERR_NULL;
  if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(s_row, 4)) return CONVROT_ERR_ALIGN;
  if (col_scale && !aligned(col_scale, 16)) return CONVROT_ERR_ALIGN;
  RowQuantArgs a{};
  a.src = static_cast<const uint16_t*>(W);
  a.vec = col_scale;
  a.dst8 = Wq;
  a.scale = s_row;
  a.rows = N;
  a.K = K;
  return col_scale ? launch_rowquant_pre<PRE_COLSCALE, QK_INT8>(a, group, as_cuda(stream))
                   : launch_rowquant_pre<PRE_NONE, QK_INT8>(a, group, as_cuda(stream));
}

convrot_status convrot_quantize_weight_w4(const void* W, int N, int K, int group,
                                          const float* col_scale, float clip_lo,
                                          float clip_hi, int clip_steps, uint8_t* Wq4,
                                          float* s_row, convrot_stream_t stream) {
  if (N < 0) return CONVROT_ERR_SHAPE;
  const convrot_status g = check_group(group, K, 32);
  if (g != CONVROT_OK) return g;
  if (clip_steps < 1 || clip_steps > 64 || !(clip_lo > 0.f) || !(clip_hi >= clip_lo))
    return CONVROT_ERR_SHAPE;
  if (N == 0) return CONVROT_OK;
  if (!W || !Wq4 || !s_row) return CONVROT_ERR_NULL;
  if (!aligned(W, 16) || !aligned(Wq4, 16) || !aligned(s_row, 4)) return CONVROT_ERR_ALIGN;
  if (col_scale && !aligned(col_scale, 16)) return CONVROT_ERR_ALIGN;
  RowQuantArgs a{};
  a.src = static_cast<const uint16_t*>(W);
  a.vec = col_scale;
  a.dst4 = Wq4;
  a.scale = s_row;
  a.rows = N;
  a.K = K;
  if (clip_steps == 1) {
    a.clip_lo = clip_hi;
    a.clip_step = 0.f;
  } else {
    a.clip_lo = clip_lo;
    a.clip_step = static_cast<float>((static_cast<double>(clip_hi) - clip_lo) / (clip_steps - 1));
  }
  a.clip_steps = clip_steps;
  return col_scale ? launch_rowquant_pre<PRE_COLSCALE, QK_INT4>(a, group, as_cuda(stream))
                   : launch_rowquant_pre<PRE_NONE, QK_INT4>(a, group, as_cuda(stream));
}

convrot_status convrot_rotate_quant_act(const void* x, int M, int K, int group,
                                        const float* norm_w, float eps, int8_t* Xq,
                                        float* s_tok, convrot_stream_t stream) {
  if (M < 0) return CONVROT_ERR_SHAPE;
  const convrot_status g = check_group(group, K, 16);
  if (g != CONVROT_OK) return g;
  if (norm_w && !(eps >= 0.f)) return CONVROT_ERR_SHAPE;
  if (M == 0) return CONVROT_OK;
  if (!x || !Xq || !s_tok) return CONVROT_ERR_NULL;
  if (!aligned(x, 16) || !aligned(Xq, 16) || !aligned(s_tok, 4)) return CONVROT_ERR_ALIGN;
  if (norm_w && !aligned(norm_w, 16)) return CONVROT_ERR_ALIGN;
  ActArgs q{};
  q.x = static_cast<const uint16_t*>(x);
  q.xq = Xq;
  q.s_tok = s_tok;
  q.M = M;
  q.K = K;
  q.eps = eps;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return CONVROT_ERR_CUDA;
  if (plan_actquant(M, K, group, norm_w != nullptr, d.sms, q)) {
    cudaStream_t st = as_cuda(stream);
    if (group == 256)
      return norm_w ? launch_actquant_t<256, true>(q, norm_w, st)
                    : launch_actquant_t<256, false>(q, norm_w, st);
    if (group == 16)
      return norm_w ? launch_actquant_t<16, true>(q, norm_w, st)
                    : launch_actquant_t<16, false>(q, norm_w, st);
    return norm_w ? launch_actquant_t<0, true>(q, norm_w, st)
                  : launch_actquant_t<0, false>(q, norm_w, st);
  }
  RowQuantArgs a{};
  a.src = static_cast<const uint16_t*>(x);
  a.vec = norm_w;
  a.dst8 = Xq;
  a.scale = s_tok;
  a.rows = M;
  a.K = K;
  a.eps = eps;
  return norm_w ? launch_rowquant_pre<PRE_NORM, QK_INT8>(a, group, as_cuda(stream))
                : launch_rowquant_pre<PRE_NONE, QK_INT8>(a, group, as_cuda(stream));
}

convrot_status convrot_smoothquant_calibrate(const void* x, int M, int K, const float* norm_w,
                                             float eps, const void* W, int N, float alpha,
                                             float* smooth, float* norm_w_folded,
                                             convrot_stream_t stream) {
  if (M <= 0 || N <= 0 || K <= 0 || K > CONVROT_MAX_K || K % 16) return CONVROT_ERR_SHAPE;
  if (!(alpha >= 0.f && alpha <= 1.f) || !(eps >= 0.f)) return CONVROT_ERR_SHAPE;
  if (!x || !W || !smooth || !norm_w_folded) return CONVROT_ERR_NULL;
  if (!aligned(x, 16) || !aligned(W, 16) || (norm_w && !aligned(norm_w, 4)) || !aligned(smooth, 4) ||
      !aligned(norm_w_folded, 4))
    return CONVROT_ERR_ALIGN;
  if (norm_w_folded == norm_w) return CONVROT_ERR_UNSUPPORTED;
  cudaStream_t st = as_cuda(stream);
  if (cudaMemsetAsync(smooth, 0, sizeof(float) * K, st) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (cudaMemsetAsync(norm_w_folded, 0, sizeof(float) * K, st) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  calib_act_colmax<<<(M + CAL_ROWS - 1) / CAL_ROWS, 256, 0, st>>>(
      static_cast<const uint16_t*>(x), M, K, norm_w, eps, reinterpret_cast<unsigned*>(smooth));
  calib_weight_colmax<<<(N + CAL_ROWS - 1) / CAL_ROWS, 256, 0, st>>>(
      static_cast<const uint16_t*>(W), N, K, reinterpret_cast<unsigned*>(norm_w_folded));
  calib_finalize<<<(K + 255) / 256, 256, 0, st>>>(norm_w, K, alpha, smooth, norm_w_folded);
  return launch_status();
}

size_t convrot_linear_workspace_bytes(int M, int N, int K, int weight_bits) {
  if (check_gemm_shape(M, N, K, weight_bits == 4) != CONVROT_OK) return 0;
  if (weight_bits != 8 && weight_bits != 4) return 0;
  if (M == 0 || N == 0) return 0;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return 0;
  // the bf16 and int32 outputs share the schedule, so either plan gives the size
  return ws_bytes(plan_for(M, N, K, weight_bits == 4, EPI_BF16, d));
}

size_t convrot_swiglu_workspace_bytes(int M, int I, int K, int weight_bits) {
  if (I <= 0 || I % SWIGLU_BLOCK || I > (1 << 29)) return 0;
  if (check_gemm_shape(M, 2 * I, K, weight_bits == 4) != CONVROT_OK) return 0;
  if (weight_bits != 8 && weight_bits != 4) return 0;
  if (M == 0) return 0;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return 0;
  return ws_bytes(plan_for(M, 2 * I, K, weight_bits == 4, EPI_SWIGLU, d));
}

static convrot_status linear_common(const int8_t* Xq, const float* s_tok, const void* Wq,
                                    bool w4, const float* s_row, int M, int N, int K, void* Y,
                                    void* workspace, size_t workspace_bytes,
                                    convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, w4);
  if (sh != CONVROT_OK) return sh;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (!Xq || !s_tok || !Wq || !s_row || !Y) return CONVROT_ERR_NULL;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(s_tok, 4) ||
      !aligned(s_row, 4))
    return CONVROT_ERR_ALIGN;
  return run_gemm(Xq, Wq, w4, s_tok, s_row, M, N, K, Y, EPI_BF16, workspace, workspace_bytes,
                  as_cuda(stream));
}

static convrot_status swiglu_common(const int8_t* Xq, const float* s_tok, const void* Wq_gu,
                                    bool w4, const float* s_row_gu, int M, int I, int K, void* H,
                                    void* workspace, size_t workspace_bytes,
                                    convrot_stream_t stream) {
  if (M < 0 || I <= 0 || I % SWIGLU_BLOCK || I > (1 << 29)) return CONVROT_ERR_SHAPE;
  const convrot_status sh = check_gemm_shape(M, 2 * I, K, w4);
  if (sh != CONVROT_OK) return sh;
  if (M == 0) return CONVROT_OK;
  if (!Xq || !s_tok || !Wq_gu || !s_row_gu || !H) return CONVROT_ERR_NULL;
  if (!aligned(Xq, 16) || !aligned(Wq_gu, 16) || !aligned(H, 16) || !aligned(s_tok, 4) ||
      !aligned(s_row_gu, 4))
    return CONVROT_ERR_ALIGN;
  return run_gemm(Xq, Wq_gu, w4, s_tok, s_row_gu, M, 2 * I, K, H, EPI_SWIGLU, workspace,
                  workspace_bytes, as_cuda(stream));
}

convrot_status convrot_int8_linear_swiglu(const int8_t* Xq, const float* s_tok,
                                          const int8_t* Wq_gu, const float* s_row_gu, int M,
                                          int I, int K, void* H, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream) {
  return swiglu_common(Xq, s_tok, Wq_gu, false, s_row_gu, M, I, K, H, workspace,
                       workspace_bytes, stream);
}

convrot_status convrot_w4a8_linear_swiglu(const int8_t* Xq, const float* s_tok,
                                          const uint8_t* Wq4_gu, const float* s_row_gu, int M,
                                          int I, int K, void* H, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream) {
  return swiglu_common(Xq, s_tok, Wq4_gu, true, s_row_gu, M, I, K, H, workspace,
                       workspace_bytes, stream);
}

convrot_status convrot_rotate_act_bf16(const void* x, int M, int K, int group,
                                       const float* norm_w, float eps, void* Xr,
                                       convrot_stream_t stream) {
  if (M < 0) return CONVROT_ERR_SHAPE;
  const convrot_status g = check_group(group, K, 16);
  if (g != CONVROT_OK) return g;
  if (norm_w && !(eps >= 0.f)) return CONVROT_ERR_SHAPE;
  if (M == 0) return CONVROT_OK;
  if (!x || !Xr) return CONVROT_ERR_NULL;
  if (!aligned(x, 16) || !aligned(Xr, 16)) return CONVROT_ERR_ALIGN;
  if (norm_w && !aligned(norm_w, 16)) return CONVROT_ERR_ALIGN;
  RowQuantArgs a{};
  a.src = static_cast<const uint16_t*>(x);
  a.vec = norm_w;
  a.dstb = static_cast<uint16_t*>(Xr);
  a.rows = M;
  a.K = K;
  a.eps = eps;
  return norm_w ? launch_rowquant_pre<PRE_NORM, QK_BF16>(a, group, as_cuda(stream))
                : launch_rowquant_pre<PRE_NONE, QK_BF16>(a, group, as_cuda(stream));
}

size_t convrot_weight_only_workspace_bytes(int M, int N, int K) {
  if (check_gemm_shape(M, N, K, false) != CONVROT_OK || M == 0 || N == 0) return 0;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return 0;
  return ws_bytes(plan_gemm(M, N, K, d.sms, 0, false, 0, true));
}

static convrot_status weight_only_common(const void* Xr, const int8_t* Wq, const float* s_row,
                                         int M, int N, int K, void* out, bool f32_out,
                                         void* workspace, size_t workspace_bytes,
                                         convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, false);
  if (sh != CONVROT_OK) return sh;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (!Xr || !Wq || !out || (!f32_out && !s_row)) return CONVROT_ERR_NULL;
  if (!aligned(Xr, 16) || !aligned(Wq, 16) || !aligned(out, 16) || (s_row && !aligned(s_row, 4)))
    return CONVROT_ERR_ALIGN;
  return run_gemm_wbf(Xr, Wq, s_row, M, N, K, out, f32_out, workspace, workspace_bytes,
                      as_cuda(stream));
}

convrot_status convrot_weight_only_linear(const void* Xr, const int8_t* Wq, const float* s_row,
                                          int M, int N, int K, void* Y, void* workspace,
                                          size_t workspace_bytes, convrot_stream_t stream) {
  return weight_only_common(Xr, Wq, s_row, M, N, K, Y, false, workspace, workspace_bytes, stream);
}

convrot_status convrot_weight_only_gemm_f32(const void* Xr, const int8_t* Wq, int M, int N, int K,
                                            float* acc, void* workspace, size_t workspace_bytes,
                                            convrot_stream_t stream) {
  return weight_only_common(Xr, Wq, nullptr, M, N, K, acc, true, workspace, workspace_bytes,
                            stream);
}

convrot_status convrot_interleave_gate_up(const void* Wg, const void* Wu, int I,
                                          size_t row_bytes, void* out, convrot_stream_t stream) {
  if (I <= 0 || I % SWIGLU_BLOCK || row_bytes == 0 || row_bytes % 4 ||
      row_bytes > (static_cast<size_t>(1) << 30))
    return CONVROT_ERR_SHAPE;
  if (!Wg || !Wu || !out) return CONVROT_ERR_NULL;
  if (!aligned(Wg, 4) || !aligned(Wu, 4) || !aligned(out, 4)) return CONVROT_ERR_ALIGN;
  const size_t words = static_cast<size_t>(2) * I * (row_bytes / 4);
  const int threads = 256;
  const size_t want = (words + threads - 1) / threads;
  const int blocks = static_cast<int>(std::min<size_t>(want, 148 * 16));
  interleave_rows_kernel<<<blocks, threads, 0, as_cuda(stream)>>>(
      static_cast<const uint32_t*>(Wg), static_cast<const uint32_t*>(Wu),
      static_cast<uint32_t*>(out), static_cast<size_t>(I), row_bytes / 4);
  return launch_status();
}

convrot_status convrot_fold_row_scales(float* s_row, const float* smooth, int n,
                                       convrot_stream_t stream) {
  if (n < 0) return CONVROT_ERR_SHAPE;
  if (n == 0) return CONVROT_OK;
  if (!s_row || !smooth) return CONVROT_ERR_NULL;
  if (!aligned(s_row, 4) || !aligned(smooth, 4)) return CONVROT_ERR_ALIGN;
  fold_row_scales_kernel<<<(n + 255) / 256, 256, 0, as_cuda(stream)>>>(s_row, smooth, n);
  return launch_status();
}

convrot_status convrot_int8_linear(const int8_t* Xq, const float* s_tok, const int8_t* Wq,
                                   const float* s_row, int M, int N, int K, void* Y,
                                   void* workspace, size_t workspace_bytes,
                                   convrot_stream_t stream) {
  return linear_common(Xq, s_tok, Wq, false, s_row, M, N, K, Y, workspace, workspace_bytes,
                       stream);
}

convrot_status convrot_w4a8_linear(const int8_t* Xq, const float* s_tok, const uint8_t* Wq4,
                                   const float* s_row, int M, int N, int K, void* Y,
                                   void* workspace, size_t workspace_bytes,
                                   convrot_stream_t stream) {
  return linear_common(Xq, s_tok, Wq4, true, s_row, M, N, K, Y, workspace, workspace_bytes,
                       stream);
}

// The raw-accumulator entry points run the same kernels and schedule with
// the int32 epilogue.
static convrot_status gemm_s32_common(const int8_t* Xq, const void* Wq, bool w4, int M, int N,
                                      int K, int32_t* acc, void* workspace,
                                      size_t workspace_bytes, convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, w4);
  if (sh != CONVROT_OK) return sh;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (!Xq || !Wq || !acc) return CONVROT_ERR_NULL;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(acc, 16)) return CONVROT_ERR_ALIGN;
  return run_gemm(Xq, Wq, w4, nullptr, nullptr, M, N, K, acc, EPI_S32, workspace, workspace_bytes,
                  as_cuda(stream));
}

convrot_status convrot_int8_gemm_s32(const int8_t* Xq, const int8_t* Wq, int M, int N, int K,
                                     int32_t* acc, void* workspace, size_t workspace_bytes,
                                     convrot_stream_t stream) {
  return gemm_s32_common(Xq, Wq, false, M, N, K, acc, workspace, workspace_bytes, stream);
}

convrot_status convrot_w4a8_gemm_s32(const int8_t* Xq, const uint8_t* Wq4, int M, int N, int K,
                                     int32_t* acc, void* workspace, size_t workspace_bytes,
                                     convrot_stream_t stream) {
  return gemm_s32_common(Xq, Wq4, true, M, N, K, acc, workspace, workspace_bytes, stream);
}

}  // extern "C"

// ===========================================================================
// Allocation-free variant of convrot_int8_linear.
//
// Some callers cannot allocate device memory at the point where they run a
// linear layer: plugins that do not own an allocator, runtimes whose device
// memory is planned once at start-up and must not grow afterwards, or code
// paths where an allocation would synchronise the device.  For them this entry
// point takes the GEMM's split-tile workspace from a fixed array that lives in
// the library itself instead of from the caller.
//
// The array is a file-scope __device__ array of kStaticWorkspaceBytes; every
// GPU that loads this library holds it until the process exits.  In host code
// the array's name is only a host-side stand-in, never a device address, so
// the device address is looked up with cudaGetSymbolAddress once per device
// (the first call on a device does that set-up; make that first call before
// any stream capture).  All calls on a device share the array and it keeps the
// last call's contents.  The split-tile counters and accumulators must start
// at zero: the set-up clears the whole array, every call that completes
// leaves what it used zero again (the unit that finalises a split tile
// re-zeroes its accumulator and counter), and after convrot_device_status has
// reported a device timeout (an aborted call may leave partial sums behind)
// the next call clears the array again before use.  Calls that overlap on
// the GPU (other streams, other threads) race on it.
// ===========================================================================
constexpr size_t kStaticWorkspaceBytes = static_cast<size_t>(24) << 20;  // 24 MiB per device
static __device__ __align__(256) uint8_t g_static_workspace[kStaticWorkspaceBytes];

namespace {
std::mutex g_static_ws_mu;
void* g_static_ws_ptr[64] = {nullptr};
// 1 + g_timeouts_reported at the array's last clear on each device (0: never)
unsigned g_static_ws_clean_at[64] = {0};

// Device address of g_static_workspace on `device` (the current device),
// cleared on `stream` if it has not been cleared since set-up or since the
// last reported device timeout.
convrot_status static_workspace(int device, cudaStream_t stream, void** out) {
  std::lock_guard<std::mutex> g(g_static_ws_mu);
  if (g_static_ws_ptr[device] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return CONVROT_ERR_CUDA;
    g_static_ws_ptr[device] = p;
  }
  const unsigned epoch = 1u + g_timeouts_reported.load(std::memory_order_relaxed);
  if (g_static_ws_clean_at[device] != epoch) {
    if (cudaMemsetAsync(g_static_ws_ptr[device], 0, kStaticWorkspaceBytes, stream) != cudaSuccess)
      return CONVROT_ERR_CUDA;
    g_static_ws_clean_at[device] = epoch;
  }
  *out = g_static_ws_ptr[device];
  return CONVROT_OK;
}
}  // namespace

extern "C" convrot_status convrot_int8_linear_noalloc(const int8_t* Xq, const float* s_tok,
                                                      const int8_t* Wq, const float* s_row,
                                                      int M, int N, int K, void* Y,
                                                      convrot_stream_t stream) {
  const convrot_status sh = check_gemm_shape(M, N, K, false);
  if (sh != CONVROT_OK) return sh;
  if (M == 0 || N == 0) return CONVROT_OK;
  if (!Xq || !s_tok || !Wq || !s_row || !Y) return CONVROT_ERR_NULL;
  if (!aligned(Xq, 16) || !aligned(Wq, 16) || !aligned(Y, 16) || !aligned(s_tok, 4) ||
      !aligned(s_row, 4))
    return CONVROT_ERR_ALIGN;
  const DeviceInfo d = current_device();
  if (d.device < 0 || d.sms <= 0) return CONVROT_ERR_CUDA;
  const size_t need = ws_bytes(plan_for(M, N, K, false, EPI_BF16, d));
  if (need > kStaticWorkspaceBytes) return CONVROT_ERR_WORKSPACE;  // shape too large for the array
  void* ws = nullptr;
  if (need > 0) {
    const convrot_status a = static_workspace(d.device, as_cuda(stream), &ws);
    if (a != CONVROT_OK) return a;
  }
  return run_gemm(Xq, Wq, false, s_tok, s_row, M, N, K, Y, EPI_BF16, ws,
                  need > 0 ? kStaticWorkspaceBytes : 0, as_cuda(stream));
}
