// dllm_api.cu - the C ABI (include/dllm.h): argument validation, workspace layout, TMA
// tensor maps, launches on the caller's stream, device status word and kernel timing.
//
// All kernels are compiled in this one translation unit so that they share the device
// status word without relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "dllm.h"
#include "ptx.cuh"
#include "compact.cuh"
#include "lmhead.cuh"
#include "merge.cuh"
#include "select.cuh"
#include "arena.cuh"

#ifndef DLLM_GATHER_HOST_CTAS
#define DLLM_GATHER_HOST_CTAS 1   // gather CTAs per SM when the rows come from host memory
#endif

namespace dllm {

// An NVTX range around each entry point of the ABI, named after it, so that a timeline
// profiler groups the kernels of one library call (header-only NVTX v3: without a tool
// attached a range costs a null-pointer check).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Device-side error bits (kStatusTimeout, kStatusBounds, kStatusCapacity); one word per device.
__device__ int g_status;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  dllm_status err = DLLM_OK;
  int sms = 0;
  int pairs = 0;                // co-resident CTA pairs of the cta_group::2 GEMM
  int* status = nullptr;        // device address of g_status on this device
};

// GEMM variant: 2 = CTA pairs (cta_group::2, 256x256 tiles), 1 = single CTAs
// (cta_group::1, 128x256 tiles), both forced (test hook).  0 = default: chosen on the
// device from the masked count (lm::auto_variant): single CTAs for one m-tile of at most
// 128 rows (a pair would compute 128 empty rows), CTA pairs above (per SM a third fewer
// bytes staged from L2 per flop, which sets the clock under the 1 kW power cap).
std::atomic<int> g_gemm_variant{0};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

// Kernel-time accounting (dllm_prof_begin / dllm_prof_end).
struct Prof {
  bool on = false;
  std::vector<cudaEvent_t> ev;  // pairs: start, stop
  size_t used = 0;
  int gemm_launches = 0;
  std::atomic<int> kernel_launches{0};
};
Prof g_prof;

inline void count_launch(int n = 1) {
  if (g_prof.on) g_prof.kernel_launches += n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with programmatic stream serialization: the kernel may start while the previous
// kernel on the stream finishes; every kernel of this library waits for its predecessors
// (griddepcontrol.wait) before it touches global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-device setup, once: check the architecture, find g_status, raise the GEMM's shared
// memory limit, resolve the tensor-map encoder.
dllm_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DLLM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DLLM_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    st.err = DLLM_OK;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      st.err = DLLM_ERR_CUDA;
    } else if (prop.major != 10 || prop.minor != 0) {
      st.err = DLLM_ERR_DEVICE;
    } else {
      st.sms = prop.multiProcessorCount;
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) st.err = DLLM_ERR_CUDA;
      st.status = static_cast<int*>(p);
      const auto smem_attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
      if (st.err == DLLM_OK &&
          (cudaFuncSetAttribute(lm::lmhead_kernel<1, lm::kModeStats>, smem_attr, lm::Cfg<1>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_kernel<1, lm::kModeStatsExt>, smem_attr, lm::Cfg<1>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_kernel<1, lm::kModeDebugStore>, smem_attr, lm::Cfg<1>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_kernel<2, lm::kModeStats>, smem_attr, lm::Cfg<2>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_kernel<2, lm::kModeStatsExt>, smem_attr, lm::Cfg<2>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_kernel<2, lm::kModeDebugStore>, smem_attr, lm::Cfg<2>::SMEM_BYTES) ||
           cudaFuncSetAttribute(lm::lmhead_auto_kernel<lm::kModeStats>, smem_attr, lm::kAutoSmemBytes) ||
           cudaFuncSetAttribute(lm::lmhead_auto_kernel<lm::kModeStatsExt>, smem_attr, lm::kAutoSmemBytes) ||
           cudaFuncSetAttribute(lm::lmhead_auto_kernel<lm::kModeDebugStore>, smem_attr, lm::kAutoSmemBytes)))
        st.err = DLLM_ERR_CUDA;
      if (st.err == DLLM_OK) {
        // how many CTA pairs of the paired GEMM can be resident at once (a persistent grid
        // larger than that would serialise)
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (st.sms / 2), 1, 1);
        cfg.blockDim = dim3(lm::kThreads, 1, 1);
        cfg.dynamicSmemBytes = lm::Cfg<2>::SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, lm::lmhead_kernel<2, lm::kModeStats>, &cfg) != cudaSuccess)
          clusters = 0;
        st.pairs = clusters < lm::kMaxCtas / 2 ? clusters : lm::kMaxCtas / 2;
      }
      if (st.err == DLLM_OK && g_encode == nullptr) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          st.err = DLLM_ERR_CUDA;
        else
          g_encode = reinterpret_cast<EncodeTiledFn>(fn);
      }
    }
    st.ready = true;
  }
  if (st.err != DLLM_OK) return st.err;
  *out = &st;
  return DLLM_OK;
}

// Workspace layout for at most `rows` masked rows (rows = B*L: any mask):
// [tile counts | unit counters | gathered rows Hm | part_m | part_s | part_a | part_t | part_m2].
struct WsLayout {
  size_t tiles_off, ctr_off, hm_off, pm_off, ps_off, pa_off, pt_off, pm2_off, total;
  long long part_cap;
  long long rows;          // masked-row capacity: rows of Hm, and the GEMM's row bound
  int n_ctr;
};

WsLayout ws_layout(int B, int L, int d, int V, long long rows) {
  WsLayout w{};
  const long long n = static_cast<long long>(B) * L;
  const long long ntiles = (n + kCompactTile - 1) / kCompactTile;
  if (rows > n) rows = n;
  if (rows < 1) rows = 1;
  w.rows = rows;
  // partial entries: worst case over the masked count (up to `rows`), the largest number of
  // work holders and either GEMM variant; fewer masked rows never need more.
  const lm::Plan w1 = lm::Plan::make(static_cast<int>(rows), V, lm::kMaxCtas, lm::Cfg<1>::kGroupM,
                                     lm::Cfg<1>::BM);
  const lm::Plan w2 = lm::Plan::make(static_cast<int>(rows), V, lm::kMaxCtas / 2, lm::Cfg<2>::kGroupM,
                                     lm::Cfg<2>::BM);
  const long long cap1 = w1.ngroups * static_cast<long long>(lm::kMaxCtas) * lm::Cfg<1>::BM;
  const long long cap2 = w2.ngroups * static_cast<long long>(lm::kMaxCtas / 2) * lm::Cfg<2>::BM;
  long long cap = cap1 > cap2 ? cap1 : cap2;
  // a masked count that fits one group may use remainder holders: (P + R) slots of G m-tiles,
  // with P * G + R <= holders and R < G <= gmax, so fewer than (holders + gmax^2) m-tile rows
  const long long r1 = (static_cast<long long>(lm::kMaxCtas) + lm::Cfg<1>::kGroupM * lm::Cfg<1>::kGroupM) *
                       lm::Cfg<1>::BM;
  const long long r2 = (static_cast<long long>(lm::kMaxCtas / 2) + lm::Cfg<2>::kGroupM * lm::Cfg<2>::kGroupM) *
                       lm::Cfg<2>::BM;
  if (r1 > cap) cap = r1;
  if (r2 > cap) cap = r2;
  if (cap < 1) cap = 1;
  w.part_cap = cap;
  // one counter per (m-tile, CTA of the pair): ceil(rows / 128) + 2 covers both variants;
  // then one progress word per work holder (the pair body's pacing), zeroed with them
  w.n_ctr = static_cast<int>((rows + 127) / 128 + 2 + lm::kMaxCtas);
  size_t off = 0;
  w.tiles_off = off; off = round_up(off + sizeof(int) * ntiles, 256);
  w.ctr_off = off;   off = round_up(off + sizeof(int) * static_cast<size_t>(w.n_ctr), 256);
  w.hm_off = off;    off = round_up(off + static_cast<size_t>(rows) * d * 2, 256);
  w.pm_off = off;    off = round_up(off + sizeof(float) * cap, 256);
  w.ps_off = off;    off = round_up(off + sizeof(float) * cap, 256);
  w.pa_off = off;    off = round_up(off + sizeof(int) * cap, 256);
  w.pt_off = off;    off = round_up(off + sizeof(float) * cap, 256);
  w.pm2_off = off;   off = round_up(off + sizeof(float) * cap, 256);
  w.total = off;
  return w;
}

// The layout a workspace of ws_bytes can hold: all B*L rows when it is at least the full
// layout, else the largest masked-row capacity whose layout fits (the total grows with the
// capacity), or rows = 0 when not even one row fits.
WsLayout ws_layout_for(int B, int L, int d, int V, size_t ws_bytes) {
  const long long n = static_cast<long long>(B) * L;
  WsLayout full = ws_layout(B, L, d, V, n);
  if (ws_bytes >= full.total) return full;
  WsLayout one = ws_layout(B, L, d, V, 1);
  if (ws_bytes < one.total) {
    one.rows = 0;
    return one;
  }
  long long lo = 1, hi = n;                   // layout(lo) fits, layout(hi) does not
  while (hi - lo > 1) {
    const long long mid = lo + (hi - lo) / 2;
    if (ws_layout(B, L, d, V, mid).total <= ws_bytes) lo = mid;
    else hi = mid;
  }
  return ws_layout(B, L, d, V, lo);
}

// A step input (H or M) may live in device memory or in page-locked host memory that the
// device can read over PCIe (zero-copy: only the bytes the kernels touch cross the bus,
// e.g. just the masked rows of H).  Resolves the pointer the kernels use; pageable host
// memory is rejected (DLLM_ERR_MEMORY) because the device cannot read it.
dllm_status resolve_input(const void* p, const void** dev, bool* on_host = nullptr) {
  cudaPointerAttributes at{};
  if (on_host) *on_host = false;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();                       // clear the sticky-free error of the query
    return DLLM_ERR_MEMORY;
  }
  if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) {
    *dev = p;
    return DLLM_OK;
  }
  if (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr) {
    *dev = at.devicePointer;
    if (on_host) *on_host = true;
    return aligned16(*dev) ? DLLM_OK : DLLM_ERR_ALIGN;
  }
  return DLLM_ERR_MEMORY;
}

bool shapes_ok(int B, int L) {
  return B >= 1 && L >= 1 && static_cast<long long>(B) * L < (1ll << 31);
}

dllm_status launch_compact(const uint8_t* M, int B, int L, const int* win_lo, const int* win_hi,
                           int* row_idx, int* seq_off, int* count, int* tiles, int* status,
                           cudaStream_t s) {
  const long long n = static_cast<long long>(B) * L;
  const unsigned ntiles = static_cast<unsigned>((n + kCompactTile - 1) / kCompactTile);
  // a single tile needs no per-tile counts: its offset is 0
  if (ntiles > 1) {
    if (launch_pdl(compact_count_kernel, dim3(ntiles), dim3(kCompactThreads), 0, s, M, n, L, win_lo,
                   win_hi, tiles) != cudaSuccess)
      return DLLM_ERR_CUDA;
    count_launch();
  }
  const bool offsets = ntiles > static_cast<unsigned>(kCompactDirectTiles);
  if (offsets) {
    if (launch_pdl(compact_scan_kernel, dim3(1), dim3(kScanThreads), 0, s, tiles,
                   static_cast<int>(ntiles)) != cudaSuccess)
      return DLLM_ERR_CUDA;
    count_launch();
  }
  if (launch_pdl(compact_scatter_kernel, dim3(ntiles), dim3(kCompactThreads), 0, s, M, B, L, win_lo,
                 win_hi, (const int*)tiles, offsets, row_idx, seq_off, count, status) != cudaSuccess)
    return DLLM_ERR_CUDA;
  count_launch();
  return DLLM_OK;
}

dllm_status make_tmap(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(lm::BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DLLM_OK : DLLM_ERR_CUDA;
}

struct LogitsArgs {
  const uint16_t* H; const uint8_t* M; const uint16_t* W;
  int B, L, d, V;
  const int* win_lo; const int* win_hi;          // rows restricted to windows, or both NULL
  uint32_t stats; float* entropy; float* margin;
  int* tok; float* conf; float* lse; float* dbg;
  int* row_idx; int* seq_off; int* count;
  void* ws; size_t ws_bytes; cudaStream_t s;
  lm::Partials raw = {nullptr, nullptr, nullptr, nullptr, nullptr};   // vocabulary-shard mode
  int a_offset = 0;
};

dllm_status validate_logits(const LogitsArgs& a, bool debug, bool prepared = false) {
  if ((!prepared && (!a.H || !a.M || !a.row_idx || !a.seq_off)) || !a.W || !a.count || !a.ws)
    return DLLM_ERR_NULL;
  const bool shard = a.raw.m != nullptr;
  if (shard) {
    if (!a.raw.s || !a.raw.a) return DLLM_ERR_NULL;
    if ((a.stats != 0) != (a.raw.t != nullptr) || (a.stats != 0) != (a.raw.m2 != nullptr))
      return DLLM_ERR_NULL;
    if (a.a_offset < 0 || static_cast<long long>(a.a_offset) + a.V >= (1ll << 31)) return DLLM_ERR_SHAPE;
  } else if (!debug && (!a.tok || !a.conf || !a.lse)) {
    return DLLM_ERR_NULL;
  }
  if (debug && !a.dbg) return DLLM_ERR_NULL;
  if ((a.win_lo == nullptr) != (a.win_hi == nullptr)) return DLLM_ERR_NULL;
  if ((a.stats & ~(DLLM_STAT_ENTROPY | DLLM_STAT_MARGIN)) != 0) return DLLM_ERR_SHAPE;
  if (!shard && ((a.stats & DLLM_STAT_ENTROPY) != 0) != (a.entropy != nullptr)) return DLLM_ERR_NULL;
  if (!shard && ((a.stats & DLLM_STAT_MARGIN) != 0) != (a.margin != nullptr)) return DLLM_ERR_NULL;
  if (!shapes_ok(a.B, a.L) || a.V < 1 || a.d < DLLM_D_MULTIPLE || a.d % DLLM_D_MULTIPLE != 0)
    return DLLM_ERR_SHAPE;
  const void* ptrs[] = {a.H, a.M, a.W, a.row_idx, a.seq_off, a.count, a.ws, a.tok, a.conf, a.lse,
                        a.dbg, a.entropy, a.margin, a.win_lo, a.win_hi, a.raw.m, a.raw.s,
                        a.raw.a, a.raw.t, a.raw.m2};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  if (ws_layout_for(a.B, a.L, a.d, a.V, a.ws_bytes).rows < 1) return DLLM_ERR_WORKSPACE;
  return DLLM_OK;
}

// a1 + gather: compaction of the mask (in the windows, if any) and the copy of the masked
// rows of H into the workspace's dense Hm; H and M may be page-locked host memory.
dllm_status prepare_rows(const LogitsArgs& a, const DeviceState& ds, const WsLayout& w) {
  const void* Hd = nullptr;
  const void* Md = nullptr;
  bool host_rows = false;
  dllm_status st = resolve_input(a.H, &Hd, &host_rows);
  if (st != DLLM_OK) return st;
  if ((st = resolve_input(a.M, &Md)) != DLLM_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  int* tiles = reinterpret_cast<int*>(ws + w.tiles_off);
  uint16_t* Hm = reinterpret_cast<uint16_t*>(ws + w.hm_off);
  int* ctr = reinterpret_cast<int*>(ws + w.ctr_off);
  const long long n = static_cast<long long>(a.B) * a.L;
  if ((st = launch_compact(static_cast<const uint8_t*>(Md), a.B, a.L, a.win_lo, a.win_hi, a.row_idx,
                           a.seq_off, a.count, tiles, ds.status, a.s)) != DLLM_OK)
    return st;
  // Rows read from device memory: 4 CTAs per SM.  Rows read over the bus from page-locked
  // host memory: the bus, not the SMs, bounds the copy (about 20 ms for cfg3's 0.97 GB), and
  // one CTA per SM keeps enough reads in flight while leaving each SM room for the next
  // GEMM's persistent CTA, which this staging overlaps.
  if (launch_pdl(gather_rows_kernel, dim3(ds.sms * (host_rows ? DLLM_GATHER_HOST_CTAS : 4)),
                 dim3(kGatherThreads), 0, a.s,
                 static_cast<const uint16_t*>(Hd), (const int*)a.row_idx, (const int*)a.count, n,
                 w.rows, a.d, Hm, ctr, w.n_ctr, ds.status) != cudaSuccess)
    return DLLM_ERR_CUDA;
  count_launch();
  return DLLM_OK;
}

// skip_prepare: the rows were prepared by an earlier dllm_prepare_rows into the same
// workspace (H and M are then not read).
dllm_status run_logits(const LogitsArgs& a, bool debug, bool skip_prepare = false) {
  dllm_status st = validate_logits(a, debug, skip_prepare);
  if (st != DLLM_OK) return st;
  DeviceState* ds = nullptr;
  if ((st = device_state(&ds)) != DLLM_OK) return st;
  const WsLayout w = ws_layout_for(a.B, a.L, a.d, a.V, a.ws_bytes);
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  uint16_t* Hm = reinterpret_cast<uint16_t*>(ws + w.hm_off);
  float* pm = reinterpret_cast<float*>(ws + w.pm_off);
  float* ps = reinterpret_cast<float*>(ws + w.ps_off);
  int* pa = reinterpret_cast<int*>(ws + w.pa_off);
  float* pt = reinterpret_cast<float*>(ws + w.pt_off);
  float* pm2 = reinterpret_cast<float*>(ws + w.pm2_off);
  int* ctr = reinterpret_cast<int*>(ws + w.ctr_off);
  const lm::Partials part{pm, ps, pa, pt, pm2};
  const lm::Outputs outs{a.tok, a.conf, a.lse, a.entropy, a.margin, a.raw, a.a_offset};
  const long long n = w.rows;        // masked-row capacity of this workspace (B*L when full)

  // GEMM variant: 0 = chosen on the device from the masked count (lm::auto_variant, one
  // launch in clusters of two CTAs), 1 / 2 = forced single CTAs / CTA pairs (test hook)
  int cg = g_gemm_variant.load();
  if (ds->pairs < 1) cg = 1;                                   // no CTA pairs on this device
  const int single_holders = cg == 0 ? 2 * ds->pairs : (ds->sms < lm::kMaxCtas ? ds->sms : lm::kMaxCtas);
  for (int v = 1; v <= 2; ++v) {
    if (cg != 0 && cg != v) continue;
    // largest partial footprint over every masked count this variant may run: all
    // positions masked, or any count that fits one group of m-tiles (remainder holders)
    const int holders = v == 2 ? ds->pairs : single_holders;
    const int bm = v == 2 ? lm::Cfg<2>::BM : lm::Cfg<1>::BM;
    const int gmax = v == 2 ? lm::Cfg<2>::kGroupM : lm::Cfg<1>::kGroupM;
    long long need = lm::Plan::make(static_cast<int>(n), a.V, holders, gmax, bm).part_entries();
    const long long mt = (n + bm - 1) / bm;
    for (long long m = 1; m <= mt && m <= gmax; ++m) {
      const long long c = m * bm < n ? m * bm : n;
      const long long e = lm::Plan::make(static_cast<int>(c), a.V, holders, gmax, bm).part_entries();
      if (e > need) need = e;
    }
    if (need > w.part_cap) return DLLM_ERR_WORKSPACE;                  // cannot happen on B200
  }

  if (!skip_prepare) {
    if ((st = prepare_rows(a, *ds, w)) != DLLM_OK) return st;
  }

  // W is staged 256 rows per CTA by single CTAs and 128 rows per CTA by pairs
  CUtensorMap tmA, tmB1, tmB2;
  if (make_tmap(&tmA, Hm, static_cast<uint64_t>(n), a.d, 128) != DLLM_OK) return DLLM_ERR_CUDA;
  if (cg != 2 && make_tmap(&tmB1, a.W, static_cast<uint64_t>(a.V), a.d, lm::BN) != DLLM_OK)
    return DLLM_ERR_CUDA;
  if (cg != 1 && make_tmap(&tmB2, a.W, static_cast<uint64_t>(a.V), a.d, lm::BN / 2) != DLLM_OK)
    return DLLM_ERR_CUDA;

  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (g_prof.on) {
    if (g_prof.used + 2 > g_prof.ev.size()) {
      for (int i = 0; i < 64; ++i) {
        cudaEvent_t e;
        if (cudaEventCreate(&e) != cudaSuccess) return DLLM_ERR_CUDA;
        g_prof.ev.push_back(e);
      }
    }
    e0 = g_prof.ev[g_prof.used];
    e1 = g_prof.ev[g_prof.used + 1];
    g_prof.used += 2;
    cudaEventRecord(e0, a.s);
  }
  {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    cfg.blockDim = dim3(lm::kThreads, 1, 1);
    cfg.stream = a.s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cg != 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = 2;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
      cfg.gridDim = dim3(2 * ds->pairs, 1, 1);
      cfg.dynamicSmemBytes = cg == 0 ? lm::kAutoSmemBytes : lm::Cfg<2>::SMEM_BYTES;
    } else {
      cfg.gridDim = dim3(single_holders, 1, 1);
      cfg.dynamicSmemBytes = lm::Cfg<1>::SMEM_BYTES;
    }
    const int n_cap = static_cast<int>(n);
    float* dbg = debug ? a.dbg : nullptr;
    const int mode = debug ? lm::kModeDebugStore : (a.stats ? lm::kModeStatsExt : lm::kModeStats);
    const int* cnt = a.count;
    cudaError_t e;
#define DLLM_LAUNCH_GEMM(CGV, MODE, TMB)                                                      \
  cudaLaunchKernelEx(&cfg, lm::lmhead_kernel<CGV, MODE>, tmA, TMB, cnt, n_cap, a.V, a.d,      \
                     lm::Cfg<CGV>::kGroupM, part, w.part_cap, ctr, outs, dbg, ds->status)
#define DLLM_LAUNCH_AUTO(MODE)                                                                 \
  cudaLaunchKernelEx(&cfg, lm::lmhead_auto_kernel<MODE>, tmA, tmB1, tmB2, cnt, n_cap, a.V, a.d, \
                     part, w.part_cap, ctr, outs, dbg, ds->status)
    if (cg == 0)
      e = mode == lm::kModeStats ? DLLM_LAUNCH_AUTO(lm::kModeStats)
        : mode == lm::kModeStatsExt ? DLLM_LAUNCH_AUTO(lm::kModeStatsExt)
        : DLLM_LAUNCH_AUTO(lm::kModeDebugStore);
    else if (cg == 2)
      e = mode == lm::kModeStats ? DLLM_LAUNCH_GEMM(2, lm::kModeStats, tmB2)
        : mode == lm::kModeStatsExt ? DLLM_LAUNCH_GEMM(2, lm::kModeStatsExt, tmB2)
        : DLLM_LAUNCH_GEMM(2, lm::kModeDebugStore, tmB2);
    else
      e = mode == lm::kModeStats ? DLLM_LAUNCH_GEMM(1, lm::kModeStats, tmB1)
        : mode == lm::kModeStatsExt ? DLLM_LAUNCH_GEMM(1, lm::kModeStatsExt, tmB1)
        : DLLM_LAUNCH_GEMM(1, lm::kModeDebugStore, tmB1);
#undef DLLM_LAUNCH_GEMM
#undef DLLM_LAUNCH_AUTO
    if (e != cudaSuccess) return DLLM_ERR_CUDA;
  }
  count_launch();
  if (g_prof.on) {
    cudaEventRecord(e1, a.s);
    g_prof.gemm_launches++;
  }
  return cudaPeekAtLastError() == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}

}  // namespace
}  // namespace dllm

// ---------------------------------------------------------------------------------------
// Allocation-free compaction (dllm_mask_compact_noalloc): the per-tile counts live in this
// fixed static device array instead of the caller's workspace.  In host code the array's
// name is only a host-side stand-in; its device address comes from cudaGetSymbolAddress,
// looked up once per device.
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) int g_noalloc_tile_counts[DLLM_NOALLOC_MAX_TILES];

static_assert(static_cast<long long>(DLLM_NOALLOC_MAX_TILES) * dllm::kCompactTile ==
                  DLLM_NOALLOC_MAX_POSITIONS,
              "scratch limit and compaction tile size disagree");

namespace {
struct NoAllocScratch {
  bool ready = false;
  dllm_status err = DLLM_OK;
  int* tiles = nullptr;           // device address of g_noalloc_tile_counts on this device
};
std::mutex g_noalloc_mu;
NoAllocScratch g_noalloc[64];

dllm_status noalloc_scratch(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DLLM_ERR_CUDA;
  if (dev < 0 || dev >= 64) return DLLM_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocScratch& st = g_noalloc[dev];
  if (!st.ready) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_tile_counts);
    st.err = (e == cudaSuccess && p != nullptr) ? DLLM_OK : DLLM_ERR_CUDA;
    st.tiles = static_cast<int*>(p);
    st.ready = true;
  }
  if (st.err != DLLM_OK) return st.err;
  *out = st.tiles;
  return DLLM_OK;
}
}  // namespace

using namespace dllm;

extern "C" {

dllm_status dllm_mask_compact_noalloc(const uint8_t* M, int32_t B, int32_t L, int32_t* row_idx,
                                      int32_t* seq_off, int32_t* count, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_mask_compact_noalloc");
  if (!M || !row_idx || !seq_off || !count) return DLLM_ERR_NULL;
  if (!shapes_ok(B, L)) return DLLM_ERR_SHAPE;
  if (static_cast<long long>(B) * L > DLLM_NOALLOC_MAX_POSITIONS) return DLLM_ERR_SCRATCH;
  if (!aligned16(M) || !aligned16(row_idx) || !aligned16(seq_off) || !aligned16(count))
    return DLLM_ERR_ALIGN;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  int* tiles = nullptr;
  if ((st = noalloc_scratch(&tiles)) != DLLM_OK) return st;
  return launch_compact(M, B, L, nullptr, nullptr, row_idx, seq_off, count, tiles, ds->status,
                        static_cast<cudaStream_t>(stream));
}

int32_t dllm_version(void) { return 10200; }

const char* dllm_status_string(dllm_status s) {
  switch (s) {
    case DLLM_OK: return "ok";
    case DLLM_ERR_NULL: return "a required pointer is NULL";
    case DLLM_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case DLLM_ERR_SHAPE: return "shape out of range";
    case DLLM_ERR_WORKSPACE: return "workspace too small";
    case DLLM_ERR_CUDA: return "CUDA error";
    case DLLM_ERR_TIMEOUT: return "a device-side wait timed out";
    case DLLM_ERR_DEVICE: return "device is not an sm_100 GPU";
    case DLLM_ERR_BOUNDS: return "a device-side bound check failed";
    case DLLM_ERR_SCRATCH: return "B*L exceeds the fixed scratch of the allocation-free entry point";
    case DLLM_ERR_MEMORY: return "an input is neither device memory nor page-locked host memory";
    case DLLM_ERR_CAPACITY: return "more masked rows than the workspace was sized for";
    default: return "unknown status";
  }
}

size_t dllm_workspace_bytes(int32_t B, int32_t L, int32_t d, int32_t V) {
  if (!shapes_ok(B, L) || V < 1 || d < DLLM_D_MULTIPLE || d % DLLM_D_MULTIPLE != 0) return 0;
  return ws_layout(B, L, d, V, static_cast<long long>(B) * L).total;
}

size_t dllm_workspace_bytes_rows(int32_t B, int32_t L, int32_t d, int32_t V, int64_t max_rows) {
  if (!shapes_ok(B, L) || V < 1 || d < DLLM_D_MULTIPLE || d % DLLM_D_MULTIPLE != 0 || max_rows < 1)
    return 0;
  return ws_layout(B, L, d, V, max_rows).total;
}

int64_t dllm_workspace_rows(int32_t B, int32_t L, int32_t d, int32_t V, size_t ws_bytes) {
  if (!shapes_ok(B, L) || V < 1 || d < DLLM_D_MULTIPLE || d % DLLM_D_MULTIPLE != 0) return 0;
  return ws_layout_for(B, L, d, V, ws_bytes).rows;
}

dllm_status dllm_mask_compact_window(const uint8_t* M, int32_t B, int32_t L, const int32_t* win_lo,
                                     const int32_t* win_hi, int32_t* row_idx, int32_t* seq_off,
                                     int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_mask_compact_window");
  if (!M || !row_idx || !seq_off || !count || !ws) return DLLM_ERR_NULL;
  if ((win_lo == nullptr) != (win_hi == nullptr)) return DLLM_ERR_NULL;
  if (!shapes_ok(B, L)) return DLLM_ERR_SHAPE;
  if (!aligned16(M) || !aligned16(row_idx) || !aligned16(seq_off) || !aligned16(count) || !aligned16(ws))
    return DLLM_ERR_ALIGN;
  if ((win_lo && !aligned16(win_lo)) || (win_hi && !aligned16(win_hi))) return DLLM_ERR_ALIGN;
  const long long n = static_cast<long long>(B) * L;
  const size_t need = sizeof(int) * static_cast<size_t>((n + kCompactTile - 1) / kCompactTile);
  if (ws_bytes < need) return DLLM_ERR_WORKSPACE;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  return launch_compact(M, B, L, win_lo, win_hi, row_idx, seq_off, count, static_cast<int*>(ws),
                        ds->status, static_cast<cudaStream_t>(stream));
}

dllm_status dllm_mask_compact(const uint8_t* M, int32_t B, int32_t L, int32_t* row_idx,
                              int32_t* seq_off, int32_t* count, void* ws, size_t ws_bytes,
                              void* stream) {
  return dllm_mask_compact_window(M, B, L, nullptr, nullptr, row_idx, seq_off, count, ws, ws_bytes,
                                  stream);
}

dllm_status dllm_masked_logits(const uint16_t* H, const uint8_t* M, const uint16_t* W, int32_t B,
                               int32_t L, int32_t d, int32_t V, int32_t* tok, float* conf,
                               float* lse, int32_t* row_idx, int32_t* seq_off, int32_t* count,
                               void* ws, size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_masked_logits");
  LogitsArgs a{H, M, W, B, L, d, V, nullptr, nullptr, 0u, nullptr, nullptr, tok, conf, lse, nullptr,
               row_idx, seq_off, count, ws, ws_bytes, static_cast<cudaStream_t>(stream)};
  return run_logits(a, false);
}

dllm_status dllm_masked_logits_ex(const uint16_t* H, const uint8_t* M, const uint16_t* W, int32_t B,
                                  int32_t L, int32_t d, int32_t V, uint32_t stats, int32_t* tok,
                                  float* conf, float* lse, float* entropy, float* margin,
                                  int32_t* row_idx, int32_t* seq_off, int32_t* count, void* ws,
                                  size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_masked_logits_ex");
  LogitsArgs a{H, M, W, B, L, d, V, nullptr, nullptr, stats, entropy, margin, tok, conf, lse, nullptr,
               row_idx, seq_off, count, ws, ws_bytes, static_cast<cudaStream_t>(stream)};
  return run_logits(a, false);
}

dllm_status dllm_masked_logits_window(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                      int32_t B, int32_t L, int32_t d, int32_t V,
                                      const int32_t* win_lo, const int32_t* win_hi, uint32_t stats,
                                      int32_t* tok, float* conf, float* lse, float* entropy,
                                      float* margin, int32_t* row_idx, int32_t* seq_off,
                                      int32_t* count, void* ws, size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_masked_logits_window");
  if (!win_lo || !win_hi) return DLLM_ERR_NULL;
  LogitsArgs a{H, M, W, B, L, d, V, win_lo, win_hi, stats, entropy, margin, tok, conf, lse, nullptr,
               row_idx, seq_off, count, ws, ws_bytes, static_cast<cudaStream_t>(stream)};
  return run_logits(a, false);
}

dllm_status dllm_masked_partials(const uint16_t* H, const uint8_t* M, const uint16_t* W_shard,
                                 int32_t B, int32_t L, int32_t d, int32_t V_shard, int32_t v_offset,
                                 const int32_t* win_lo, const int32_t* win_hi, uint32_t stats,
                                 float* part_m, float* part_s, int32_t* part_a, float* part_t,
                                 float* part_m2, int32_t* row_idx, int32_t* seq_off, int32_t* count,
                                 void* ws, size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_masked_partials");
  if (!part_m) return DLLM_ERR_NULL;
  LogitsArgs a{H, M, W_shard, B, L, d, V_shard, win_lo, win_hi, stats, nullptr, nullptr, nullptr,
               nullptr, nullptr, nullptr, row_idx, seq_off, count, ws, ws_bytes,
               static_cast<cudaStream_t>(stream)};
  a.raw = lm::Partials{part_m, part_s, part_a, part_t, part_m2};
  a.a_offset = v_offset;
  return run_logits(a, false);
}

dllm_status dllm_lse_merge(const float* part_m, const float* part_s, const int32_t* part_a,
                           const float* part_t, const float* part_m2, int64_t split_stride,
                           int32_t n_split, const int32_t* count, int32_t n_cap, uint32_t stats,
                           int32_t* tok, float* conf, float* lse, float* entropy, float* margin,
                           void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_lse_merge");
  if (!part_m || !part_s || !part_a || !count || !tok || !conf || !lse) return DLLM_ERR_NULL;
  if ((stats & ~(DLLM_STAT_ENTROPY | DLLM_STAT_MARGIN)) != 0) return DLLM_ERR_SHAPE;
  if ((stats != 0) != (part_t != nullptr) || (stats != 0) != (part_m2 != nullptr)) return DLLM_ERR_NULL;
  if (((stats & DLLM_STAT_ENTROPY) != 0) != (entropy != nullptr)) return DLLM_ERR_NULL;
  if (((stats & DLLM_STAT_MARGIN) != 0) != (margin != nullptr)) return DLLM_ERR_NULL;
  if (n_split < 1 || n_cap < 1 || split_stride < n_cap) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {part_m, part_s, part_a, part_t, part_m2, count, tok, conf, lse, entropy, margin};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  int blocks = (n_cap + kMergeThreads - 1) / kMergeThreads;
  if (blocks > ds->sms * 8) blocks = ds->sms * 8;
  const lm::Partials part{const_cast<float*>(part_m), const_cast<float*>(part_s),
                          const_cast<int*>(part_a), const_cast<float*>(part_t),
                          const_cast<float*>(part_m2)};
  const lm::Outputs outs{tok, conf, lse, entropy, margin, lm::Partials{nullptr, nullptr, nullptr, nullptr, nullptr}, 0};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = stats != 0
      ? launch_pdl(lse_merge_kernel<true>, dim3(blocks), dim3(kMergeThreads), 0, s, part,
                   static_cast<long long>(split_stride), static_cast<int>(n_split), count,
                   static_cast<int>(n_cap), outs)
      : launch_pdl(lse_merge_kernel<false>, dim3(blocks), dim3(kMergeThreads), 0, s, part,
                   static_cast<long long>(split_stride), static_cast<int>(n_split), count,
                   static_cast<int>(n_cap), outs);
  if (e != cudaSuccess) return DLLM_ERR_CUDA;
  count_launch();
  return DLLM_OK;
}

dllm_status dllm_prepare_rows(const uint16_t* H, const uint8_t* M, int32_t B, int32_t L, int32_t d,
                              int32_t V, const int32_t* win_lo, const int32_t* win_hi,
                              int32_t* row_idx, int32_t* seq_off, int32_t* count, void* ws,
                              size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_prepare_rows");
  if (!H || !M || !row_idx || !seq_off || !count || !ws) return DLLM_ERR_NULL;
  if ((win_lo == nullptr) != (win_hi == nullptr)) return DLLM_ERR_NULL;
  if (!shapes_ok(B, L) || V < 1 || d < DLLM_D_MULTIPLE || d % DLLM_D_MULTIPLE != 0) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {H, M, row_idx, seq_off, count, ws, win_lo, win_hi};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  const WsLayout w = ws_layout_for(B, L, d, V, ws_bytes);
  if (w.rows < 1) return DLLM_ERR_WORKSPACE;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  LogitsArgs a{H, M, nullptr, B, L, d, V, win_lo, win_hi, 0u, nullptr, nullptr, nullptr, nullptr, nullptr,
               nullptr, row_idx, seq_off, count, ws, ws_bytes, static_cast<cudaStream_t>(stream)};
  return prepare_rows(a, *ds, w);
}

dllm_status dllm_masked_logits_prepared(const uint16_t* W, int32_t B, int32_t L, int32_t d, int32_t V,
                                        uint32_t stats, int32_t* tok, float* conf, float* lse,
                                        float* entropy, float* margin, const int32_t* count,
                                        void* ws, size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_masked_logits_prepared");
  LogitsArgs a{nullptr, nullptr, W, B, L, d, V, nullptr, nullptr, stats, entropy, margin, tok, conf,
               lse, nullptr, nullptr, nullptr, const_cast<int32_t*>(count), ws, ws_bytes,
               static_cast<cudaStream_t>(stream)};
  return run_logits(a, false, true);
}

dllm_status dllm_debug_lmhead_logits(const uint16_t* H, const uint8_t* M, const uint16_t* W,
                                     int32_t B, int32_t L, int32_t d, int32_t V, float* logits_out,
                                     int32_t* row_idx, int32_t* seq_off, int32_t* count, void* ws,
                                     size_t ws_bytes, void* stream) {
  LogitsArgs a{H, M, W, B, L, d, V, nullptr, nullptr, 0u, nullptr, nullptr, nullptr, nullptr, nullptr,
               logits_out, row_idx, seq_off, count, ws, ws_bytes, static_cast<cudaStream_t>(stream)};
  return run_logits(a, true);
}

}  // extern "C"

namespace {
dllm_status run_select(const float* conf, const int32_t* row_idx, const int32_t* seq_off,
                       int32_t B, int32_t L, int32_t k, bool use_threshold, float threshold,
                       int32_t min_sel, bool ascending, const int32_t* win_lo, const int32_t* win_hi,
                       const int32_t* tok, int32_t* idx, int32_t* n_sel, int32_t* tok_sel,
                       float* conf_sel, void* stream) {
  if (!conf || !row_idx || !seq_off || !idx || !n_sel) return DLLM_ERR_NULL;
  if (use_threshold && (min_sel < 0 || threshold != threshold)) return DLLM_ERR_SHAPE;
  if ((win_lo == nullptr) != (win_hi == nullptr)) return DLLM_ERR_NULL;
  if (tok_sel && !tok) return DLLM_ERR_NULL;
  if (!shapes_ok(B, L) || k < 1 || k > DLLM_MAX_K) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {conf, row_idx, seq_off, win_lo, win_hi, tok, idx, n_sel, tok_sel, conf_sel};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  if (launch_pdl(select_unmask_kernel, dim3(B), dim3(kSelThreads), 0, static_cast<cudaStream_t>(stream),
                 conf, row_idx, seq_off, B * L, L, k, use_threshold, threshold, min_sel, ascending,
                 win_lo, win_hi, tok, idx, n_sel, tok_sel, conf_sel) != cudaSuccess)
    return DLLM_ERR_CUDA;
  count_launch();
  return DLLM_OK;
}
}  // namespace

extern "C" {

dllm_status dllm_select_unmask(const float* conf, const int32_t* row_idx, const int32_t* seq_off,
                               int32_t B, int32_t L, int32_t k, const int32_t* win_lo,
                               const int32_t* win_hi, const int32_t* tok, int32_t* idx,
                               int32_t* n_sel, int32_t* tok_sel, float* conf_sel, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_select_unmask");
  return run_select(conf, row_idx, seq_off, B, L, k, false, 0.f, 0, false, win_lo, win_hi, tok, idx,
                    n_sel, tok_sel, conf_sel, stream);
}

dllm_status dllm_select_unmask_ex(const float* score, const int32_t* row_idx, const int32_t* seq_off,
                                  int32_t B, int32_t L, int32_t k, float threshold, int32_t min_sel,
                                  int32_t ascending, const int32_t* win_lo, const int32_t* win_hi,
                                  const int32_t* tok, int32_t* idx, int32_t* n_sel, int32_t* tok_sel,
                                  float* score_sel, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_select_unmask_ex");
  if (ascending != 0 && ascending != 1) return DLLM_ERR_SHAPE;
  return run_select(score, row_idx, seq_off, B, L, k, true, threshold, min_sel, ascending != 0,
                    win_lo, win_hi, tok, idx, n_sel, tok_sel, score_sel, stream);
}

dllm_status dllm_decode_step(const uint16_t* H, const uint8_t* M, const uint16_t* W, int32_t B,
                             int32_t L, int32_t d, int32_t V, int32_t k, const int32_t* win_lo,
                             const int32_t* win_hi, int32_t* tok, float* conf, float* lse,
                             int32_t* row_idx, int32_t* seq_off, int32_t* count, int32_t* idx,
                             int32_t* n_sel, int32_t* tok_sel, float* conf_sel, void* ws,
                             size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_decode_step");
  // validate the selection's own arguments first so that nothing is launched on error
  if (!idx || !n_sel) return DLLM_ERR_NULL;
  if ((win_lo == nullptr) != (win_hi == nullptr)) return DLLM_ERR_NULL;
  if (k < 1 || k > DLLM_MAX_K) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {win_lo, win_hi, idx, n_sel, tok_sel, conf_sel};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  dllm_status st = dllm_masked_logits(H, M, W, B, L, d, V, tok, conf, lse, row_idx, seq_off, count,
                                      ws, ws_bytes, stream);
  if (st != DLLM_OK) return st;
  return dllm_select_unmask(conf, row_idx, seq_off, B, L, k, win_lo, win_hi, tok, idx, n_sel,
                            tok_sel, conf_sel, stream);
}

dllm_status dllm_decode_block_step(const uint16_t* H, const uint8_t* M, const uint16_t* W, int32_t B,
                                   int32_t L, int32_t d, int32_t V, int32_t k, const int32_t* win_lo,
                                   const int32_t* win_hi, int32_t* tok, float* conf, float* lse,
                                   int32_t* row_idx, int32_t* seq_off, int32_t* count, int32_t* idx,
                                   int32_t* n_sel, int32_t* tok_sel, float* conf_sel, void* ws,
                                   size_t ws_bytes, void* stream) {
  const dllm::NvtxRange nvtx_range("dllm_decode_block_step");
  if (!idx || !n_sel || !win_lo || !win_hi) return DLLM_ERR_NULL;
  if (k < 1 || k > DLLM_MAX_K) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {idx, n_sel, tok_sel, conf_sel};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return DLLM_ERR_ALIGN;
  dllm_status st = dllm_masked_logits_window(H, M, W, B, L, d, V, win_lo, win_hi, 0u, tok, conf, lse,
                                             nullptr, nullptr, row_idx, seq_off, count, ws, ws_bytes,
                                             stream);
  if (st != DLLM_OK) return st;
  // every compacted row already lies in its window: no window test is needed in the selection
  return dllm_select_unmask(conf, row_idx, seq_off, B, L, k, nullptr, nullptr, tok, idx, n_sel,
                            tok_sel, conf_sel, stream);
}

dllm_status dllm_debug_lse_merge(const float* part_m, const float* part_s, const int32_t* part_a,
                                 int32_t n_rows, int32_t n_split, int32_t* tok, float* conf,
                                 float* lse, void* stream) {
  if (!part_m || !part_s || !part_a || !tok || !conf || !lse) return DLLM_ERR_NULL;
  if (n_rows < 1 || n_split < 1) return DLLM_ERR_SHAPE;
  const void* ptrs[] = {part_m, part_s, part_a, tok, conf, lse};
  for (const void* p : ptrs)
    if (!aligned16(p)) return DLLM_ERR_ALIGN;
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  int blocks = (n_rows + kMergeThreads - 1) / kMergeThreads;
  if (blocks > ds->sms * 8) blocks = ds->sms * 8;
  lse_merge_plain_kernel<<<blocks, kMergeThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      part_m, part_s, part_a, n_rows, n_split, tok, conf, lse);
  count_launch();
  return cudaPeekAtLastError() == cudaSuccess ? DLLM_OK : DLLM_ERR_CUDA;
}

dllm_status dllm_debug_set_gemm_variant(int32_t cta_group) {
  if (cta_group != 0 && cta_group != 1 && cta_group != 2) return DLLM_ERR_SHAPE;
  g_gemm_variant.store(cta_group);
  return DLLM_OK;
}

dllm_status dllm_get_status(void* stream) {
  DeviceState* ds = nullptr;
  dllm_status st = device_state(&ds);
  if (st != DLLM_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DLLM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return DLLM_ERR_CUDA;
  const int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return DLLM_ERR_CUDA;
  if (v & kStatusTimeout) return DLLM_ERR_TIMEOUT;
  if (v & kStatusBounds) return DLLM_ERR_BOUNDS;
  if (v & kStatusCapacity) return DLLM_ERR_CAPACITY;
  return DLLM_OK;
}

dllm_status dllm_prof_begin(void) {
  g_prof.on = true;
  g_prof.used = 0;
  g_prof.gemm_launches = 0;
  g_prof.kernel_launches = 0;
  return DLLM_OK;
}

dllm_status dllm_prof_end(double* gemm_ms, int32_t* gemm_launches, int32_t* kernel_launches) {
  double total = 0.0;
  dllm_status st = DLLM_OK;
  for (size_t i = 0; i + 1 < g_prof.used; i += 2) {
    if (cudaEventSynchronize(g_prof.ev[i + 1]) != cudaSuccess) { st = DLLM_ERR_CUDA; break; }
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof.ev[i], g_prof.ev[i + 1]) != cudaSuccess) { st = DLLM_ERR_CUDA; break; }
    total += ms;
  }
  if (gemm_ms) *gemm_ms = total;
  if (gemm_launches) *gemm_launches = g_prof.gemm_launches;
  if (kernel_launches) *kernel_launches = g_prof.kernel_launches;
  g_prof.on = false;
  g_prof.used = 0;
  return st;
}

}  // extern "C"
