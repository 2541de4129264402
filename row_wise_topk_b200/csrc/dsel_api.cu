// C ABI of the row-wise TopK library: argument checks, planning, launches.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "../../include/dsel.h"
#include "dsel_kernels.cuh"
#include "dsel_plan.h"
#include "dsel_resident.cuh"
#include "dsel_slice.cuh"

namespace dsel {
namespace {

static_assert(sizeof(Ctl) <= kSharedFixedBytes, "control block outgrew its reservation");
static_assert(sizeof(SliceCtl) <= kSliceCtlBytes, "slice control block outgrew its reservation");

struct DevInfo {
  bool ready = false;
  int sms = 0;
  int smem_optin = 0;
  int major = 0;
  bool attrs_set[2][3] = {{false, false, false}, {false, false, false}};   // [dtype][shape]
  bool res_attrs_set[2] = {false, false};                                  // [dtype], resident kernel
  bool slice_attrs_set[4] = {false, false, false, false};                  // [dtype][shape], slice kernel
  int slice_cluster = 0;   // largest cluster the slice kernel launches with (16 when schedulable, else 8)
  bool stream_fit_ready = false;
  int32_t stream_fit[kSliceMaxCluster + 1] = {};   // streaming-kernel clusters of each size held at once
};

std::mutex g_mu;
DevInfo g_dev[64];

struct Workspace {
  int dev;
  void* stream;
  void* ptr;
  size_t bytes;
  uint64_t used;   // last use (a counter), for eviction
};
std::vector<Workspace> g_ws;
uint64_t g_ws_clock = 0;
constexpr int kMaxWorkspaces = 16;   // per device

int device_info(int dev, DevInfo** out) {
  if (dev < 0 || dev >= 64) return DSEL_ERR_DEVICE;
  DevInfo& d = g_dev[dev];
  if (!d.ready) {
    int minor = 0;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return DSEL_ERR_CUDA;
    if (d.major != 10 || minor != 0) return DSEL_ERR_DEVICE;
    d.ready = true;
  }
  *out = &d;
  return DSEL_OK;
}

// The split-row workspace of (device, stream), grown stream-ordered on that stream
// (cudaFreeAsync of the old buffer, cudaMallocAsync of the new one: the kernels
// that used the old buffer were launched on the same stream, so nothing waits on
// the host).  Never allocates inside a stream capture: the caller's first call of a
// split-row shape on a stream comes before capturing.  At most kMaxWorkspaces
// streams per device keep one; a further stream evicts the least recently used
// entry with cudaFree, which waits for the device.
int workspace(int dev, void* stream, size_t bytes, void** out) {
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  Workspace* w = nullptr;
  int on_dev = 0;
  Workspace* lru = nullptr;
  for (auto& e : g_ws) {
    if (e.dev != dev) continue;
    ++on_dev;
    if (e.stream == stream) w = &e;
    if (lru == nullptr || e.used < lru->used) lru = &e;
  }
  if (w != nullptr && w->bytes >= bytes) {
    w->used = ++g_ws_clock;
    *out = w->ptr;
    return DSEL_OK;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(cs, &cap) != cudaSuccess) return DSEL_ERR_CUDA;
  if (cap != cudaStreamCaptureStatusNone) return DSEL_ERR_WORKSPACE;
  if (w != nullptr) {   // grow in stream order
    if (cudaFreeAsync(w->ptr, cs) != cudaSuccess) return DSEL_ERR_CUDA;
    w->ptr = nullptr;
    w->bytes = 0;
    if (cudaMallocAsync(&w->ptr, bytes, cs) != cudaSuccess) {
      w->ptr = nullptr;
      return DSEL_ERR_WORKSPACE;
    }
    w->bytes = bytes;
    w->used = ++g_ws_clock;
    *out = w->ptr;
    return DSEL_OK;
  }
  if (on_dev >= kMaxWorkspaces && lru != nullptr) {   // evict: its stream may be gone
    if (cudaFree(lru->ptr) != cudaSuccess) return DSEL_ERR_CUDA;
    *lru = g_ws.back();
    g_ws.pop_back();
  }
  void* p = nullptr;
  if (cudaMallocAsync(&p, bytes, cs) != cudaSuccess) return DSEL_ERR_WORKSPACE;
  g_ws.push_back({dev, stream, p, bytes, ++g_ws_clock});
  *out = p;
  return DSEL_OK;
}

template <typename Kern>
cudaError_t launch_cluster(Kern kern, unsigned grid, int threads, int cluster, uint32_t smem, cudaStream_t st,
                           const KParams& kp) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(threads), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cluster);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the kernels set up shared memory, then wait
  // for the previous grid (griddepcontrol.wait) before touching global memory,
  // so their prologue overlaps the tail of the launch before them
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, kp);
}

template <int DT, int THREADS>
int run_shape(const KParams& base, const dsel_plan_t& pl, int64_t rows, cudaStream_t st, DevInfo* di) {
  auto sk = topk_stream_kernel<DT, THREADS>;
  auto mk = topk_merge_kernel<DT, kThreads>;
  constexpr int shp = THREADS == kThreads ? 0 : (THREADS == kThreadsMid ? 1 : 2);
  if (!di->attrs_set[DT][shp]) {
    if (cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(sk, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
        cudaFuncSetAttribute(mk, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(mk, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return DSEL_ERR_CUDA;
    di->attrs_set[DT][shp] = true;
  }
  const int eb = elem_bytes(DT);
  const SmemLayout sl = stream_layout(pl.stages, pl.block, pl.capacity, int64_t(base.k) + pl.b2, eb);
  KParams kp = base;
  kp.off_bars = sl.bars;
  kp.off_blk = sl.blk;
  kp.off_cb = sl.cb;
  kp.off_ci = sl.ci;
  kp.off_holes = sl.holes;
  kp.off_ctl = sl.ctl;
  kp.gather = int64_t(pl.cluster) * base.k <= pl.capacity;
  const int64_t grid = rows * pl.groups * pl.cluster;
  if (grid > 0x7FFFFFFF) return DSEL_ERR_ROWS;
  if (launch_cluster(sk, unsigned(grid), THREADS, pl.cluster, sl.total, st, kp) != cudaSuccess) return DSEL_ERR_CUDA;
  if (pl.groups > 1) {
    const SmemLayout ml = merge_layout(pl.capacity, int64_t(base.k) + pl.b2, eb);
    KParams mp = kp;
    mp.off_cb = ml.cb;
    mp.off_ci = ml.ci;
    mp.off_holes = ml.holes;
    mp.off_ctl = ml.ctl;
    const int mc = merge_cluster(pl, base.k);
    mp.gather = int64_t(mc) * base.k <= pl.capacity;
    if (launch_cluster(mk, unsigned(rows * mc), kThreads, mc, ml.total, st, mp) != cudaSuccess) return DSEL_ERR_CUDA;
  }
  return DSEL_OK;
}

template <int DT, int THREADS>
int run_slice_shape(const KParams& base, const dsel_plan_t& pl, int64_t rows, cudaStream_t st, DevInfo* di) {
  auto k1 = topk_slice_kernel<DT, THREADS, false>;
  auto kc = topk_slice_kernel<DT, THREADS, true>;
  const int slot = DT * 2 + (THREADS == kSliceThreadsLarge ? 1 : 0);
  if (!di->slice_attrs_set[slot]) {
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(kc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return DSEL_ERR_CUDA;
    di->slice_attrs_set[slot] = true;
  }
  const SliceLayout sl = slice_layout(pl.stages, pl.capacity, elem_bytes(DT));
  KParams kp = base;
  kp.off_tab = sl.tab;
  kp.off_bars = sl.bars;
  kp.off_cb = sl.cb;
  kp.off_ci = sl.ci;
  kp.off_cv = sl.cv;
  kp.off_hist = sl.hist;
  kp.off_ctl = sl.ctl;
  kp.vpt_cap = pl.stages;
  kp.capacity = pl.capacity;
  // geometry of rows of row_stride elements, so that those launches issue their
  // copies without computing it
  kp.sl_full = uint32_t((base.row_stride + pl.cluster - 1) / pl.cluster + 15) / 16u * 16u;
  kp.nch_full = int((int64_t(kp.sl_full) * elem_bytes(DT) + kSliceChunkBytes - 1) / kSliceChunkBytes);
  kp.pa_full = chunk_stride(uint32_t(kp.nch_full));
  kp.seg = pl.capacity / (THREADS / 32);   // each CTA's list, one segment per warp
  const int64_t grid = rows * pl.cluster;
  if (grid > 0x7FFFFFFF) return DSEL_ERR_ROWS;
  const cudaError_t e = pl.cluster > 1 ? launch_cluster(kc, unsigned(grid), THREADS, pl.cluster, sl.total, st, kp)
                                       : launch_cluster(k1, unsigned(grid), THREADS, 1, sl.total, st, kp);
  return e == cudaSuccess ? DSEL_OK : DSEL_ERR_CUDA;
}

template <int DT>
int run_slice(const KParams& base, const dsel_plan_t& pl, int64_t rows, cudaStream_t st, DevInfo* di) {
  if (pl.threads == kSliceThreadsLarge) return run_slice_shape<DT, kSliceThreadsLarge>(base, pl, rows, st, di);
  if (pl.threads == kSliceThreadsSmall) return run_slice_shape<DT, kSliceThreadsSmall>(base, pl, rows, st, di);
  return DSEL_ERR_DEVICE;
}

// Largest cluster the slice kernel may launch with on this device: 16 CTAs when
// such a cluster of the largest slices can be scheduled, else the portable 8.
int slice_cluster_limit(DevInfo* di) {
  if (di->slice_cluster != 0) return di->slice_cluster;
  auto kc = topk_slice_kernel<DSEL_F32, kSliceThreadsLarge, true>;
  int lim = kMaxCluster;
  if (cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) == cudaSuccess &&
      cudaFuncSetAttribute(kc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kSliceMaxCluster, 1, 1);
    cfg.blockDim = dim3(kSliceThreadsLarge, 1, 1);
    cfg.dynamicSmemBytes = uint32_t(di->smem_optin);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSliceMaxCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, kc, &cfg) == cudaSuccess && nclusters >= 1) lim = kSliceMaxCluster;
  }
  cudaGetLastError();   // a refused query leaves no sticky error
  di->slice_cluster = lim;
  return lim;
}

// For each cluster size: how many clusters of streaming CTAs the device holds at
// once, for the largest configuration (512 threads, all opt-in shared memory: one
// CTA per SM), so a lower bound for the others; 0 where the query fails.  A split
// row's plan keeps every cluster of its launch inside one wave with these counts.
const int32_t* stream_cluster_fit(DevInfo* di) {
  if (di->stream_fit_ready) return di->stream_fit;
  auto kc = topk_stream_kernel<DSEL_F32, kThreads>;
  di->stream_fit[1] = di->sms;
  if (cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) == cudaSuccess &&
      cudaFuncSetAttribute(kc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
    for (int c = 2; c <= kSliceMaxCluster; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(unsigned(c), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = uint32_t(di->smem_optin);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = unsigned(c);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, kc, &cfg) == cudaSuccess) di->stream_fit[c] = nc;
    }
  }
  cudaGetLastError();   // a refused query leaves no sticky error
  di->stream_fit_ready = true;
  return di->stream_fit;
}

// The plan of a call on this device (sorted_index DSEL_ORDER_VALUE also stands for
// the sampling call): the slice kernel up to its schedulable cluster size unless
// the order is by value; a split row over the streaming kernel's clusters and
// groups that the device holds in one wave.
int device_plan(DevInfo* di, int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                dsel_plan_t* pl) {
  return make_plan_ex(dtype, rows, row_stride, k, di->sms, di->smem_optin, kMaxCluster,
                      sorted_index == DSEL_ORDER_VALUE ? 0 : slice_cluster_limit(di), pl, stream_cluster_fit(di));
}

template <int DT>
int run_resident(const KParams& base, int64_t rows, cudaStream_t st, DevInfo* di) {
  auto rk = topk_resident_kernel<DT>;
  if (!di->res_attrs_set[DT]) {
    if (cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, di->smem_optin) != cudaSuccess ||
        cudaFuncSetAttribute(rk, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared) !=
            cudaSuccess)
      return DSEL_ERR_CUDA;
    di->res_attrs_set[DT] = true;
  }
  const ResLayout rl = resident_layout(base.row_stride, base.k, elem_bytes(DT));
  KParams kp = base;
  kp.off_bars = rl.bars;
  kp.off_hist = rl.hist;
  kp.off_cv = rl.el;
  kp.off_tab = rl.vl;
  kp.off_cb = rl.cb;
  kp.off_ci = rl.ci;
  kp.off_ctl = rl.ctl;
  kp.seg = rl.seg;
  if (rows > 0x7FFFFFFF) return DSEL_ERR_ROWS;
  if (launch_cluster(rk, unsigned(rows), kResThreads, 1, rl.total, st, kp) != cudaSuccess) return DSEL_ERR_CUDA;
  return DSEL_OK;
}

// The planner returns split-row plans (groups > 1) only with the 512-thread shape.
template <int DT>
int run(const KParams& base, const dsel_plan_t& pl, int64_t rows, cudaStream_t st, DevInfo* di) {
  if (pl.kernel == DSEL_KERNEL_RESIDENT) return run_resident<DT>(base, rows, st, di);
  if (pl.kernel == DSEL_KERNEL_SLICE) return run_slice<DT>(base, pl, rows, st, di);
  if (pl.threads == kThreadsShort) return run_shape<DT, kThreadsShort>(base, pl, rows, st, di);
  if (pl.threads == kThreadsMid) return run_shape<DT, kThreadsMid>(base, pl, rows, st, di);
  if (pl.threads == kThreads) return run_shape<DT, kThreads>(base, pl, rows, st, di);
  return DSEL_ERR_DEVICE;
}

}  // namespace
}  // namespace dsel

using namespace dsel;

extern "C" {

DSEL_API int64_t dsel_stride_requirement(int dtype) {
  return (dtype == DSEL_BF16 || dtype == DSEL_F32) ? kStrideReq : -1;
}

DSEL_API const char* dsel_status_string(int status) {
  switch (status) {
    case DSEL_OK: return "ok";
    case DSEL_ERR_DTYPE: return "dtype must be DSEL_BF16 or DSEL_F32";
    case DSEL_ERR_INDEX_DTYPE: return "index_dtype must be DSEL_I32 or DSEL_I64";
    case DSEL_ERR_K: return "k must be in [1, 4096]";
    case DSEL_ERR_ROWS: return "rows must be >= 0 (and the grid must fit)";
    case DSEL_ERR_STRIDE: return "row_stride must be a positive multiple of dsel_stride_requirement() and <= INT32_MAX";
    case DSEL_ERR_ALIGN: return "x must be 16-byte aligned";
    case DSEL_ERR_NULL: return "x and indices_out must not be NULL";
    case DSEL_ERR_VALUES: return "values_out must be non-NULL exactly when return_value is set";
    case DSEL_ERR_NAN_MODE: return "nan_mode must be DSEL_NAN_TRAP or DSEL_NAN_FLAG";
    case DSEL_ERR_ORDER: return "sorted_index must be 0, 1 or 2 (2, value order, needs float32 input)";
    case DSEL_ERR_DEVICE: return "the current device is not an sm_100 GPU";
    case DSEL_ERR_WORKSPACE:
      return "could not allocate the split-row workspace (a stream capture cannot allocate it: make the "
             "first call of this shape on the stream before capturing)";
    case DSEL_ERR_CUDA: return "a CUDA runtime call failed";
    case DSEL_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case DSEL_ERR_UNAVAILABLE: return "not available in this build";
    case DSEL_ERR_SCRATCH_LIMIT:
      return "the split-row scratch this call needs exceeds the static scratch of dsel_topk_noalloc "
             "(DSEL_NOALLOC_SCRATCH_BYTES per device)";
    default: return "unknown status";
  }
}

DSEL_API int dsel_debug_stats(uint64_t* host_out, int64_t n_ctas, void* stream) {
#ifdef DSEL_STATS
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (n_ctas <= -2) {   // select the CTA whose timeline later launches record
    const int cta = static_cast<int>(-n_ctas - 2);
    return cudaMemcpyToSymbolAsync(g_trace_cta, &cta, sizeof(int), 0, cudaMemcpyHostToDevice, cs) == cudaSuccess &&
                   cudaStreamSynchronize(cs) == cudaSuccess
               ? DSEL_OK
               : DSEL_ERR_CUDA;
  }
  if (host_out == nullptr) return DSEL_ERR_NULL;
  const int64_t n = n_ctas < kStatsCtas ? n_ctas : kStatsCtas;
  if (n_ctas == -1) {   // the per-round timeline instead (4 x 64 x 6 values)
    if (cudaMemcpyFromSymbolAsync(host_out, g_trace, sizeof(long long) * kTraceSize, 0,
                                  cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess)
      return DSEL_ERR_CUDA;
    return DSEL_OK;
  }
  if (cudaMemcpyFromSymbolAsync(host_out, g_stats, size_t(n) * kStatsFields * sizeof(uint64_t), 0,
                                cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess)
    return DSEL_ERR_CUDA;
  return DSEL_OK;
#else
  (void)host_out;
  (void)n_ctas;
  (void)stream;
  return DSEL_ERR_UNAVAILABLE;
#endif
}

DSEL_API const char* dsel_version(void) { return "dsel 0.1.0 (sm_100a)"; }

DSEL_API int dsel_plan(int dtype, int64_t rows, int64_t row_stride, int32_t k, int32_t num_sms,
                       int32_t smem_optin, int32_t max_cluster, dsel_plan_t* out) {
  return make_plan(dtype, rows, row_stride, k, num_sms, smem_optin, max_cluster, out);
}

DSEL_API int dsel_plan_for(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                           int32_t num_sms, int32_t smem_optin, int32_t max_cluster, dsel_plan_t* out) {
  if (sorted_index < DSEL_ORDER_NONE || sorted_index > DSEL_ORDER_VALUE) return DSEL_ERR_ORDER;
  return make_plan_ex(dtype, rows, row_stride, k, num_sms, smem_optin, max_cluster,
                      sorted_index == DSEL_ORDER_VALUE ? 0 : kSliceMaxCluster, out);
}

DSEL_API int dsel_plan_fit(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                           int32_t num_sms, int32_t smem_optin, const int32_t* cluster_fit, dsel_plan_t* out) {
  if (sorted_index < DSEL_ORDER_NONE || sorted_index > DSEL_ORDER_VALUE) return DSEL_ERR_ORDER;
  if (cluster_fit == nullptr || out == nullptr) return DSEL_ERR_NULL;
  return make_plan_ex(dtype, rows, row_stride, k, num_sms, smem_optin, kMaxCluster,
                      sorted_index == DSEL_ORDER_VALUE ? 0 : kSliceMaxCluster, out, cluster_fit);
}

DSEL_API int dsel_plan_device(int dtype, int64_t rows, int64_t row_stride, int32_t k, int sorted_index,
                              dsel_plan_t* out) {
  if (sorted_index < DSEL_ORDER_NONE || sorted_index > DSEL_ORDER_VALUE) return DSEL_ERR_ORDER;
  if (out == nullptr) return DSEL_ERR_NULL;
  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSEL_ERR_CUDA;
  DevInfo* di = nullptr;
  const int st = device_info(dev, &di);
  if (st != DSEL_OK) return st;
  return device_plan(di, dtype, rows, row_stride, k, sorted_index, out);
}

DSEL_API int dsel_topk(const void* x, int dtype, int64_t rows, int64_t row_stride, const int32_t* end,
                       int32_t k, int sorted_index, int return_value, int index_dtype, int nan_mode,
                       void* values_out, void* indices_out, void* stream) {
  int st = check_shape(dtype, rows, row_stride, k);
  if (st != DSEL_OK) return st;
  if (index_dtype != DSEL_I32 && index_dtype != DSEL_I64) return DSEL_ERR_INDEX_DTYPE;
  if (nan_mode != DSEL_NAN_TRAP && nan_mode != DSEL_NAN_FLAG) return DSEL_ERR_NAN_MODE;
  if (sorted_index < DSEL_ORDER_NONE || sorted_index > DSEL_ORDER_VALUE ||
      (sorted_index == DSEL_ORDER_VALUE && dtype != DSEL_F32))
    return DSEL_ERR_ORDER;
  if (return_value != 0 && return_value != 1) return DSEL_ERR_VALUES;
  if (rows == 0) return DSEL_OK;
  if (x == nullptr || indices_out == nullptr) return DSEL_ERR_NULL;
  if ((return_value != 0) != (values_out != nullptr)) return DSEL_ERR_VALUES;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0) return DSEL_ERR_ALIGN;

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSEL_ERR_CUDA;
  DevInfo* di = nullptr;
  st = device_info(dev, &di);
  if (st != DSEL_OK) return st;
  dsel_plan_t pl;
  st = device_plan(di, dtype, rows, row_stride, k, sorted_index, &pl);
  if (st != DSEL_OK) return st;

  KParams kp = {};
  kp.x = x;
  kp.end = end;
  kp.values_out = values_out;
  kp.indices_out = indices_out;
  kp.rows = rows;
  kp.row_stride = row_stride;
  kp.k = k;
  kp.groups = pl.groups;
  kp.b2 = pl.b2;
  kp.stages = pl.stages;
  kp.idx_bits = pl.idx_bits;
  kp.order = sorted_index;
  kp.return_value = return_value;
  kp.index_i64 = index_dtype == DSEL_I64;
  kp.nan_flag = nan_mode == DSEL_NAN_FLAG;
  kp.capacity = pl.capacity;
  if (pl.groups > 1) {
    void* ws = nullptr;
    st = workspace(dev, stream, size_t(pl.workspace_bytes), &ws);
    if (st != DSEL_OK) return st;
    kp.ws_pairs = static_cast<uint2*>(ws);
    kp.ws_meta = reinterpret_cast<int2*>(static_cast<char*>(ws) + rows * pl.groups * int64_t(k) * 8);
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dtype == DSEL_BF16 ? run<DSEL_BF16>(kp, pl, rows, cs, di) : run<DSEL_F32>(kp, pl, rows, cs, di);
}

DSEL_API int dsel_topk_sample(const void* x, int64_t rows, int64_t row_stride, const int32_t* end, int32_t k,
                              float temperature, float top_p, const float* u, int nan_mode, void* values_out,
                              void* indices_out, int64_t* token_out, float* prob_out, void* stream) {
  int st = check_shape(DSEL_F32, rows, row_stride, k);
  if (st != DSEL_OK) return st;
  if (nan_mode != DSEL_NAN_TRAP && nan_mode != DSEL_NAN_FLAG) return DSEL_ERR_NAN_MODE;
  if (rows == 0) return DSEL_OK;
  if (x == nullptr || u == nullptr || token_out == nullptr) return DSEL_ERR_NULL;
  if ((values_out == nullptr) != (indices_out == nullptr)) return DSEL_ERR_VALUES;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0) return DSEL_ERR_ALIGN;

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSEL_ERR_CUDA;
  DevInfo* di = nullptr;
  st = device_info(dev, &di);
  if (st != DSEL_OK) return st;
  dsel_plan_t pl;
  st = device_plan(di, DSEL_F32, rows, row_stride, k, DSEL_ORDER_VALUE, &pl);
  if (st != DSEL_OK) return st;

  KParams kp = {};
  kp.x = x;
  kp.end = end;
  kp.values_out = values_out;
  kp.indices_out = indices_out;
  kp.rows = rows;
  kp.row_stride = row_stride;
  kp.k = k;
  kp.groups = pl.groups;
  kp.b2 = pl.b2;
  kp.stages = pl.stages;
  kp.idx_bits = pl.idx_bits;
  kp.order = DSEL_ORDER_VALUE;
  kp.return_value = values_out != nullptr;
  kp.index_i64 = 1;
  kp.nan_flag = nan_mode == DSEL_NAN_FLAG;
  kp.capacity = pl.capacity;
  kp.u = u;
  kp.token_out = token_out;
  kp.prob_out = prob_out;
  kp.temperature = temperature;
  kp.top_p = top_p;
  if (pl.groups > 1) {
    void* ws = nullptr;
    st = workspace(dev, stream, size_t(pl.workspace_bytes), &ws);
    if (st != DSEL_OK) return st;
    kp.ws_pairs = static_cast<uint2*>(ws);
    kp.ws_meta = reinterpret_cast<int2*>(static_cast<char*>(ws) + rows * pl.groups * int64_t(k) * 8);
  }
  return run<DSEL_F32>(kp, pl, rows, static_cast<cudaStream_t>(stream), di);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of dsel_topk.
//
// Some callers cannot let a library allocate device memory: engines that own
// the whole device heap through their own allocator and a fixed memory budget,
// hosts that forbid side allocations by plug-ins, and latency-critical loops in
// which a cudaMalloc or cudaFree (either may synchronise the device) is not
// acceptable.  dsel_topk itself allocates only for split-row plans (one row
// spread over several thread-block clusters), whose clusters exchange partial
// results through a workspace.  dsel_topk_noalloc takes that workspace from
// the static array below instead; it never calls cudaMalloc, cudaFree or any
// allocating routine.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char dsel_noalloc_scratch[DSEL_NOALLOC_SCRATCH_BYTES];

namespace dsel {
namespace {
void* g_noalloc_scratch_addr[64];   // device address of dsel_noalloc_scratch, per device
}  // namespace
}  // namespace dsel

DSEL_API int dsel_topk_noalloc(const void* x, int dtype, int64_t rows, int64_t row_stride,
                               const int32_t* end, int32_t k, int sorted_index, int return_value,
                               int index_dtype, int nan_mode, void* values_out, void* indices_out,
                               void* stream) {
  int st = check_shape(dtype, rows, row_stride, k);
  if (st != DSEL_OK) return st;
  if (index_dtype != DSEL_I32 && index_dtype != DSEL_I64) return DSEL_ERR_INDEX_DTYPE;
  if (nan_mode != DSEL_NAN_TRAP && nan_mode != DSEL_NAN_FLAG) return DSEL_ERR_NAN_MODE;
  if (sorted_index < DSEL_ORDER_NONE || sorted_index > DSEL_ORDER_VALUE ||
      (sorted_index == DSEL_ORDER_VALUE && dtype != DSEL_F32))
    return DSEL_ERR_ORDER;
  if (return_value != 0 && return_value != 1) return DSEL_ERR_VALUES;
  if (rows == 0) return DSEL_OK;
  if (x == nullptr || indices_out == nullptr) return DSEL_ERR_NULL;
  if ((return_value != 0) != (values_out != nullptr)) return DSEL_ERR_VALUES;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0) return DSEL_ERR_ALIGN;

  std::lock_guard<std::mutex> lock(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSEL_ERR_CUDA;
  DevInfo* di = nullptr;
  st = device_info(dev, &di);
  if (st != DSEL_OK) return st;
  // Set-up, once per device, with that device current, on the first call whatever
  // its plan: host code only knows a stand-in for the array's name, so ask the
  // runtime for its device address.
  if (g_noalloc_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, dsel_noalloc_scratch) != cudaSuccess || ptr == nullptr) return DSEL_ERR_CUDA;
    g_noalloc_scratch_addr[dev] = ptr;
  }
  // the portable split of a long row (clusters of up to 8, the split dsel_plan
  // gives), not the one fitted to this device's cluster capacity: the scratch a
  // call needs, and so whether it is refused, is known on the host before any launch
  dsel_plan_t pl;
  st = make_plan_ex(dtype, rows, row_stride, k, di->sms, di->smem_optin, kMaxCluster,
                    sorted_index == DSEL_ORDER_VALUE ? 0 : slice_cluster_limit(di), &pl, nullptr);
  if (st != DSEL_OK) return st;

  KParams kp = {};
  kp.x = x;
  kp.end = end;
  kp.values_out = values_out;
  kp.indices_out = indices_out;
  kp.rows = rows;
  kp.row_stride = row_stride;
  kp.k = k;
  kp.groups = pl.groups;
  kp.b2 = pl.b2;
  kp.stages = pl.stages;
  kp.idx_bits = pl.idx_bits;
  kp.order = sorted_index;
  kp.return_value = return_value;
  kp.index_i64 = index_dtype == DSEL_I64;
  kp.nan_flag = nan_mode == DSEL_NAN_FLAG;
  kp.capacity = pl.capacity;
  if (pl.groups > 1) {
    if (pl.workspace_bytes > DSEL_NOALLOC_SCRATCH_BYTES) return DSEL_ERR_SCRATCH_LIMIT;
    // Nothing in the scratch has to start at zero: the merge launch reads only the
    // slots the streaming launch of the same call has just written.
    char* ws = static_cast<char*>(g_noalloc_scratch_addr[dev]);
    kp.ws_pairs = reinterpret_cast<uint2*>(ws);
    kp.ws_meta = reinterpret_cast<int2*>(ws + rows * pl.groups * int64_t(k) * 8);
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dtype == DSEL_BF16 ? run<DSEL_BF16>(kp, pl, rows, cs, di) : run<DSEL_F32>(kp, pl, rows, cs, di);
}

DSEL_API int dsel_device_status(int* status_out, void* stream) {
  if (status_out == nullptr) return DSEL_ERR_NULL;
  int v = 0, zero = 0;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess)
    return DSEL_ERR_CUDA;
  *status_out = v;
  return DSEL_OK;
}

}  // extern "C"
