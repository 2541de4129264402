// Row-wise TopK kernels: the streaming filter (one pass over every row) and the
// merge used when one row is split over several clusters.
#pragma once

#include "dsel_device.cuh"
#include "dsel_plan.h"

namespace dsel {

// Everything a launch needs; shared-memory offsets come from the host planner.
struct KParams {
  const void* x;
  const int32_t* end;
  void* values_out;
  void* indices_out;
  uint2* ws_pairs;          // [rows][groups][k] {index, bits}, split-row plans only
  int2* ws_meta;            // [rows][groups]    {count, nan}
  int64_t rows;
  int64_t row_stride;
  int32_t k;
  int32_t groups;
  int32_t b2;
  int32_t stages;
  int32_t idx_bits;
  int32_t order;            // DSEL_ORDER_*
  int32_t return_value;
  int32_t index_i64;
  int32_t nan_flag;         // 1: DSEL_NAN_FLAG, 0: DSEL_NAN_TRAP
  int32_t gather;           // final phase gathers the cluster's partial results on rank 0
  uint32_t off_bars, off_blk, off_cb, off_ci, off_holes, off_ctl;
};

#ifdef DSEL_STATS
constexpr int kStatsCtas = 8192;
constexpr int kStatsFields = 16;
__device__ unsigned long long g_stats[kStatsCtas * kStatsFields];
// per-round timeline of CTA 0 for warps 0, 5, 10, 15 (lane 0): [warp][round][event]
constexpr int kTraceRounds = 64;
constexpr int kTraceEvents = 8;
__device__ long long g_trace[4 * kTraceRounds * kTraceEvents];
#endif

constexpr int kSeedBits = 11;                 // round-0 histogram: 2048 bins
constexpr int kSeedBins = 1 << kSeedBits;

// ---------------------------------------------------------------------------
// Output writers (all threads of one CTA).
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__device__ void write_rows_out(const KParams& p, int64_t row, int off, int m,
                               const typename Elem<DT>::bits_t* cb, const uint32_t* ci) {
  using bits_t = typename Elem<DT>::bits_t;
  const int64_t base = row * p.k + off;
  for (int i = threadIdx.x; i < m; i += THREADS) {
    const uint32_t idx = ci[i];
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = static_cast<int64_t>(idx);
    else static_cast<int32_t*>(p.indices_out)[base + i] = static_cast<int32_t>(idx);
    if (p.return_value) static_cast<bits_t*>(p.values_out)[base + i] = cb[i];
  }
}

template <int DT, int THREADS>
__device__ void write_ws(const KParams& p, int64_t row, int g, int off, int m,
                         const typename Elem<DT>::bits_t* cb, const uint32_t* ci) {
  uint2* dst = p.ws_pairs + (row * p.groups + g) * static_cast<int64_t>(p.k) + off;
  for (int i = threadIdx.x; i < m; i += THREADS) dst[i] = make_uint2(ci[i], static_cast<uint32_t>(cb[i]));
}

template <int DT, int THREADS>
__device__ void write_sentinel_row(const KParams& p, int64_t row, int32_t code) {
  using bits_t = typename Elem<DT>::bits_t;
  const int64_t base = row * p.k;
  for (int i = threadIdx.x; i < p.k; i += THREADS) {
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = code;
    else static_cast<int32_t*>(p.indices_out)[base + i] = code;
    if (p.return_value) static_cast<bits_t*>(p.values_out)[base + i] = static_cast<bits_t>(Elem<DT>::kQNaN);
  }
}

// Rows no longer than k: every entry, in index order, then padding.  No NaN check.
template <int DT, int THREADS>
__device__ void write_short_row(const KParams& p, int64_t row, int64_t n) {
  using bits_t = typename Elem<DT>::bits_t;
  const bits_t* xr = static_cast<const bits_t*>(p.x) + row * p.row_stride;
  const int64_t base = row * p.k;
  for (int i = threadIdx.x; i < p.k; i += THREADS) {
    const bool in = i < n;
    const int32_t idx = in ? i : DSEL_IDX_PAD;
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = idx;
    else static_cast<int32_t*>(p.indices_out)[base + i] = idx;
    if (p.return_value)
      static_cast<bits_t*>(p.values_out)[base + i] = in ? xr[i] : static_cast<bits_t>(Elem<DT>::kNegInf);
  }
}

// Valid length of a row, with the end[] rules; *bad is set for an invalid end in
// flag mode (trap mode clamps instead).
__device__ __forceinline__ int64_t row_length(const KParams& p, int64_t row, bool* bad) {
  *bad = false;
  if (p.end == nullptr) return p.row_stride;
  int64_t e = p.end[row];
  if (e < 0 || e > p.row_stride) {
    *bad = p.nan_flag != 0;
    e = e < 0 ? 0 : p.row_stride;
  }
  return e;
}

// Largest V over the CTA, from per-thread maxima (barrier inside).
template <int THREADS>
__device__ __forceinline__ uint64_t cta_vmax(uint64_t vmax, Ctl& ctl) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  vmax = warp_max_u64(vmax);
  if (lane == 0) ctl.wv[warp] = vmax;
  __syncthreads();
  const uint64_t m = lane < NW ? ctl.wv[lane] : 0ull;
  return warp_max_u64(m);
}

// Exact selection of the `need` best candidates of this CTA's buffer (all in
// [vlo, vhi]), moved to its front.  Returns the kept count.
template <int DT, int THREADS>
__device__ int local_select(typename Elem<DT>::bits_t* cb, uint32_t* ci, int cnt, int need, int idx_bits,
                            uint64_t vlo, uint64_t vhi, Ctl& ctl, uint32_t* holes,
                            cg::cluster_group& cluster) {
  if (cnt <= need) return cnt;
  const SelResult sel =
      radix_select<DT, THREADS, false>(cb, ci, cnt, need, 0, idx_bits, vlo, vhi, ctl, cluster);
  return holes_compact<DT, THREADS>(cb, ci, cnt, sel.kept, sel, idx_bits, ctl, holes);
}

template <int DT, int THREADS>
__device__ __forceinline__ void sort_kept(typename Elem<DT>::bits_t* cb, uint32_t* ci, int m, int sort_mode) {
  if (sort_mode == 1) bitonic_sort<DT, THREADS, false>(cb, ci, m);
  else if (sort_mode == 2) bitonic_sort<DT, THREADS, true>(cb, ci, m);
}

// Writes the m kept entries (output row, or this group's workspace slot).
template <int DT, int THREADS>
__device__ __forceinline__ void emit(const KParams& p, int64_t row, int g, bool to_workspace, int off, int m,
                                     int total, bool write_meta, const typename Elem<DT>::bits_t* cb,
                                     const uint32_t* ci) {
  if (to_workspace) {
    write_ws<DT, THREADS>(p, row, g, off, m, cb, ci);
    if (write_meta && threadIdx.x == 0) p.ws_meta[row * p.groups + g] = make_int2(total, 0);
  } else {
    write_rows_out<DT, THREADS>(p, row, off, m, cb, ci);
  }
}

template <int DT, int THREADS>
__device__ __forceinline__ void emit_nan(const KParams& p, int64_t row, int g, bool to_workspace) {
  if (to_workspace) {
    if (threadIdx.x == 0) p.ws_meta[row * p.groups + g] = make_int2(0, 1);
  } else {
    write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_NAN);
  }
}

// ---------------------------------------------------------------------------
// Final phase, shared by the streaming and merge kernels.  The cluster's CTAs
// together hold a superset of the row's (or row part's) best entries; exactly
// min(k, total) of them are kept, optionally sorted, and written to the output
// (or, for a split row, to the workspace).
//   * one CTA: local exact select;
//   * gather (cluster * k fits one buffer): each CTA keeps its own best k, rank 0
//     copies the peers' lists over distributed shared memory and selects again;
//   * otherwise: a cluster-wide radix select on summed histograms, each CTA
//     writing its share (slices are in index order, so per-CTA index sorts
//     concatenate into a sorted row); value order gathers on rank 0 at the end.
//   sort_mode 0: none, 1: ascending index, 2: value descending.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__device__ __noinline__ void finalize(const KParams& p, int64_t row, int g, typename Elem<DT>::bits_t* cb,
                         uint32_t* ci, uint32_t* holes, Ctl& ctl, cg::cluster_group& cluster,
                         int cnt, bool nan_local, uint64_t vlo, uint64_t vmax_thread,
                         bool to_workspace, int sort_mode) {
  using bits_t = typename Elem<DT>::bits_t;
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t idx_mask = mask_bits(p.idx_bits);

  if (nan_local) ctl.nan_found = 1;
  const uint64_t vhi = cta_vmax<THREADS>(vmax_thread, ctl);   // barrier: nan_found visible
  const bool nan_cta = ctl.nan_found != 0;

  if (C == 1) {
    if (nan_cta) {
      emit_nan<DT, THREADS>(p, row, g, to_workspace);
      return;
    }
    const int m = local_select<DT, THREADS>(cb, ci, cnt, p.k, p.idx_bits, vlo, vhi, ctl, holes, cluster);
    sort_kept<DT, THREADS>(cb, ci, m, sort_mode);
    emit<DT, THREADS>(p, row, g, to_workspace, 0, m, m, true, cb, ci);
    return;
  }

  if (p.gather) {
    const int m =
        nan_cta ? 0 : local_select<DT, THREADS>(cb, ci, cnt, p.k, p.idx_bits, vlo, vhi, ctl, holes, cluster);
    if (tid == 0) {
      ctl.x_kept = m;
      ctl.x_nan = nan_cta ? 1 : 0;
    }
    cluster.sync();
    if (crank != 0) return;
    int nn = lane < C ? cluster.map_shared_rank(&ctl, lane)->x_nan : 0;
    if (__any_sync(0xffffffffu, nn != 0)) {
      emit_nan<DT, THREADS>(p, row, g, to_workspace);
      return;
    }
    // rank 0 appends the peers' lists after its own
    int off = m;
    uint64_t vmx = 0;
    for (int i = tid; i < m; i += THREADS) {
      const uint64_t v = make_v<DT>(cb[i], ci[i], p.idx_bits, idx_mask);
      vmx = v > vmx ? v : vmx;
    }
    for (int r = 1; r < C; ++r) {
      const int mr = cluster.map_shared_rank(&ctl, r)->x_kept;
      const bits_t* rcb = cluster.map_shared_rank(cb, r);
      const uint32_t* rci = cluster.map_shared_rank(ci, r);
      for (int i = tid; i < mr; i += THREADS) {
        const bits_t b = rcb[i];
        const uint32_t ix = rci[i];
        cb[off + i] = b;
        ci[off + i] = ix;
        const uint64_t v = make_v<DT>(b, ix, p.idx_bits, idx_mask);
        vmx = v > vmx ? v : vmx;
      }
      off += mr;
    }
    const uint64_t ghi = cta_vmax<THREADS>(vmx, ctl);   // barrier: the gathered list is complete
    const int mm = local_select<DT, THREADS>(cb, ci, off, p.k, p.idx_bits, 0ull, ghi, ctl, holes, cluster);
    sort_kept<DT, THREADS>(cb, ci, mm, sort_mode);
    emit<DT, THREADS>(p, row, g, to_workspace, 0, mm, mm, true, cb, ci);
    return;
  }

  // ---- distributed select over the cluster ----
  for (int i = tid; i < 3 * kBins; i += THREADS) (&ctl.hist[0][0])[i] = 0;
  if (tid == 0) {
    ctl.hb = 0;
    ctl.x_cnt = cnt;
    ctl.x_nan = nan_cta ? 1 : 0;
    ctl.x_vlo = cnt > 0 ? vlo : ~0ull;
    ctl.x_vhi = cnt > 0 ? vhi : 0ull;
  }
  cluster.sync();
  int tot = 0, nn = 0;
  unsigned long long lo = ~0ull, hi = 0ull;
  if (lane < C) {
    Ctl* pc = cluster.map_shared_rank(&ctl, lane);
    tot = pc->x_cnt;
    nn = pc->x_nan;
    lo = pc->x_vlo;
    hi = pc->x_vhi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
    nn |= __shfl_xor_sync(0xffffffffu, nn, o);
    const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o);
    const unsigned long long h2 = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = l2 < lo ? l2 : lo;
    hi = h2 > hi ? h2 : hi;
  }
  if (nn) {
    if (crank == 0) emit_nan<DT, THREADS>(p, row, g, to_workspace);
    return;
  }
  const int need = min(p.k, tot);
  int m = cnt;
  if (tot > need) {
    const SelResult sel =
        radix_select<DT, THREADS, true>(cb, ci, cnt, need, 0, p.idx_bits, lo, hi, ctl, cluster);
    m = holes_compact<DT, THREADS>(cb, ci, cnt, -1, sel, p.idx_bits, ctl, holes);
  }
  if (sort_mode == 1) bitonic_sort<DT, THREADS, false>(cb, ci, m);
  if (tid == 0) ctl.x_kept = m;
  cluster.sync();
  if (sort_mode == 2) {   // gather the winners on rank 0 and sort them by value
    if (crank == 0) {
      int off = m;
      for (int r = 1; r < C; ++r) {
        const int mr = cluster.map_shared_rank(&ctl, r)->x_kept;
        const bits_t* rcb = cluster.map_shared_rank(cb, r);
        const uint32_t* rci = cluster.map_shared_rank(ci, r);
        for (int i = tid; i < mr; i += THREADS) {
          cb[off + i] = rcb[i];
          ci[off + i] = rci[i];
        }
        off += mr;
      }
      __syncthreads();
      bitonic_sort<DT, THREADS, true>(cb, ci, off);
      emit<DT, THREADS>(p, row, g, to_workspace, 0, off, off, true, cb, ci);
    }
    return;
  }
  int off = lane < crank ? cluster.map_shared_rank(&ctl, lane)->x_kept : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
  emit<DT, THREADS>(p, row, g, to_workspace, off, m, need, crank == 0, cb, ci);
}

// ---------------------------------------------------------------------------
// Round-0 threshold seed (cold path, kept out of the per-round loop).  Builds a
// 2048-bin histogram of the round's keys over the bits where they differ and
// returns the lower edge of the bin holding the k-th largest: at least k of the
// round's elements (hence of the slice) are >= it, so it is a valid starting T.
// voff[v]: byte offset in the ring of this thread's vector v (~0u: none).
// ---------------------------------------------------------------------------
struct SeedOut {
  unsigned long long t;
  uint64_t vlo;
  bool ok;
};

template <int DT, int THREADS, int VPT>
__device__ __noinline__ SeedOut seed_threshold(const unsigned char* ring, const uint32_t (&voff)[VPT],
                                               const uint32_t (&eidx)[VPT], uint32_t uhi, int k, int idx_bits,
                                               Ctl& ctl, int* seed_hist) {
  using E = Elem<DT>;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint4 val[VPT];
#pragma unroll
  for (int v = 0; v < VPT; ++v)
    val[v] = voff[v] != 0xFFFFFFFFu ? *reinterpret_cast<const uint4*>(ring + voff[v]) : make_uint4(0u, 0u, 0u, 0u);
  int nvalid = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
#pragma unroll
    for (int e = 0; e < PV; ++e) {
      const uint32_t b = vec_elem<DT>(val[v], e);
      if (voff[v] != 0xFFFFFFFFu && eidx[v] + e < uhi && !E::is_nan(b)) {
        const uint32_t kk = E::key(b);
        kmin = min(kmin, kk);
        kmax = max(kmax, kk);
        ++nvalid;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    ctl.wc[1][warp] = nvalid;
    ctl.wv[warp] = (static_cast<unsigned long long>(kmax) << 32) | kmin;
  }
  __syncthreads();
  int tot_valid;
  warp_prefix_of<NW>(ctl.wc[1], warp, lane, tot_valid);
  uint32_t gmin = 0xFFFFFFFFu, gmax = 0u;
  if (lane < NW) {
    gmin = static_cast<uint32_t>(ctl.wv[lane]);
    gmax = static_cast<uint32_t>(ctl.wv[lane] >> 32);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
    gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
  }
  SeedOut out{0ull, 0ull, false};
  if (tot_valid <= k || gmin == gmax) return out;   // uniform
  // window: the kSeedBits bits below the leading bits shared by gmin, gmax
  const int top = 32 - __clz(gmin ^ gmax);           // low bits in which keys differ
  const int ws = top > kSeedBits ? top - kSeedBits : 0;
  const uint32_t kbase = gmin & ~mask_bits(top);
#pragma unroll
  for (int v = 0; v < VPT; ++v) {
#pragma unroll
    for (int e = 0; e < PV; ++e) {
      const uint32_t b = vec_elem<DT>(val[v], e);
      if (voff[v] != 0xFFFFFFFFu && eidx[v] + e < uhi && !E::is_nan(b))
        atomicAdd(&seed_hist[(E::key(b) - kbase) >> ws], 1);
    }
  }
  __syncthreads();
  // the bin holding the k-th largest: per-warp slice sums, then the slice
  constexpr int SLICE = kSeedBins / NW;
  constexpr int PER_LANE = SLICE / 32;
  const int sbase = kSeedBins - (warp + 1) * SLICE;  // warp 0 sums the top slice
  int sl = 0;
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) sl += seed_hist[sbase + lane * PER_LANE + j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
  if (lane == 0) ctl.wm[warp] = sl;
  __syncthreads();
  const int c = lane < NW ? ctl.wm[lane] : 0;
  const int incl = warp_incl_scan(c, lane);
  const bool mine = (incl - c) < k && k <= incl;
  const int slc = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
  const int need = k - __shfl_sync(0xffffffffu, incl - c, slc);
  const int b0 = kSeedBins - (slc + 1) * SLICE;
  int cc[PER_LANE];
  int sm = 0;
#pragma unroll
  for (int j = 0; j < PER_LANE; ++j) {   // bins of that slice from its top
    cc[j] = seed_hist[b0 + SLICE - 1 - (lane * PER_LANE + j)];
    sm += cc[j];
  }
  const int inc2 = warp_incl_scan(sm, lane);
  const bool mine2 = (inc2 - sm) < need && need <= inc2;
  int bin = 0;
  if (mine2) {
    int acc = inc2 - sm;
    bool done = false;
#pragma unroll
    for (int j = 0; j < PER_LANE; ++j) {
      if (!done && acc + cc[j] >= need) {
        bin = b0 + SLICE - 1 - (lane * PER_LANE + j);
        done = true;
      }
      acc += cc[j];
    }
  }
  bin = __shfl_sync(0xffffffffu, bin, __ffs(__ballot_sync(0xffffffffu, mine2)) - 1);
  // every key >= the bin's lower edge passes, and at least k elements do
  const uint32_t key_t = kbase + (static_cast<uint32_t>(bin) << ws);
  out.t = make_w(key_t, 0xFFFFFFFFu);
  out.vlo = static_cast<uint64_t>(key_t) << idx_bits;
  out.ok = true;
  return out;
}

// ---------------------------------------------------------------------------
// Mid-stream compaction (cold path): cut the buffer back to between k and
// k + slack candidates and return the new count, threshold word and lower bound.
// ---------------------------------------------------------------------------
struct CompactOut {
  int cnt;
  unsigned long long tw;
  uint64_t vlo;
};

template <int DT, int THREADS>
__device__ __noinline__ CompactOut compact_buffer(typename Elem<DT>::bits_t* cb, uint32_t* ci, uint32_t* holes,
                                                  Ctl& ctl, cg::cluster_group& cluster, int cnt, int k, int slack,
                                                  int idx_bits, uint64_t vmax, uint64_t vlo) {
  const uint64_t vhi = cta_vmax<THREADS>(vmax, ctl);   // barrier: survivors written
  const SelResult sel = radix_select<DT, THREADS, false>(cb, ci, cnt, k, slack, idx_bits, vlo, vhi, ctl, cluster);
  CompactOut out;
  out.cnt = holes_compact<DT, THREADS>(cb, ci, cnt, sel.kept, sel, idx_bits, ctl, holes);
  out.tw = threshold_of(sel, Elem<DT>::kKeyBits, idx_bits);
  out.vlo = v_floor(sel, Elem<DT>::kKeyBits + idx_bits);
  return out;
}

// ---------------------------------------------------------------------------
// Streaming kernel.  Grid: rows x groups x cluster CTAs, clusters of `cluster`
// CTAs along x.  CTA (row, g, rank) filters slice g*cluster + rank of the row.
//
// Per round every thread screens VPT 16-byte vectors from the shared-memory
// ring; survivors are written at offsets from per-warp counts (one barrier, no
// atomics).  Round 0 first seeds T from a histogram of its own elements, so
// that T starts near the k-th value instead of at -inf.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__global__ void __launch_bounds__(THREADS, 1) topk_stream_kernel(const __grid_constant__ KParams p) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  constexpr int B = kBlockElems;
  constexpr int VPB = B / PV;                          // 16-byte vectors per block
  constexpr int R = round_elems_for(E::kBytes);       // elements per round
  constexpr int Q = R / B;                             // blocks per round
  constexpr int VPT = R / (THREADS * PV);              // vectors per thread per round
  static_assert(VPB % 32 == 0, "a warp must stay inside one block");
  static_assert(VPT >= 1 && VPT * THREADS * PV == R && Q * B == R, "round shape");
  static_assert(Q <= NW, "one refill per warp");
  static_assert(kSeedBins % (NW * 32) == 0, "seed histogram split");

  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint32_t* blk_off = reinterpret_cast<uint32_t*>(smem + p.off_blk);
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  uint32_t* holes = reinterpret_cast<uint32_t*>(smem + p.off_holes);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + p.off_ctl);
  int* seed_hist = reinterpret_cast<int*>(ci);         // round-0 histogram, dead before any append

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) / (C * p.groups);
  const int g = static_cast<int>((blockIdx.x / C) % p.groups);
  const int D = p.stages;
#ifdef DSEL_STATS
  const long long st_t0 = clock64();
  long long st_t1 = st_t0;
  int st_rounds = 0;
  long long st_ev[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  long long st_wait = 0;
#define DSEL_EV(i) do { if (tid == 0) st_ev[i] = clock64() - st_t0; } while (0)
  const int tr_w = (blockIdx.x == 0 && lane == 0 && warp % 5 == 0) ? warp / 5 : -1;
#define DSEL_TR(r, e) do { if (tr_w >= 0 && (r) < kTraceRounds) \
    g_trace[(tr_w * kTraceRounds + (r)) * kTraceEvents + (e)] = clock64() - st_t0; } while (0)
#else
#define DSEL_EV(i) do { } while (0)
#define DSEL_TR(r, e) do { } while (0)
#endif

  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);

  for (int i = tid; i < 3 * kBins; i += THREADS) (&ctl.hist[0][0])[i] = 0;
  for (int i = tid; i < kSeedBins; i += THREADS) seed_hist[i] = 0;
  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.nan_found = 0;
    ctl.abort = 0;
    ctl.hb = 0;
#ifdef DSEL_STATS
    ctl.st_compact_cycles = 0;
    ctl.st_compactions = 0;
    ctl.st_appended = 0;
    ctl.st_slow_vectors = 0;
#endif
    for (int s = 0; s < D; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  if (C > 1) cluster.sync();   // peers' control blocks are ready before anyone touches them remotely
  else __syncthreads();
  DSEL_EV(0);

  const bool leader = (g == 0 && crank == 0);
  if (bad_end || n <= p.k) {
    if (p.groups == 1 && leader) {
      if (bad_end) write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_BAD_END);
      else write_short_row<DT, THREADS>(p, row, n);
    }
  } else {
    // ---- this CTA's slice: [lo, hi), a multiple of 16 elements wide ----
    const int S = p.groups * C;
    const int sid = g * C + crank;
    const int64_t slice = ((n + S - 1) / S + 15) / 16 * 16;
    const int64_t lo = min(n, static_cast<int64_t>(sid) * slice);
    const int64_t hi = min(n, lo + slice);
    const int nb = static_cast<int>((hi - lo + B - 1) / B);
    const char* rowp = static_cast<const char*>(p.x) + row * p.row_stride * E::kBytes;

    // ---- block visiting order: j -> (pa * j + pc) mod nb, pa coprime with nb ----
    uint32_t pa = 1, pc = 0;
    if (nb > 1) {
      const uint32_t unb = static_cast<uint32_t>(nb);
      pa = static_cast<uint32_t>((static_cast<uint64_t>(unb) * 618u + 500u) / 1000u) | 1u;
      for (;;) {
        uint32_t a = pa, b = unb;
        while (b) { const uint32_t t = a % b; a = b; b = t; }
        if (a == 1u) break;
        pa += 2u;
      }
      pa %= unb;
      const uint64_t h = (static_cast<uint64_t>(row) + 1) * 0x9E3779B97F4A7C15ull ^
                         (static_cast<uint64_t>(sid) + 1) * 0xBF58476D1CE4E5B9ull;
      pc = static_cast<uint32_t>((h >> 29) % unb);
    }
    auto issue = [&](int j) {
      const uint32_t m = static_cast<uint32_t>((static_cast<uint64_t>(pa) * static_cast<uint32_t>(j) + pc) %
                                               static_cast<uint32_t>(nb));
      const int64_t e0 = lo + static_cast<int64_t>(m) * B;
      const int64_t ce = min(static_cast<int64_t>(B), hi - e0);
      const uint32_t bytes = static_cast<uint32_t>((ce * E::kBytes + 15) & ~static_cast<int64_t>(15));
      const int s = j % D;
      blk_off[s] = static_cast<uint32_t>(e0);
      const uint32_t bar = smem_u32(&bars[s]);
      mbar_expect_tx(bar, bytes);
      bulk_g2s(smem_u32(ring + static_cast<size_t>(s) * B * E::kBytes), rowp + e0 * E::kBytes, bytes, bar);
    };
    {   // prologue: the first D blocks, one per thread
      const int first = min(D, nb);
      for (int j = tid; j < first; j += THREADS) issue(j);
    }
    DSEL_EV(1);

    // per-slot state: which block of the round, which vector in it, ring stage/phase
    int qv[VPT], ov[VPT], stg[VPT];
    uint32_t phs[VPT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) {
      const int u = v * THREADS + tid;
      qv[v] = u / VPB;
      ov[v] = u % VPB;
      stg[v] = qv[v];   // q < Q <= D
      phs[v] = 0;
    }

    const uint32_t uhi = static_cast<uint32_t>(hi);
    const uint32_t idx_mask = mask_bits(p.idx_bits);
    uint64_t vmax = 0;             // largest radix word this thread appended
    uint64_t vlo = 0;              // every candidate's radix word is >= vlo
    unsigned long long t_own = 0;  // this CTA's threshold word
    int cnt = 0;                   // candidates in the buffer (same value in every thread)
    bool nan_thread = false;
    const int rounds = (nb + Q - 1) / Q;
    for (int r = 0; r < rounds; ++r) {
      DSEL_TR(r, 0);
      // ---- 1. wait for and load this round's vectors ----
      uint4 val[VPT];
      uint32_t eidx[VPT];
      bool have[VPT];
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int j = r * Q + qv[v];
        val[v] = make_uint4(0u, 0u, 0u, 0u);
        eidx[v] = 0;
        have[v] = false;
        if (j < nb) {   // warp-uniform
          const int s = stg[v];
#ifdef DSEL_STATS
          const long long w0 = clock64();
#endif
          if (!mbar_wait(smem_u32(&bars[s]), phs[v])) ctl.abort = 1;
#ifdef DSEL_STATS
          st_wait += clock64() - w0;
#endif
          eidx[v] = blk_off[s] + static_cast<uint32_t>(ov[v] * PV);
          if (eidx[v] < uhi) {
            have[v] = true;
            val[v] = *reinterpret_cast<const uint4*>(ring + static_cast<size_t>(s) * B * E::kBytes + ov[v] * 16);
          }
        }
        stg[v] += Q;
        if (stg[v] >= D) {
          stg[v] -= D;
          phs[v] ^= 1u;
        }
      }

      DSEL_TR(r, 1);
      // ---- 2. round 0: seed T from a histogram of the round's keys ----
      if (r == 0) {
        uint32_t voff[VPT];
#pragma unroll
        for (int v = 0; v < VPT; ++v) {   // where this thread's round-0 vectors sit
          int s0 = stg[v] - Q;
          if (s0 < 0) s0 += D;
          voff[v] = have[v] ? static_cast<uint32_t>(s0 * B * E::kBytes + ov[v] * 16) : 0xFFFFFFFFu;
        }
        const SeedOut so = seed_threshold<DT, THREADS, VPT>(ring, voff, eidx, uhi, p.k, p.idx_bits, ctl, seed_hist);
        if (so.ok) {
          t_own = so.t;
          vlo = so.vlo;
        }
      }

      // ---- 3. screen + exact test against T; per-warp survivor counts ----
      const unsigned long long tp = *reinterpret_cast<volatile unsigned long long*>(&ctl.t_w);
      const unsigned long long w = tp > t_own ? tp : t_own;   // a peer may have raised it
      const uint32_t tk = static_cast<uint32_t>(w >> 32);
      const uint32_t ti = ~static_cast<uint32_t>(w);
      uint32_t tv = E::bits_of_key(tk);
      if (DT == DSEL_BF16) tv |= tv << 16;
      uint32_t keep[VPT];
      int mine = 0;   // survivors of this thread in this round
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        keep[v] = 0;
        const bool tail = have[v] && (eidx[v] + PV > uhi);
        const bool maybe = have[v] && (tail || screen<DT>(val[v], tv));
        if (__any_sync(0xffffffffu, maybe)) {   // warp-uniform
#ifdef DSEL_STATS
          if (lane == 0) atomicAdd(&ctl.st_slow_vectors, 1);
#endif
          uint32_t cm = maybe ? candidate_mask<DT>(val[v], tv) : 0u;
          if (tail) cm &= (1u << (uhi - eidx[v])) - 1u;   // elements at or past hi are not this row's
          while (cm) {   // exact test, only for the elements the float compare let through
            const int e = __ffs(cm) - 1;
            cm &= cm - 1u;
            const uint32_t b = vec_elem_dyn<DT>(val[v], e);
            const uint32_t idx = eidx[v] + e;
            if (E::is_nan(b)) {
              if (!p.nan_flag) nan_trap();   // the pages' default policy: abort on NaN
              nan_thread = true;
            } else {
              const uint32_t kk = E::key(b);
              if (kk > tk || (kk == tk && idx < ti)) {
                keep[v] |= 1u << e;
                const uint64_t vv = (static_cast<uint64_t>(kk) << p.idx_bits) | (idx_mask - idx);
                vmax = vv > vmax ? vv : vmax;
              }
            }
          }
          mine += __popc(keep[v]);
        }
      }
      const int wcount = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(mine)));
      if (lane == 0) ctl.wc[r & 1][warp] = wcount;
      if (r == 0) DSEL_EV(2);
      DSEL_TR(r, 2);
      __syncthreads();
      DSEL_TR(r, 3);
      if (r == 0) DSEL_EV(3);
      // refill the stages this round consumed: warp q issues block r*Q + q + D
      if (warp < Q && lane == 0) {
        const int j = r * Q + warp + D;
        if (j < nb) issue(j);
      }
      // ---- 4. write survivors at offsets from the per-warp counts ----
      int total;
      const int woff = cnt + warp_prefix_of<NW>(ctl.wc[r & 1], warp, lane, total);
      DSEL_TR(r, 6);
#ifdef DSEL_STATS
      if (tr_w >= 0 && r < kTraceRounds) g_trace[(tr_w * kTraceRounds + r) * kTraceEvents + 7] = wcount;
#endif
      if (wcount != 0) {   // warp-uniform
        const int incl = warp_incl_scan(mine, lane);
        int pos = woff + incl - mine;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          uint32_t km = keep[v];
          while (km) {
            const int e = __ffs(km) - 1;
            km &= km - 1u;
            cb[pos] = static_cast<bits_t>(vec_elem_dyn<DT>(val[v], e));
            ci[pos] = eidx[v] + e;
            ++pos;
          }
        }
      }
      cnt += total;
      DSEL_TR(r, 4);
#ifdef DSEL_STATS
      if (tid == 0) ctl.st_appended += total;
      ++st_rounds;
#endif
      // ---- 5. cut the buffer back when it holds k + B2 ----
      if (cnt >= p.k + p.b2) {   // uniform: cnt is the same register value everywhere
#ifdef DSEL_STATS
        const long long sc0 = clock64();
#endif
        const CompactOut co = compact_buffer<DT, THREADS>(cb, ci, holes, ctl, cluster, cnt, p.k, p.b2 / 2,
                                                          p.idx_bits, vmax, vlo);
        cnt = co.cnt;
        const unsigned long long tw = co.tw;
        t_own = tw > t_own ? tw : t_own;
        vlo = co.vlo;
        // any CTA's threshold is a valid bound for the whole row: push it to the peers
        if (C > 1 && warp == 0 && lane < C && lane != crank)
          atomicMax(cluster.map_shared_rank(&ctl.t_w, lane), tw);
#ifdef DSEL_STATS
        if (tid == 0) {
          ctl.st_compactions += 1;
          ctl.st_compact_cycles += static_cast<unsigned long long>(clock64() - sc0);
        }
#endif
        if (r == 0) DSEL_EV(4);
      }
      DSEL_TR(r, 5);
    }
    // A wait that gave up may leave a copy in flight: wait for it (bounded) before
    // this CTA's shared memory can go away.
    __syncthreads();
    if (ctl.abort && tid == 0) {
      for (int j = max(0, nb - D); j < nb; ++j) mbar_wait(smem_u32(&bars[j % D]), (j / D) & 1);
    }
#ifdef DSEL_STATS
    st_t1 = clock64();
#endif
    DSEL_EV(5);

    const bool to_ws = p.groups > 1;
    const int sort_mode = to_ws ? (p.order == DSEL_ORDER_INDEX ? 1 : 0) : p.order;
    finalize<DT, THREADS>(p, row, g, cb, ci, holes, ctl, cluster, cnt, nan_thread, vlo, vmax, to_ws,
                          sort_mode);
  }
#ifdef DSEL_STATS
  if (tid == 0 && blockIdx.x < kStatsCtas) {
    unsigned long long* st = g_stats + static_cast<size_t>(blockIdx.x) * kStatsFields;
    st[0] = static_cast<unsigned long long>(st_t1 - st_t0);
    st[1] = static_cast<unsigned long long>(clock64() - st_t1);
    st[2] = ctl.st_compact_cycles;
    st[3] = static_cast<unsigned long long>(ctl.st_compactions);
    st[4] = static_cast<unsigned long long>(ctl.st_appended);
    st[5] = static_cast<unsigned long long>(ctl.st_slow_vectors);
    st[6] = static_cast<unsigned long long>(st_rounds);
    st[7] = 0;
    for (int i = 0; i < 6; ++i) st[8 + i] = static_cast<unsigned long long>(st_ev[i]);
    st[14] = static_cast<unsigned long long>(st_wait);
    st[15] = static_cast<unsigned long long>(clock64() - st_t0);
  }
#endif
#undef DSEL_EV
#undef DSEL_TR
  if (C > 1) cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// Merge kernel for split-row plans.  Grid: rows x cluster CTAs.  The groups'
// partial results (each at most k entries) are concatenated in group order;
// CTA rank r of the row's cluster loads a contiguous share of that list and the
// cluster runs the final phase.  When the output is index-sorted, the groups'
// lists are index-sorted and cover increasing index ranges, so per-CTA index
// sorts concatenate into a sorted row.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__global__ void __launch_bounds__(THREADS, 1) topk_merge_kernel(const __grid_constant__ KParams p) {
  using bits_t = typename Elem<DT>::bits_t;
  extern __shared__ __align__(1024) unsigned char smem[];
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  uint32_t* holes = reinterpret_cast<uint32_t*>(smem + p.off_holes);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + p.off_ctl);

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int64_t row = static_cast<int64_t>(blockIdx.x) / C;

  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);
  for (int i = tid; i < 3 * kBins; i += THREADS) (&ctl.hist[0][0])[i] = 0;
  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.nan_found = 0;
    ctl.abort = 0;
    ctl.hb = 0;
  }
  if (C > 1) cluster.sync();
  else __syncthreads();
  if (bad_end || n <= p.k) {
    if (crank == 0) {
      if (bad_end) write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_BAD_END);
      else write_short_row<DT, THREADS>(p, row, n);
    }
  } else {
    // group prefix sums (groups <= kBins) in the histogram scratch
    int* pref = ctl.hsum;
    const int2* meta = p.ws_meta + row * p.groups;
    if (tid == 0) {
      int acc = 0, nan = 0;
      for (int gg = 0; gg < p.groups; ++gg) {
        const int2 mt = meta[gg];
        pref[gg] = acc;
        acc += mt.x;
        nan |= mt.y;
      }
      pref[p.groups] = acc;
      ctl.nan_found = nan;
    }
    __syncthreads();
    const int total = pref[p.groups];
    const bool nan = ctl.nan_found != 0;
    const int a = static_cast<int>(static_cast<int64_t>(total) * crank / C);
    const int b = static_cast<int>(static_cast<int64_t>(total) * (crank + 1) / C);
    uint64_t vmx = 0;
    if (!nan) {
      const uint2* src = p.ws_pairs + row * p.groups * static_cast<int64_t>(p.k);
      const uint32_t idx_mask = mask_bits(p.idx_bits);
      for (int i = a + tid; i < b; i += THREADS) {
        int lo = 0, hi = p.groups - 1;   // last group whose prefix <= i
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (pref[mid] <= i) lo = mid;
          else hi = mid - 1;
        }
        const uint2 pr = src[static_cast<int64_t>(lo) * p.k + (i - pref[lo])];
        cb[i - a] = static_cast<bits_t>(pr.y);
        ci[i - a] = pr.x;
        const uint64_t v = make_v<DT>(pr.y, pr.x, p.idx_bits, idx_mask);
        vmx = v > vmx ? v : vmx;
      }
    }
    __syncthreads();   // pref (histogram scratch) is dead from here on
    finalize<DT, THREADS>(p, row, 0, cb, ci, holes, ctl, cluster, nan ? 0 : (b - a), nan, 0ull, vmx, false,
                          p.order);
  }
  if (C > 1) cluster.sync();
}

}  // namespace dsel
