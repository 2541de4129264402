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
  uint32_t off_bars, off_blk, off_cb, off_ci, off_ctl;
};

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

// ---------------------------------------------------------------------------
// Slow path of the filter (warp-collective): exact composite test of the
// elements of a screened vector, NaN detection, and a warp-aggregated append to
// the candidate buffer.
// ---------------------------------------------------------------------------
template <int DT>
__device__ __forceinline__ void filter_append(const uint4& val, uint32_t e_idx, uint32_t hi, bool act,
                                              uint32_t tk, uint32_t ti, typename Elem<DT>::bits_t* cb,
                                              uint32_t* ci, Ctl& ctl, int nan_flag, int lane) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int PV = E::kPerVec;
  uint32_t keep = 0;
  bool nan = false;
  if (act) {
#pragma unroll
    for (int e = 0; e < PV; ++e) {
      const uint32_t b = vec_elem<DT>(val, e);
      const uint32_t idx = e_idx + e;
      if (idx < hi) {
        if (E::is_nan(b)) {
          nan = true;
        } else {
          const uint32_t kk = E::key(b);
          if (kk > tk || (kk == tk && idx < ti)) keep |= 1u << e;
        }
      }
    }
  }
  if (nan) {
    if (!nan_flag) nan_trap();   // the pages' default policy: abort on NaN
    ctl.nan_found = 1;
  }
  const int c = __popc(keep);
  const int incl = warp_incl_scan(c, lane);
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  if (total == 0) return;
  int base = 0;
  if (lane == 31) base = atomicAdd(&ctl.cnt, total);
  base = __shfl_sync(0xffffffffu, base, 31);
  int pos = base + incl - c;
#pragma unroll
  for (int e = 0; e < PV; ++e) {
    if (keep & (1u << e)) {
      cb[pos] = static_cast<bits_t>(vec_elem<DT>(val, e));
      ci[pos] = e_idx + e;
      ++pos;
    }
  }
}

// ---------------------------------------------------------------------------
// Final phase, shared by the streaming and merge kernels.  The cluster's CTAs
// together hold a superset of the row's (or row part's) top entries; they pick
// exactly min(k, total) of them with a cluster-wide radix select, optionally sort,
// and write them to the output (or to the split-row workspace).
//   sort_mode 0: none, 1: ascending index per CTA (slices are in index order, so
//   the concatenation is sorted), 2: value order after gathering on rank 0.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__device__ void finalize(const KParams& p, int64_t row, int g, typename Elem<DT>::bits_t* cb,
                         uint32_t* ci, Ctl& ctl, cg::cluster_group& cluster, bool to_workspace,
                         int sort_mode) {
  using bits_t = typename Elem<DT>::bits_t;
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    ctl.x_cnt = ctl.cnt;
    ctl.x_nan = ctl.nan_found;
  }
  cluster.sync();
  if (warp == 0) {
    int c = 0, nn = 0;
    if (lane < C) {
      Ctl* pc = cluster.map_shared_rank(&ctl, lane);
      c = pc->x_cnt;
      nn = pc->x_nan;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      c += __shfl_xor_sync(0xffffffffu, c, o);
      nn |= __shfl_xor_sync(0xffffffffu, nn, o);
    }
    if (lane == 0) {
      ctl.tot = c;
      ctl.any_nan = nn;
    }
  }
  __syncthreads();
  const int tot = ctl.tot;
  if (ctl.any_nan) {
    if (to_workspace) {
      if (crank == 0 && tid == 0) p.ws_meta[row * p.groups + g] = make_int2(0, 1);
    } else if (crank == 0) {
      write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_NAN);
    }
    return;
  }
  const int need = min(p.k, tot);
  const int cnt = ctl.cnt;
  int m = cnt;
  if (tot > need) {
    const SelResult sel = radix_select<DT, THREADS, true>(cb, ci, cnt, need, p.idx_bits, ctl, cluster);
    m = stable_compact<DT, THREADS>(cb, ci, cnt, sel, p.idx_bits, ctl);
  }
  if (sort_mode == 1) bitonic_sort<DT, THREADS, false>(cb, ci, m);
  if (tid == 0) ctl.x_kept = m;
  cluster.sync();
  if (sort_mode == 2) {
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
      write_rows_out<DT, THREADS>(p, row, 0, off, cb, ci);
    }
    return;
  }
  if (warp == 0) {
    int c = 0;
    if (lane < crank) c = cluster.map_shared_rank(&ctl, lane)->x_kept;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) ctl.kept_off = c;
  }
  __syncthreads();
  const int off = ctl.kept_off;
  if (to_workspace) {
    uint2* dst = p.ws_pairs + (row * p.groups + g) * static_cast<int64_t>(p.k) + off;
    for (int i = tid; i < m; i += THREADS) dst[i] = make_uint2(ci[i], static_cast<uint32_t>(cb[i]));
    if (crank == 0 && tid == 0) p.ws_meta[row * p.groups + g] = make_int2(need, 0);
  } else {
    write_rows_out<DT, THREADS>(p, row, off, m, cb, ci);
  }
}

// ---------------------------------------------------------------------------
// Streaming kernel.  Grid: rows x groups x cluster CTAs, clusters of `cluster`
// CTAs along x.  CTA (row, g, rank) filters slice g*cluster + rank of the row.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__global__ void __launch_bounds__(THREADS, 1) topk_stream_kernel(const __grid_constant__ KParams p) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int PV = E::kPerVec;
  constexpr int B = kBlockElems;
  constexpr int VPB = B / PV;                          // 16-byte vectors per block
  constexpr int Q = kRoundElems / B;                   // blocks per round
  constexpr int VPT = kRoundElems / (THREADS * PV);    // vectors per thread per round
  static_assert(VPB % 32 == 0, "a warp must stay inside one block");
  static_assert(VPT >= 1 && VPT * THREADS * PV == kRoundElems, "round shape");

  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char* ring = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  uint32_t* blk_off = reinterpret_cast<uint32_t*>(smem + p.off_blk);
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + p.off_ctl);

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) / (C * p.groups);
  const int g = static_cast<int>((blockIdx.x / C) % p.groups);
  const int D = p.stages;

  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);

  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.cnt = 0;
    ctl.nan_found = 0;
    ctl.abort = 0;
    for (int s = 0; s < D; ++s) mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  cluster.sync();   // peers' control blocks are ready before anyone reads them remotely

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
    if (tid == 0) {
      const int first = min(D, nb);
      for (int j = 0; j < first; ++j) issue(j);
    }

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

    uint32_t tk = 0, ti = 0xFFFFFFFFu;
    uint32_t tv = E::bits_of_key(0);
    if (DT == DSEL_BF16) tv |= tv << 16;
    const uint32_t uhi = static_cast<uint32_t>(hi);
    const int rounds = (nb + Q - 1) / Q;
    for (int r = 0; r < rounds; ++r) {
      unsigned long long peer_t = 0ull;
      if (C > 1 && warp == 0 && lane < C && lane != crank)
        peer_t = *reinterpret_cast<volatile unsigned long long*>(cluster.map_shared_rank(&ctl.t_w, lane));
#pragma unroll
      for (int v = 0; v < VPT; ++v) {
        const int j = r * Q + qv[v];
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        uint32_t e_idx = 0;
        bool have = false;
        if (j < nb) {   // warp-uniform
          const int s = stg[v];
          if (!mbar_wait(smem_u32(&bars[s]), phs[v])) ctl.abort = 1;
          e_idx = blk_off[s] + static_cast<uint32_t>(ov[v] * PV);
          if (e_idx < uhi) {
            have = true;
            val = *reinterpret_cast<const uint4*>(ring + static_cast<size_t>(s) * B * E::kBytes + ov[v] * 16);
          }
        }
        const bool maybe = have && ((e_idx + PV > uhi) || screen<DT>(val, tv));
        if (__any_sync(0xffffffffu, maybe))
          filter_append<DT>(val, e_idx, uhi, maybe, tk, ti, cb, ci, ctl, p.nan_flag, lane);
        stg[v] += Q;
        if (stg[v] >= D) {
          stg[v] -= D;
          phs[v] ^= 1u;
        }
      }
      __syncthreads();
      if (tid == 0) {   // refill the stages this round consumed
#pragma unroll
        for (int q = 0; q < Q; ++q) {
          const int j = r * Q + q;
          if (j + D < nb) issue(j + D);
        }
      }
      if (ctl.cnt >= p.k + p.b2) {   // cut the buffer back to k and raise T
        const int cnt = ctl.cnt;
        const SelResult sel = radix_select<DT, THREADS, false>(cb, ci, cnt, p.k, p.idx_bits, ctl, cluster);
        const int kept = stable_compact<DT, THREADS>(cb, ci, cnt, sel, p.idx_bits, ctl);
        if (tid == 0) {
          ctl.cnt = kept;
          const unsigned long long w = threshold_of(sel, E::kKeyBits, p.idx_bits);
          if (w > ctl.t_w) ctl.t_w = w;
        }
      }
      if (C > 1 && warp == 0) {   // adopt a peer's higher threshold (any peer's T is a valid bound)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long y = __shfl_xor_sync(0xffffffffu, peer_t, o);
          peer_t = y > peer_t ? y : peer_t;
        }
        if (lane == 0 && peer_t > ctl.t_w) ctl.t_w = peer_t;
      }
      __syncthreads();
      const unsigned long long w = ctl.t_w;
      tk = static_cast<uint32_t>(w >> 32);
      ti = ~static_cast<uint32_t>(w);
      tv = E::bits_of_key(tk);
      if (DT == DSEL_BF16) tv |= tv << 16;
    }
    // A wait that gave up may leave a copy in flight: wait for it (bounded) before
    // this CTA's shared memory can go away.
    if (ctl.abort && tid == 0) {
      for (int j = max(0, nb - D); j < nb; ++j) mbar_wait(smem_u32(&bars[j % D]), (j / D) & 1);
    }
    __syncthreads();

    const bool to_ws = p.groups > 1;
    const int sort_mode = to_ws ? (p.order == DSEL_ORDER_INDEX ? 1 : 0) : p.order;
    finalize<DT, THREADS>(p, row, g, cb, ci, ctl, cluster, to_ws, sort_mode);
  }
  cluster.sync();   // no CTA leaves while a peer may still read its shared memory
}

// ---------------------------------------------------------------------------
// Merge kernel for split-row plans.  Grid: rows x cluster CTAs.  The groups'
// partial results (each at most k entries, in index order when the output is
// index-sorted) are concatenated in group order; CTA rank r of the row's cluster
// loads a contiguous share of that list and the cluster runs the final phase.
// Because the compaction is stable and the groups cover increasing index ranges,
// index order survives without another sort.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__global__ void __launch_bounds__(THREADS, 1) topk_merge_kernel(const __grid_constant__ KParams p) {
  using bits_t = typename Elem<DT>::bits_t;
  extern __shared__ __align__(1024) unsigned char smem[];
  bits_t* cb = reinterpret_cast<bits_t*>(smem + p.off_cb);
  uint32_t* ci = reinterpret_cast<uint32_t*>(smem + p.off_ci);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + p.off_ctl);

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x;
  const int64_t row = static_cast<int64_t>(blockIdx.x) / C;

  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);
  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.cnt = 0;
    ctl.nan_found = 0;
    ctl.abort = 0;
  }
  __syncthreads();
  cluster.sync();
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
    const int a = static_cast<int>(static_cast<int64_t>(total) * crank / C);
    const int b = static_cast<int>(static_cast<int64_t>(total) * (crank + 1) / C);
    if (!ctl.nan_found) {
      const uint2* src = p.ws_pairs + row * p.groups * static_cast<int64_t>(p.k);
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
      }
    }
    __syncthreads();
    if (tid == 0) ctl.cnt = ctl.nan_found ? 0 : (b - a);
    __syncthreads();
    finalize<DT, THREADS>(p, row, 0, cb, ci, ctl, cluster, false,
                          p.order == DSEL_ORDER_VALUE ? 2 : 0);
  }
  cluster.sync();
}

}  // namespace dsel
