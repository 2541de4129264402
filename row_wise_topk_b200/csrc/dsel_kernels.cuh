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
  int32_t capacity;         // candidate-buffer slots
  uint32_t off_bars, off_blk, off_cb, off_ci, off_holes, off_ctl;
  uint32_t off_hist, off_tab;   // row-resident kernel: histograms, scan table
  uint32_t off_cv;              // slice kernel: candidate-vector list
  int32_t vpt_cap;          // slice kernel: chunks of the largest slice (one mbarrier each)
  uint32_t sl_full;         // slice kernel, rows of row_stride elements: slice length,
  int32_t nch_full;         //   its chunks,
  uint32_t pa_full;         //   the chunk visiting stride (coprime with nch_full),
  int32_t seg;              //   candidate-list entries per (slice, warp) segment
  // sampling step after TopK (fp32 only; token_out == nullptr: no draw)
  const float* u;           // [rows] the caller's uniforms in [0, 1)
  int64_t* token_out;       // [rows] drawn index, or a negative row code
  float* prob_out;          // [rows] its probability after the top-p cut (may be nullptr)
  float temperature;        // <= 0: greedy
  float top_p;              // >= 1: no cut
};

#ifdef DSEL_STATS
constexpr int kStatsCtas = 8192;
constexpr int kStatsFields = 16;
__device__ unsigned long long g_stats[kStatsCtas * kStatsFields];
// per-round timeline of CTA 0 (lane 0 of every warp): [warp][round][event]
constexpr int kTraceWarps = 16;
constexpr int kTraceRounds = 12;
constexpr int kTraceEvents = 10;
constexpr int kTraceSize = kTraceWarps * kTraceRounds * kTraceEvents;
__device__ long long g_trace[kTraceSize];
__device__ int g_trace_cta = 0;   // the CTA whose timeline is recorded
#endif

// Per-warp marks inside a phase (CTA 0, lane 0 of each warp), stats builds
// only: absolute clocks in trace row kTraceRounds - 2.
__device__ __forceinline__ void trace_mark(int e) {
#ifdef DSEL_STATS
  if (blockIdx.x == g_trace_cta && (threadIdx.x & 31) == 0 && (threadIdx.x >> 5) < kTraceWarps)
    g_trace[((threadIdx.x >> 5) * kTraceRounds + kTraceRounds - 2) * kTraceEvents + e] = clock64();
#else
  (void)e;
#endif
}

// Final-phase timeline of CTA 0 (thread 0), stats builds only: absolute clocks
// in trace row kTraceRounds - 1 of warp 0; slot kTraceEvents - 1 holds the
// kernel-start clock.
__device__ __forceinline__ void trace_final(int e) {
#ifdef DSEL_STATS
  if (blockIdx.x == g_trace_cta && threadIdx.x == 0) g_trace[(kTraceRounds - 1) * kTraceEvents + e] = clock64();
#else
  (void)e;
#endif
}

constexpr int kSeedBits = 11;                 // round-0 histogram: 2048 bins
constexpr int kSeedBins = 1 << kSeedBits;

// ---------------------------------------------------------------------------
// Output writers (all threads of one CTA).
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__device__ void write_rows_out(const KParams& p, int64_t row, int off, int m,
                               const typename Elem<DT>::bits_t* cb, const uint32_t* ci) {
  using bits_t = typename Elem<DT>::bits_t;
  if (p.indices_out == nullptr) return;   // a sampling call that wants only the token
  const int64_t base = row * p.k + off;
#pragma unroll 1
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
#pragma unroll 1
  for (int i = threadIdx.x; i < m; i += THREADS) dst[i] = make_uint2(ci[i], static_cast<uint32_t>(cb[i]));
}

template <int DT, int THREADS>
__device__ __noinline__ void write_sentinel_row(const KParams& p, int64_t row, int32_t code) {
  using bits_t = typename Elem<DT>::bits_t;
  if (p.token_out != nullptr && threadIdx.x == 0) {   // the row's draw carries the same code
    p.token_out[row] = code;
    if (p.prob_out != nullptr) p.prob_out[row] = __int_as_float(0x7FC00000);
  }
  if (p.indices_out == nullptr) return;
  const int64_t base = row * p.k;
#pragma unroll 1
  for (int i = threadIdx.x; i < p.k; i += THREADS) {
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = code;
    else static_cast<int32_t*>(p.indices_out)[base + i] = code;
    if (p.return_value) static_cast<bits_t*>(p.values_out)[base + i] = static_cast<bits_t>(Elem<DT>::kQNaN);
  }
}

// Slots n..k-1 of a short row: index DSEL_IDX_PAD, value -inf.
template <int DT, int THREADS>
__device__ void write_short_pad(const KParams& p, int64_t row, int64_t n) {
  using bits_t = typename Elem<DT>::bits_t;
  if (p.indices_out == nullptr) return;
  const int64_t base = row * p.k;
#pragma unroll 1
  for (int64_t i = n + threadIdx.x; i < p.k; i += THREADS) {
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = DSEL_IDX_PAD;
    else static_cast<int32_t*>(p.indices_out)[base + i] = DSEL_IDX_PAD;
    if (p.return_value) static_cast<bits_t*>(p.values_out)[base + i] = static_cast<bits_t>(Elem<DT>::kNegInf);
  }
}

// Rows no longer than k: every entry, in index order, then padding.  No NaN check.
template <int DT, int THREADS>
__device__ __noinline__ void write_short_row(const KParams& p, int64_t row, int64_t n) {
  using bits_t = typename Elem<DT>::bits_t;
  if (p.indices_out == nullptr) return;
  const bits_t* xr = static_cast<const bits_t*>(p.x) + row * p.row_stride;
  const int64_t base = row * p.k;
#pragma unroll 1
  for (int i = threadIdx.x; i < p.k; i += THREADS) {
    const bool in = i < n;
    const int32_t idx = in ? i : DSEL_IDX_PAD;
    if (p.index_i64) static_cast<int64_t*>(p.indices_out)[base + i] = idx;
    else static_cast<int32_t*>(p.indices_out)[base + i] = idx;
    if (p.return_value)
      static_cast<bits_t*>(p.values_out)[base + i] = in ? xr[i] : static_cast<bits_t>(Elem<DT>::kNegInf);
  }
}

// ---------------------------------------------------------------------------
// Sampling step on a row's m candidates, fp32 logits zb[0, m) in value order
// (descending, ties by ascending index) with their indices ci (all threads of
// one CTA).  Reading of the pages (which name temperature and top-p among the
// sampler settings but print no formula): weights e_i = exp((z_i - z_1) / t),
// e_i = 1 where z_i equals the largest logit z_1; the shortest prefix whose
// weight sum E_c reaches top_p of the total is kept; with the caller's uniform
// u the token is the first kept candidate whose prefix sum exceeds u * E_c, and
// its probability is e / E_c.  t <= 0 draws greedily (the first candidate).
// Float32 throughout; each thread sums a contiguous chunk, so prefix sums are
// the chunk's running sum on top of a block scan of the chunk sums.
// ---------------------------------------------------------------------------
template <int THREADS, class CtlT>
__device__ __noinline__ void sample_draw(const KParams& p, int64_t row, const uint32_t* zb, const uint32_t* ci,
                                         int m, CtlT& ctl) {
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (m <= 0) {   // uniform: nothing to draw from
    if (tid == 0) {
      p.token_out[row] = DSEL_IDX_PAD;
      if (p.prob_out != nullptr) p.prob_out[row] = __int_as_float(0x7FC00000);
    }
    return;
  }
  const float t = p.temperature;
  if (!(t > 0.0f)) {   // greedy
    if (tid == 0) {
      p.token_out[row] = static_cast<int64_t>(ci[0]);
      if (p.prob_out != nullptr) p.prob_out[row] = 1.0f;
    }
    return;
  }
  const float z1 = __uint_as_float(zb[0]);
  auto weight = [&](int i) -> float {
    const float z = __uint_as_float(zb[i]);
    return z == z1 ? 1.0f : expf((z - z1) / t);
  };
  const int per = (m + THREADS - 1) / THREADS;
  const int a = min(m, tid * per), b = min(m, a + per);
  float s = 0.0f;
#pragma unroll 1
  for (int i = a; i < b; ++i) s += weight(i);
  float incl = s;   // warp inclusive scan of the chunk sums
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) ctl.smp_w[warp] = incl;
  if (tid == 0) {
    ctl.smp_c = m - 1;        // last kept candidate: all, unless the top-p cut says fewer
    ctl.smp_pos = m;          // none drawn yet
  }
  __syncthreads();
  float before = 0.0f, total = 0.0f;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const float ws = ctl.smp_w[w];
    before += w < warp ? ws : 0.0f;
    total += ws;
  }
  const float off = before + incl - s;   // weight sum of the candidates before this chunk
  if (p.top_p < 1.0f) {
    const float tp = p.top_p * total;
    float run = off;
#pragma unroll 1
    for (int i = a; i < b; ++i) {
      run += weight(i);
      if (run >= tp) {   // first prefix sum reaching the cut
        atomicMin(&ctl.smp_c, i);
        break;
      }
    }
  }
  __syncthreads();
  const int cl = ctl.smp_c;
  if (a <= cl && cl < b) {   // the chunk holding the last kept candidate: E_c
    float run = off;
#pragma unroll 1
    for (int i = a; i <= cl; ++i) run += weight(i);
    ctl.smp_ec = run;
  }
  __syncthreads();
  const float ec = ctl.smp_ec;
  const float target = p.u[row] * ec;
  {
    float run = off;
#pragma unroll 1
    for (int i = a; i < b && i <= cl; ++i) {
      run += weight(i);
      if (run > target) {   // first prefix sum past the target
        atomicMin(&ctl.smp_pos, i);
        break;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    const int pos = min(ctl.smp_pos, cl);
    p.token_out[row] = static_cast<int64_t>(ci[pos]);
    if (p.prob_out != nullptr) p.prob_out[row] = weight(pos) / ec;
  }
}

// Rows no longer than k: the TopK output -- every entry, in index order, or in
// value order for DSEL_ORDER_VALUE (value descending, ties by index; such rows skip
// the NaN check, and a NaN takes its IEEE totalOrder place, which the
// order-preserving key gives it: sign clear above +inf, sign set below -inf) --
// then padding; for a sampling call, the draw among the n entries, which are
// checked for NaN first (the softmax has no meaning with one).
template <int DT, int THREADS, class CtlT>
__device__ __noinline__ void finish_short_row(const KParams& p, int64_t row, int64_t n,
                                              typename Elem<DT>::bits_t* cb, uint32_t* ci, CtlT& ctl) {
  const bool sampling = DT == DSEL_F32 && p.token_out != nullptr;
  if (p.order != DSEL_ORDER_VALUE && !sampling) {
    write_short_row<DT, THREADS>(p, row, n);
    return;
  }
  using bits_t = typename Elem<DT>::bits_t;
  const bits_t* xr = static_cast<const bits_t*>(p.x) + row * p.row_stride;
  bool nan = false;
#pragma unroll 1
  for (int i = threadIdx.x; i < n; i += THREADS) {
    const bits_t bits = xr[i];
    cb[i] = bits;
    ci[i] = static_cast<uint32_t>(i);
    nan |= Elem<DT>::is_nan(bits);
  }
  nan = __syncthreads_or(nan) != 0;   // uniform; also: the entries are in place
  bitonic_sort<DT, THREADS, true>(cb, ci, static_cast<int>(n));
  write_rows_out<DT, THREADS>(p, row, 0, static_cast<int>(n), cb, ci);
  write_short_pad<DT, THREADS>(p, row, n);
  if (!sampling) return;
  if (nan) {
    if (!p.nan_flag) nan_trap();   // the pages' default NaN policy
    if (threadIdx.x == 0) {
      p.token_out[row] = DSEL_IDX_NAN;
      if (p.prob_out != nullptr) p.prob_out[row] = __int_as_float(0x7FC00000);
    }
    return;
  }
  sample_draw<THREADS>(p, row, reinterpret_cast<const uint32_t*>(cb), ci, static_cast<int>(n), ctl);
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
__device__ __noinline__ int local_select(typename Elem<DT>::bits_t* cb, uint32_t* ci, int cnt, int need, int idx_bits,
                            uint64_t vlo, uint64_t vhi, Ctl& ctl, uint32_t* holes,
                            cg::cluster_group& cluster) {
  if (cnt <= need) return cnt;
  const SelResult sel =
      radix_select<DT, THREADS, false>(cb, ci, cnt, need, 0, idx_bits, vlo, vhi, ctl, cluster);
  trace_final(4);
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
// Write the kept entries of the list cb/ci[0, n) at output slots off ..
// off + m - 1.  The kept ones are those whose radix word has top sel.depth bits
// >= sel.prefix (all of them when sel.depth is 0); there are m = sel.kept.
//   * any order: each warp takes slots for its kept entries with one shared
//     atomic per 32 entries;
//   * ascending index, when the bitmap of the candidates' index span fits in
//     `scratch` (the idle bulk-copy ring): each entry's slot is the number of
//     kept indices below it, from a prefix popcount over the bitmap;
//   * otherwise (and for value order) the kept entries are compacted to the
//     front, sorted by a bitonic network and written in order.
// ---------------------------------------------------------------------------
template <int DT, int THREADS>
__device__ __noinline__ void finish_sorted(const KParams& p, int64_t row, int g, bool to_workspace,
                                           typename Elem<DT>::bits_t* cb, uint32_t* ci, int n, SelResult sel,
                                           int sort_mode, Ctl& ctl, uint32_t* holes, unsigned char* scratch,
                                           uint32_t scratch_bytes, uint32_t span_lo, uint32_t span_len, int off,
                                           int total, bool write_meta) {
  using bits_t = typename Elem<DT>::bits_t;
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t idx_mask = mask_bits(p.idx_bits);
  const int shv = Elem<DT>::kKeyBits + p.idx_bits - sel.depth;   // < 64
  auto keep = [&](int i) -> bool {
    return (make_v<DT>(cb[i], ci[i], p.idx_bits, idx_mask) >> shv) >= sel.prefix;
  };
  const int64_t obase = row * p.k + off;
  uint2* wsd = to_workspace ? p.ws_pairs + (row * p.groups + g) * static_cast<int64_t>(p.k) + off : nullptr;
  auto put = [&](int slot, int i) {
    if (!to_workspace && p.indices_out == nullptr) return;
    if (to_workspace) {
      wsd[slot] = make_uint2(ci[i], static_cast<uint32_t>(cb[i]));
    } else {
      if (p.index_i64) static_cast<int64_t*>(p.indices_out)[obase + slot] = static_cast<int64_t>(ci[i]);
      else static_cast<int32_t*>(p.indices_out)[obase + slot] = static_cast<int32_t>(ci[i]);
      if (p.return_value) static_cast<bits_t*>(p.values_out)[obase + slot] = cb[i];
    }
  };
  if (sort_mode == 0) {
    if (tid == 0) ctl.sel_flag = 0;   // next free slot
    __syncthreads();
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll 1
    for (int i0 = 0; i0 < n; i0 += THREADS) {   // same trip count in every thread
      const int i = i0 + tid;
      const bool kp = i < n && keep(i);
      const unsigned bal = __ballot_sync(0xffffffffu, kp);
      int base = 0;
      if (lane == 0 && bal != 0u) base = atomicAdd(&ctl.sel_flag, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (kp) put(base + __popc(bal & below), i);
    }
    if (to_workspace && write_meta && tid == 0) p.ws_meta[row * p.groups + g] = make_int2(total, 0);
    return;
  }
  const uint32_t words = (span_len + 31u) / 32u;
  if (sort_mode == 1 && scratch != nullptr && 8ull * words <= scratch_bytes) {
    uint32_t* bm = reinterpret_cast<uint32_t*>(scratch);
    uint32_t* wp = bm + words;
#pragma unroll 1
    for (uint32_t i = tid; i < words; i += THREADS) bm[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int i = tid; i < n; i += THREADS) {
      if (keep(i)) {
        const uint32_t d = ci[i] - span_lo;
        atomicOr(&bm[d >> 5], 1u << (d & 31u));
      }
    }
    __syncthreads();
    // prefix popcount: warp w walks its contiguous share of words, lanes side by side
    const uint32_t per = ((words + NW - 1) / NW + 31u) & ~31u;
    const uint32_t a = min(words, warp * per), b = min(words, a + per);
    int sum = 0;
#pragma unroll 1
    for (uint32_t w0 = a; w0 < b; w0 += 32) {
      const uint32_t w = w0 + lane;
      sum += __popc(w < b ? bm[w] : 0u);
    }
    sum = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(sum)));
    if (lane == 0) ctl.wm[warp] = sum;
    __syncthreads();
    int tot;
    int base = warp_prefix_of<NW>(ctl.wm, warp, lane, tot);
#pragma unroll 1
    for (uint32_t w0 = a; w0 < b; w0 += 32) {
      const uint32_t w = w0 + lane;
      const int c = __popc(w < b ? bm[w] : 0u);
      const int incl = warp_incl_scan(c, lane);
      if (w < b) wp[w] = static_cast<uint32_t>(base + incl - c);
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncthreads();
#pragma unroll 1
    for (int i = tid; i < n; i += THREADS) {
      if (keep(i)) {
        const uint32_t d = ci[i] - span_lo;
        put(static_cast<int>(wp[d >> 5]) + __popc(bm[d >> 5] & ((1u << (d & 31u)) - 1u)), i);
      }
    }
    if (to_workspace && write_meta && tid == 0) p.ws_meta[row * p.groups + g] = make_int2(total, 0);
    return;
  }
  const int m = sel.depth == 0 ? n : holes_compact<DT, THREADS>(cb, ci, n, sel.kept, sel, p.idx_bits, ctl, holes);
  sort_kept<DT, THREADS>(cb, ci, m, sort_mode);
  if (DT == DSEL_F32 && p.token_out != nullptr && !to_workspace && sort_mode == 2)   // the row's final candidates
    sample_draw<THREADS>(p, row, reinterpret_cast<const uint32_t*>(cb), ci, m, ctl);
  emit<DT, THREADS>(p, row, g, to_workspace, off, m, total, write_meta, cb, ci);
}

// The best min(k, n) entries of cb/ci[0, n) (all within [vlo, vhi]), as a
// selection result for finish_sorted (depth 0: all of them).
template <int DT, int THREADS>
__device__ __forceinline__ SelResult select_best(const KParams& p, typename Elem<DT>::bits_t* cb, uint32_t* ci, int n,
                                                 uint64_t vlo, uint64_t vhi, Ctl& ctl, uint32_t* holes,
                                                 cg::cluster_group& cluster) {
  if (n <= p.k) return SelResult{0ull, 0, n};
  // When the candidates' keys differ only in their low 8 bits, the radix
  // select's first 256-bin pass already resolves the key; otherwise its first
  // digit would be cut at key bits (for floats: the exponent) and one pass of
  // range-adaptive bins does better.  The hole list (k + B2 >= 1025 slots) is
  // idle here and holds those bins.
  const uint32_t kx = static_cast<uint32_t>(vlo >> p.idx_bits) ^ static_cast<uint32_t>(vhi >> p.idx_bits);
  if (32 - __clz(kx) <= kDigitBits)
    return radix_select<DT, THREADS, false>(cb, ci, n, p.k, 0, p.idx_bits, vlo, vhi, ctl, cluster);
  return select_by_key_hist<DT, THREADS>(cb, ci, n, p.k, p.idx_bits, vlo, vhi, ctl, reinterpret_cast<int*>(holes),
                                         cluster);
}

template <int DT, int THREADS>
__device__ __noinline__ void finalize(const KParams& p, int64_t row, int g, typename Elem<DT>::bits_t* cb,
                         uint32_t* ci, uint32_t* holes, Ctl& ctl, cg::cluster_group& cluster,
                         int cnt, bool nan_local, uint64_t vlo, uint64_t vmax_thread,
                         bool to_workspace, int sort_mode, unsigned char* ring, uint32_t ring_bytes,
                         uint32_t span_lo, uint32_t span_len) {
  using bits_t = typename Elem<DT>::bits_t;
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31;
  const uint32_t idx_mask = mask_bits(p.idx_bits);

  trace_final(0);
  if (nan_local) ctl.nan_found = 1;
  const uint64_t vhi = cta_vmax<THREADS>(vmax_thread, ctl);   // barrier: nan_found visible
  const bool nan_cta = ctl.nan_found != 0;
  trace_final(1);

  if (C == 1) {
    if (nan_cta) {
      emit_nan<DT, THREADS>(p, row, g, to_workspace);
      return;
    }
    const SelResult sel = select_best<DT, THREADS>(p, cb, ci, cnt, vlo, vhi, ctl, holes, cluster);
    trace_final(5);
    finish_sorted<DT, THREADS>(p, row, g, to_workspace, cb, ci, cnt, sel, sort_mode, ctl, holes, ring, ring_bytes,
                               span_lo, span_len, 0, sel.kept, true);
    trace_final(6);
    return;
  }

  if (p.gather) {
    // exchange counts, bounds and NaN state
    if (tid == 0) {
      ctl.x_cnt = cnt;
      ctl.x_nan = nan_cta ? 1 : 0;
      ctl.x_vlo = cnt > 0 ? vlo : ~0ull;
      ctl.x_vhi = cnt > 0 ? vhi : 0ull;
    }
    cluster.sync();
    trace_final(2);
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
    // the raw candidates fit rank 0's buffer: gather them as they are; otherwise
    // every CTA keeps its own best k first
    const bool direct = tot <= p.capacity;   // uniform over the cluster
    int m = cnt;
    if (!direct) {
      m = local_select<DT, THREADS>(cb, ci, cnt, p.k, p.idx_bits, vlo, vhi, ctl, holes, cluster);
      if (tid == 0) ctl.x_kept = m;
      cluster.sync();
      lo = 0ull;
    }
    // the CTA holding the most candidates gathers the others' (ties: the lower
    // rank), so that the fewest cross the cluster: under a drift across the row
    // one slice holds nearly all of them
    int held = 0;
    if (lane < C) {
      Ctl* pc = cluster.map_shared_rank(&ctl, lane);
      held = direct ? pc->x_cnt : pc->x_kept;
    }
    const unsigned lkey = __reduce_max_sync(
        0xffffffffu, lane < C ? (static_cast<unsigned>(held) << 8) | static_cast<unsigned>(255 - lane) : 0u);
    const int leader = 255 - static_cast<int>(lkey & 255u);
    if (crank != leader) return;
    int off = m;
#pragma unroll 1
    for (int r = 0; r < C; ++r) {
      if (r == leader) continue;
      Ctl* pr = cluster.map_shared_rank(&ctl, r);
      const int mr = direct ? pr->x_cnt : pr->x_kept;
      const bits_t* rcb = cluster.map_shared_rank(cb, r);
      const uint32_t* rci = cluster.map_shared_rank(ci, r);
#pragma unroll 1
      for (int i = tid; i < mr; i += THREADS) {
        cb[off + i] = rcb[i];
        ci[off + i] = rci[i];
      }
      off += mr;
    }
    __syncthreads();   // the gathered list is complete
    trace_final(3);
    const SelResult sel = select_best<DT, THREADS>(p, cb, ci, off, lo, hi, ctl, holes, cluster);
    trace_final(5);
    finish_sorted<DT, THREADS>(p, row, g, to_workspace, cb, ci, off, sel, sort_mode, ctl, holes, ring, ring_bytes,
                               span_lo, span_len, 0, sel.kept, true);
    trace_final(6);
    return;
  }

  // ---- distributed select over the cluster ----
#pragma unroll 1
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
  if (tid == 0) ctl.x_kept = m;
  cluster.sync();
  if (sort_mode == 2) {   // gather the winners on rank 0 and sort them by value
    if (crank == 0) {
      int off = m;
#pragma unroll 1
      for (int r = 1; r < C; ++r) {
        const int mr = cluster.map_shared_rank(&ctl, r)->x_kept;
        const bits_t* rcb = cluster.map_shared_rank(cb, r);
        const uint32_t* rci = cluster.map_shared_rank(ci, r);
#pragma unroll 1
        for (int i = tid; i < mr; i += THREADS) {
          cb[off + i] = rcb[i];
          ci[off + i] = rci[i];
        }
        off += mr;
      }
      __syncthreads();
      finish_sorted<DT, THREADS>(p, row, g, to_workspace, cb, ci, off, SelResult{0ull, 0, off}, 2, ctl, holes, nullptr,
                                 0u, 0u, 0u, 0, off, true);
    }
    return;
  }
  int off = lane < crank ? cluster.map_shared_rank(&ctl, lane)->x_kept : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
  // each CTA orders its own share (its slice is an index range of its own)
  finish_sorted<DT, THREADS>(p, row, g, to_workspace, cb, ci, m, SelResult{0ull, 0, m}, sort_mode, ctl, holes, ring,
                             ring_bytes, span_lo, span_len, off, need, crank == 0);
}

// Survivor bits of one thread in one round (up to 128 elements), kept in two
// registers; bit positions are run-time values, so no array indexing.
struct Keep128 {
  uint64_t w[2];
  __device__ __forceinline__ void set(int b) {
    if (b < 64) w[0] |= 1ull << b;
    else w[1] |= 1ull << (b - 64);
  }
  __device__ __forceinline__ void clr(int b) {
    if (b < 64) w[0] &= ~(1ull << b);
    else w[1] &= ~(1ull << (b - 64));
  }
  __device__ __forceinline__ int count() const { return __popcll(w[0]) + __popcll(w[1]); }
};

// ---------------------------------------------------------------------------
// Where this thread's vectors sit in the current round.  A warp owns one whole
// block per round (B = 32 lanes x VPT vectors); vector v of a lane is 16-byte
// slot v * 32 + lane of that block, at ring byte offset sb + v * 512, starting
// at row element eb + v * 32 * PV.
// ---------------------------------------------------------------------------
template <int DT>
struct WarpRound {
  static constexpr int PV = Elem<DT>::kPerVec;
  uint32_t sb;   // ring byte offset of the lane's first vector
  uint32_t eb;   // row element of the lane's first vector
  int j0;        // the owned block (visit order)
  bool owns;     // the block exists this round (warp-uniform)
  uint32_t uhi;  // end of this CTA's slice
  // Ring byte offset and first row element of vector v; false when the vector
  // lies past the slice end or the warp owns no block this round.
  __device__ __forceinline__ bool locate(int v, uint32_t& voff, uint32_t& eidx) const {
    if (!owns) return false;
    eidx = eb + static_cast<uint32_t>(v * 32 * PV);
    if (eidx >= uhi) return false;
    voff = sb + static_cast<uint32_t>(v * 512);
    return true;
  }
};

// Key of the largest element of a 16-byte vector; true (key unset) when the
// vector holds a NaN.
template <int DT>
__device__ __forceinline__ bool vec_max_key(const uint4 x, uint32_t& key) {
  using E = Elem<DT>;
  if (DT == DSEL_BF16) {
    const uint32_t m2 = bf16x2_max_nan(bf16x2_max_nan(x.x, x.y), bf16x2_max_nan(x.z, x.w));
    const uint32_t lo = m2 & 0xFFFFu, hi = m2 >> 16;
    if (E::is_nan(lo) || E::is_nan(hi)) return true;
    const uint32_t klo = E::key(lo), khi = E::key(hi);
    key = klo > khi ? klo : khi;
    return false;
  } else {
    const float a = __uint_as_float(x.x), b = __uint_as_float(x.y), c = __uint_as_float(x.z), d = __uint_as_float(x.w);
    if (a != a || b != b || c != c || d != d) return true;
    key = E::key(__float_as_uint(fmaxf(fmaxf(a, b), fmaxf(c, d))));
    return false;
  }
}

// A key t such that at least k of the CTA's non-empty group maxima (gm != 0)
// are >= t, close below the k-th largest of them; 0 when the CTA holds fewer
// than k.  One histogram pass: the maxima fall into 1024 bins spread evenly
// over [kmin, kmax] (bins of 2^sh keys, sh = 0 when the span is below 1024),
// and t is the lower edge of the bin that holds the k-th largest.  `hist` has
// 1024 zeroed ints, 16-byte aligned.  Two barriers; no warp reduction in a loop.
template <int THREADS, int G>
__device__ __forceinline__ uint32_t cta_kth_largest(const uint32_t (&gm)[G], int k, Ctl& ctl, int* hist) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  trace_mark(0);
  int nz = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gm[g] != 0u) {
      ++nz;
      kmin = min(kmin, gm[g]);
      kmax = max(kmax, gm[g]);
    }
  }
  nz = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nz)));
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    ctl.wm[warp] = nz;
    ctl.wv[warp] = (static_cast<unsigned long long>(kmax) << 32) | kmin;
  }
  __syncthreads();   // ctl.wm / wv are written again only after later barriers
  trace_mark(1);
  nz = 0;
  kmin = 0xFFFFFFFFu;
  kmax = 0u;
#pragma unroll
  for (int w = 0; w < NW; ++w) {   // every thread: the same loads
    nz += ctl.wm[w];
    const unsigned long long wv = ctl.wv[w];
    kmin = min(kmin, static_cast<uint32_t>(wv));
    kmax = max(kmax, static_cast<uint32_t>(wv >> 32));
  }
  trace_mark(2);
  if (nz < k) return 0u;   // uniform
  constexpr int NB = 1024;                  // bins
  constexpr int PER_LANE = NB / 32;
  const uint32_t span = kmax - kmin;
  const int sh = max(0, (32 - __clz(span)) - 10);   // (span >> sh) < NB
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (gm[g] != 0u) atomicAdd(&hist[(gm[g] - kmin) >> sh], 1);
  }
  trace_mark(3);
  __syncthreads();
  trace_mark(4);
  // every warp: lane l sums the PER_LANE consecutive bins below NB - 1 - l * PER_LANE
  const int top = NB - 1 - lane * PER_LANE;
  // lane l's bins are NB-32-32l .. NB-1-32l, int4s 8(31-l) .. 8(31-l)+7
  const int sum = chunk_sum4<PER_LANE / 4>(reinterpret_cast<const int4*>(hist), 0, 31 - lane);
  trace_mark(5);
  const int incl = warp_incl_scan(sum, lane);
  const bool mine = incl - sum < k && k <= incl;   // this lane's bins hold the k-th largest
  int bin = 0;
  if (mine) {   // walk down the lane's bins, four at a time
    int acc = incl - sum;
#pragma unroll 1
    for (int j = 0; j < PER_LANE; j += 4) {
      const int4 q = *reinterpret_cast<const int4*>(hist + top - j - 3);
      if (acc + q.w >= k) { bin = top - j; break; }
      if (acc + q.w + q.z >= k) { bin = top - j - 1; break; }
      if (acc + q.w + q.z + q.y >= k) { bin = top - j - 2; break; }
      acc += q.w + q.z + q.y + q.x;
      if (acc >= k) { bin = top - j - 3; break; }
    }
  }
  const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
  bin = __shfl_sync(0xffffffffu, bin, src);
  trace_mark(6);
  return kmin + (static_cast<uint32_t>(bin) << sh);
}

// ---------------------------------------------------------------------------
// Round-0 threshold seed (cold path, kept out of the per-round loop).  A
// histogram of the round's keys over the bits where they differ, refined once
// inside the chosen bin, gives the lower edge of a bin holding the k-th largest
// key: at least k of the round's elements (hence of the slice) are >= it, so it
// is a valid starting T.
// ---------------------------------------------------------------------------
struct SeedOut {
  unsigned long long t;
  uint64_t vlo;
  bool ok;
};

template <int DT, int THREADS, int VPT>
__device__ __noinline__ SeedOut seed_threshold(const unsigned char* ring, WarpRound<DT> wr, int k, int idx_bits,
                                               Ctl& ctl, int* seed_hist) {
  using E = Elem<DT>;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t uhi = wr.uhi;
  int nvalid = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
#pragma unroll 1
  for (int v = 0; v < VPT; ++v) {
    uint32_t voff, eidx;
    if (!wr.locate(v, voff, eidx)) continue;
    const uint4 val = *reinterpret_cast<const uint4*>(ring + voff);
#pragma unroll
    for (int e = 0; e < PV; ++e) {
      const uint32_t b = vec_elem<DT>(val, e);
      if (eidx + e < uhi && !E::is_nan(b)) {
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
    ctl.wm[warp] = nvalid;
    ctl.wv[warp] = (static_cast<unsigned long long>(kmax) << 32) | kmin;
  }
  __syncthreads();
  int tot_valid;
  warp_prefix_of<NW>(ctl.wm, warp, lane, tot_valid);
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
  // Level 1: the kSeedBits bits below the leading bits shared by gmin and gmax.
  // Level 2 (when bits remain): the next kSeedBits bits, inside level 1's bin.
  const int top = 32 - __clz(gmin ^ gmax);           // low bits in which keys differ
  uint32_t kbase = gmin & ~mask_bits(top);            // keys in the current bin share these bits
  int width = top;                                    // bits below kbase that still vary
  int need = k;
  constexpr int SLICE = kSeedBins / NW;
  constexpr int PER_LANE = SLICE / 32;
#pragma unroll 1
  for (int level = 0; level < 2; ++level) {           // uniform
    int* hist = seed_hist + level * kSeedBins;
    const int ws = width > kSeedBits ? width - kSeedBits : 0;
#pragma unroll 1
    for (int v = 0; v < VPT; ++v) {
      uint32_t voff, eidx;
      if (!wr.locate(v, voff, eidx)) continue;
      const uint4 val = *reinterpret_cast<const uint4*>(ring + voff);
#pragma unroll
      for (int e = 0; e < PV; ++e) {
        const uint32_t b = vec_elem<DT>(val, e);
        if (eidx + e < uhi && !E::is_nan(b)) {
          const uint32_t d = E::key(b) - kbase;
          if ((width >= 32) || d < (1u << width)) atomicAdd(&hist[d >> ws], 1);
        }
      }
    }
    __syncthreads();   // histogram complete; every warp is past its reads of wm
    // the bin holding the need-th largest: per-warp slice sums, then the slice
    const int sbase = kSeedBins - (warp + 1) * SLICE;  // warp 0 sums the top slice
    static_assert(PER_LANE % 4 == 0 && SLICE % 4 == 0, "slices are read as int4s");
    const int4* hist4 = reinterpret_cast<const int4*>(hist);
    int sl = chunk_sum4<PER_LANE / 4>(hist4, sbase / 4, lane);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
    if (lane == 0) ctl.wm[warp] = sl;
    __syncthreads();
    const int c = lane < NW ? ctl.wm[lane] : 0;
    const int incl = warp_incl_scan(c, lane);
    const bool mine = (incl - c) < need && need <= incl;
    const int slc = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    need -= __shfl_sync(0xffffffffu, incl - c, slc);
    const int b0 = kSeedBins - (slc + 1) * SLICE;
    // lane l: the PER_LANE bins below b0 + SLICE - 1 - l * PER_LANE (chunk 31 - l)
    const int sm = chunk_sum4<PER_LANE / 4>(hist4, b0 / 4, 31 - lane);
    const int inc2 = warp_incl_scan(sm, lane);
    const bool mine2 = (inc2 - sm) < need && need <= inc2;
    int bin = 0, above = 0;
    if (mine2) {   // one lane walks its bins from the top
      int acc = inc2 - sm;
#pragma unroll 1
      for (int j = 0; j < PER_LANE; ++j) {
        const int bj = b0 + SLICE - 1 - (lane * PER_LANE + j);
        const int cj = hist[bj];
        if (acc + cj >= need) {
          bin = bj;
          above = acc;
          break;
        }
        acc += cj;
      }
    }
    const int src2 = __ffs(__ballot_sync(0xffffffffu, mine2)) - 1;
    bin = __shfl_sync(0xffffffffu, bin, src2);
    need -= __shfl_sync(0xffffffffu, above, src2);
    kbase += static_cast<uint32_t>(bin) << ws;
    width = ws;
    if (ws == 0) break;
    __syncthreads();   // all warps have read wm before the next level writes it
  }
  // every key >= the final bin's lower edge passes, and at least k elements do
  out.t = make_w(kbase, 0xFFFFFFFFu);
  out.vlo = static_cast<uint64_t>(kbase) << idx_bits;
  out.ok = true;
  return out;
}

// ---------------------------------------------------------------------------
// Bulk copy of the j-th block in visiting order, (pa * j + pc) mod nb, of the
// slice [lo, hi) into ring stage jg mod D (jg: the CTA's running block count).  Out of line: it is called from the
// prologue and from every refill, and inlining would repeat its 64-bit modulo.
// ---------------------------------------------------------------------------
template <int DT>
__device__ __noinline__ void issue_block(int j, int jg, uint32_t pa, uint32_t pc, int nb, int64_t lo, int64_t hi,
                                         int D, const char* rowp, unsigned char* ring, uint64_t* bars,
                                         uint32_t* blk_off) {
  using E = Elem<DT>;
  constexpr int B = block_elems_for(E::kBytes);
  // pa, j mod nb and pc are below nb: 32-bit products while nb < 2^16
  const uint32_t jj = static_cast<uint32_t>(j) % static_cast<uint32_t>(nb);
  const uint32_t m = nb < 65536 ? (pa * jj + pc) % static_cast<uint32_t>(nb)
                                : static_cast<uint32_t>((static_cast<uint64_t>(pa) * jj + pc) %
                                                        static_cast<uint32_t>(nb));
  const int64_t e0 = lo + static_cast<int64_t>(m) * B;
  const int64_t ce = min(static_cast<int64_t>(B), hi - e0);
  const uint32_t bytes = static_cast<uint32_t>((ce * E::kBytes + 15) & ~static_cast<int64_t>(15));
  const int s = jg % D;   // jg counts every block this CTA has issued: stages and phases run on
  blk_off[s] = static_cast<uint32_t>(e0);
  const uint32_t bar = smem_u32(&bars[s]);
  mbar_expect_tx(bar, bytes);
  bulk_g2s(smem_u32(ring + static_cast<size_t>(s) * B * E::kBytes), rowp + e0 * E::kBytes, bytes, bar);
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
__global__ void __launch_bounds__(THREADS, kThreads / THREADS) topk_stream_kernel(const __grid_constant__ KParams p) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  constexpr int B = block_elems_for(E::kBytes);       // elements per block: one warp's share of a round
  constexpr int R = round_elems_for(E::kBytes, THREADS);   // elements per round
  constexpr int Q = R / B;                             // blocks per round: one per warp
  constexpr int VPT = R / (THREADS * PV);              // vectors per thread per round
  static_assert(Q == NW && VPT * 32 * PV == B && VPT * THREADS * PV == R, "round shape");
  static_assert(VPT <= 32, "screen flags fit one 32-bit mask");
  constexpr int SG = THREADS == kThreads ? 4 : 8;      // round-0 seed: group maxima per thread
  constexpr int VPG = VPT / SG;                        // vectors per group
  static_assert(VPG * SG == VPT, "seed groups");
  static_assert(VPT * PV <= 128 && 64 % PV == 0, "keep bits fit two 64-bit words, vectors not straddling");
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
  if (blockIdx.x == g_trace_cta && threadIdx.x == 0) g_trace[(kTraceRounds - 1) * kTraceEvents + kTraceEvents - 1] = st_t0;
  long long st_t1 = st_t0;
  int st_rounds = 0;
  long long st_ev[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  long long st_wait = 0;
#define DSEL_EV(i) do { if (tid == 0) st_ev[i] = clock64() - st_t0; } while (0)
  const int tr_w = (blockIdx.x == g_trace_cta && lane == 0 && warp < kTraceWarps) ? warp : -1;
#define DSEL_TR(r, e) do { if (tr_w >= 0 && (r) < kTraceRounds - 2) \
    g_trace[(tr_w * kTraceRounds + (r)) * kTraceEvents + (e)] = clock64() - st_t0; } while (0)
#else
#define DSEL_EV(i) do { } while (0)
#define DSEL_TR(r, e) do { } while (0)
#endif

#pragma unroll 1
  for (int i = tid; i < 3 * kBins; i += THREADS) (&ctl.hist[0][0])[i] = 0;
  {   // round-0 seed histograms: two levels of kSeedBins for large k, else 1024 bins
    static_assert(2 * kSeedBins <= kSeedSlots, "seed histograms fit the index array");
    const int nz = 2 * p.k > SG * THREADS ? 2 * kSeedBins : 1024;
#pragma unroll 1
    for (int i = tid; i < nz; i += THREADS) seed_hist[i] = 0;
  }
  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.add[0] = ctl.add[1] = ctl.add[2] = 0;
    ctl.nan_found = 0;
    ctl.abort = 0;
    ctl.hb = 0;
#ifdef DSEL_STATS
    ctl.st_compact_cycles = 0;
    ctl.st_compactions = 0;
    ctl.st_appended = 0;
    ctl.st_slow_vectors = 0;
    ctl.st_refetch = 0;
#endif
  }
#pragma unroll 1
  for (int s = tid; s < D; s += THREADS) {   // each thread fences the barriers it initialised
    mbar_init(smem_u32(&bars[s]), 1);
    fence_mbar_init();
  }
  if (C > 1) cluster.sync();   // peers' control blocks are ready before anyone touches them remotely
  else __syncthreads();
  DSEL_EV(0);
  // the set-up above touched shared memory only: it may overlap the previous launch
  grid_dependency_wait();
  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);

  const bool leader = (g == 0 && crank == 0);
  if (bad_end || n <= p.k) {
    if (p.groups == 1 && leader) {
      if (bad_end) write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_BAD_END);
      else finish_short_row<DT, THREADS>(p, row, n, cb, ci, ctl);
    }
  } else {
    // ---- this CTA's slice: [lo, hi), a multiple of 16 elements wide ----
    const int S = p.groups * C;
    const int sid = g * C + crank;
    // 32-bit arithmetic: n <= row_stride <= INT32_MAX (64-bit division is a software routine)
    const int64_t slice = static_cast<int64_t>(((static_cast<uint32_t>(n) + static_cast<uint32_t>(S) - 1u) /
                                                    static_cast<uint32_t>(S) + 15u) / 16u * 16u);
    const int64_t lo = min(n, static_cast<int64_t>(sid) * slice);
    const int64_t hi = min(n, lo + slice);
    const int nb = static_cast<int>((hi - lo + B - 1) / B);
    const char* rowp = static_cast<const char*>(p.x) + row * p.row_stride * E::kBytes;

    // ---- block visiting order: j -> (pa * j + pc) mod nb, pa coprime with nb ----
    uint32_t pa = 1, pc = 0;
    if (nb > 1) {
      const uint32_t unb = static_cast<uint32_t>(nb);
      pa = (unb < 6000000u ? (unb * 618u + 500u) / 1000u
                           : static_cast<uint32_t>((static_cast<uint64_t>(unb) * 618u + 500u) / 1000u)) | 1u;
#pragma unroll 1
      for (;;) {
        uint32_t a = pa, b = unb;
        while (b) { const uint32_t t = a % b; a = b; b = t; }
        if (a == 1u) break;
        pa += 2u;
      }
      pa %= unb;
      const uint64_t h = (static_cast<uint64_t>(row) + 1) * 0x9E3779B97F4A7C15ull ^
                         (static_cast<uint64_t>(sid) + 1) * 0xBF58476D1CE4E5B9ull;
      pc = static_cast<uint32_t>(h >> 29) % unb;   // the low 32 bits of h >> 29
    }
    int jb = 0;   // blocks issued in earlier passes over the slice
    auto issue = [&](int j) {
      issue_block<DT>(j, jb + j, pa, pc, nb, lo, hi, D, rowp, ring, bars, blk_off);
    };

    const uint32_t uhi = static_cast<uint32_t>(hi);
    const uint32_t idx_mask = mask_bits(p.idx_bits);
    const int cap = p.capacity;
    uint64_t vmax = 0;             // largest radix word this thread kept
    uint64_t vlo = 0;              // every candidate's radix word is >= vlo
    unsigned long long t_own = 0;  // this CTA's threshold word
    int cnt = 0;                   // candidates in the buffer (same value in every thread)
    int par = 0;                   // which of the two per-warp count arrays is next
    bool nan_thread = false;
    // cut the buffer back to k..k+slack, raise T and tell the peers (all threads)
    auto compact = [&](int slack) {
      const CompactOut co = compact_buffer<DT, THREADS>(cb, ci, holes, ctl, cluster, cnt, p.k, slack, p.idx_bits,
                                                        vmax, vlo);
      cnt = co.cnt;
      t_own = co.tw > t_own ? co.tw : t_own;
      vlo = co.vlo;
      // any CTA's threshold is a valid bound for the whole row: push it to the peers
      if (C > 1 && warp == 0 && lane < C && lane != crank) atomicMax(cluster.map_shared_rank(&ctl.t_w, lane), co.tw);
    };
    // every CTA runs round 0, even on an empty slice: the cluster meets there
    const int rounds = max(1, (nb + Q - 1) / Q);
    int rg = 0;              // rounds run so far over all passes (per-round counters rotate on it)
    bool spec = false;       // round 0 seeded T from a sample: certified at the end of the pass
    bool compacted = false;  // a compaction ran in this pass
#pragma unroll 1
    for (int pass = 0;; ++pass) {
    {   // prologue: the pass's first D blocks, each issued by lane 0 of the warp that owns its stage
      if (pass > 0) {   // the previous pass's reads of the ring come before these copies
        __syncthreads();
      }
      const int first = min(D, nb);
#pragma unroll 1
      for (int j = warp; j < first; j += Q) {
        if (lane == 0) {
          if (pass > 0) fence_proxy_async();
          issue(j);
        }
      }
    }
    DSEL_EV(1);
#pragma unroll 1
    for (int r = 0; r < rounds; ++r, ++rg) {
      DSEL_TR(r, 0);
      WarpRound<DT> wr;
      wr.j0 = r * Q + warp;                            // the block this warp owns in the round
      wr.owns = wr.j0 < nb;
      wr.uhi = uhi;
      wr.sb = 0u;
      wr.eb = 0u;
      const int j0 = wr.j0;
      // ---- 1. wait for the owned block ----
      if (wr.owns) {   // warp-uniform
        const int jg = jb + j0;
        const int st = jg % D;
#ifdef DSEL_STATS
        const long long w0 = clock64();
#endif
        if (!mbar_wait(smem_u32(&bars[st]), static_cast<uint32_t>((jg / D) & 1))) ctl.abort = 1;
#ifdef DSEL_STATS
        st_wait += clock64() - w0;
#endif
        wr.sb = static_cast<uint32_t>(st * B * E::kBytes + lane * 16);
        wr.eb = blk_off[st] + static_cast<uint32_t>(lane * PV);
      }
      DSEL_TR(r, 8);
      unsigned long long w = *reinterpret_cast<volatile unsigned long long*>(&ctl.t_w);
      w = w > t_own ? w : t_own;   // a peer may have raised it
      uint32_t tk, ti;
      uint32_t maybe_mask = 0;     // bit v: vector v may hold a survivor (or a NaN)
      if (r == 0) {
        // ---- 2a. round 0: one pass for each vector's largest key, seed T from
        //      those maxima, and screen with them (no second read) ----
        // gk[v]: largest key of vector v (0 = none: partial and NaN vectors are
        // left out and always tested exactly); gm[g]: largest of group g's keys
        uint32_t gk[VPT], gm[SG];
        uint32_t forced = 0u, valid = 0u;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          gk[v] = 0u;
          const uint32_t eidx = wr.eb + static_cast<uint32_t>(v * 32 * PV);
          if (wr.owns && eidx < uhi) {
            valid |= 1u << v;
            const uint4 val = *reinterpret_cast<const uint4*>(ring + wr.sb + v * 512);
            uint32_t kx = 0u;
            if (vec_max_key<DT>(val, kx) || eidx + PV > uhi) forced |= 1u << v;
            else gk[v] = kx;
          }
        }
#pragma unroll
        for (int g = 0; g < SG; ++g) {
          uint32_t m = 0u;
#pragma unroll
          for (int i = 0; i < VPG; ++i) m = max(m, gk[g * VPG + i]);
          gm[g] = m;
        }
        DSEL_TR(r, 1);
        SeedOut so{0ull, 0ull, false};
        // Sampled seed: when this CTA streams a whole row in several rounds, the
        // round's blocks (visited in random order) are a random sample of the row;
        // T goes near the expected number of the row's top k in it, plus a wide
        // margin (6 standard deviations).  It is certified after the pass.
        int kseed = p.k;
        if (pass == 0 && C == 1 && p.groups == 1 && rounds > 1) {
          const float n_sl = static_cast<float>(hi - lo);
          const float m0 = fminf(n_sl, static_cast<float>(R));
          const float e = static_cast<float>(p.k) * m0 / n_sl;
          const int j = static_cast<int>(ceilf(e + 6.0f * sqrtf(e) + 16.0f));
          if (j < p.k) {
            kseed = j;
            spec = true;
          }
        }
        if (pass > 0) {   // the histograms still hold the previous pass's seed
#pragma unroll 1
          for (int i = tid; i < 2 * kSeedBins; i += THREADS) seed_hist[i] = 0;
          __syncthreads();
        }
        if (2 * kseed <= SG * THREADS) {
          // the kseed-th largest group maximum: kseed distinct elements are at or above it
          const uint32_t tkey = cta_kth_largest<THREADS, SG>(gm, kseed, ctl, seed_hist);
          if (tkey != 0u) {   // uniform
            so.t = make_w(tkey, 0xFFFFFFFFu);     // passes every key >= tkey
            so.vlo = static_cast<uint64_t>(tkey) << p.idx_bits;
            so.ok = true;
          } else {
            // fewer than k group maxima (a short slice): seed from the elements
            // themselves rather than start at -inf and take the whole slice in
#pragma unroll 1
            for (int i = tid; i < 2 * kSeedBins; i += THREADS) seed_hist[i] = 0;
            __syncthreads();
            so = seed_threshold<DT, THREADS, VPT>(ring, wr, kseed, p.idx_bits, ctl, seed_hist);
          }
        } else {
          so = seed_threshold<DT, THREADS, VPT>(ring, wr, kseed, p.idx_bits, ctl, seed_hist);
        }
        spec = spec && so.ok;
        DSEL_TR(r, 9);
        if (so.ok) {
          t_own = so.t;
          vlo = so.vlo;
          w = so.t > w ? so.t : w;
        }
        if (C > 1) {
          // every CTA's seed bounds the whole row: share them, so that a slice of
          // low values screens against its neighbours' higher threshold
          if (so.ok && warp == 0 && lane < C && lane != crank)
            atomicMax(cluster.map_shared_rank(&ctl.t_w, lane), so.t);
          cluster.sync();
          const unsigned long long wp = *reinterpret_cast<volatile unsigned long long*>(&ctl.t_w);
          w = wp > w ? wp : w;
        }
        tk = static_cast<uint32_t>(w >> 32);
        ti = ~static_cast<uint32_t>(w);
        // a vector whose largest key is below T's key holds no survivor
        maybe_mask = forced;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
          if (gk[v] >= tk && gk[v] != 0u) maybe_mask |= 1u << v;
        }
      } else {
        // ---- 2b. later rounds: screen every vector against T ----
        tk = static_cast<uint32_t>(w >> 32);
        ti = ~static_cast<uint32_t>(w);
        uint32_t tv = E::bits_of_key(tk);
        if (DT == DSEL_BF16) tv |= tv << 16;
#pragma unroll 2
        for (int v = 0; v < VPT; ++v) {
          const uint32_t eidx = wr.eb + static_cast<uint32_t>(v * 32 * PV);
          if (wr.owns && eidx < uhi) {
            const uint4 val = *reinterpret_cast<const uint4*>(ring + wr.sb + v * 512);
            if ((eidx + PV > uhi) || screen<DT>(val, tv)) maybe_mask |= 1u << v;
          }
        }
        DSEL_TR(r, 1);
      }
      uint32_t tv = E::bits_of_key(tk);
      if (DT == DSEL_BF16) tv |= tv << 16;

      DSEL_TR(r, 7);

      // ---- 3. exact test of the flagged vectors, appended at once: per batch of
      //      one vector per lane, the warp reserves slots with one shared atomic
      //      on this round's counter; survivors past the buffer's end wait ----
      const int radd = rg % 3;
      if (tid == 0) ctl.add[(rg + 1) % 3] = 0;   // last read before the previous round's barrier
      Keep128 pend;            // survivors of this thread: bit v*PV + e
      pend.w[0] = pend.w[1] = 0ull;
      {
#ifdef DSEL_STATS
        if (lane == 0) atomicAdd(&ctl.st_slow_vectors, __popc(maybe_mask));
#endif
        uint32_t mm = maybe_mask;   // flagged vectors lie inside the slice
#pragma unroll 1
        while (mm) {
          const int v = __ffs(mm) - 1;
          mm &= mm - 1u;
          const uint32_t eidx = wr.eb + static_cast<uint32_t>(v * 32 * PV);
          const uint4 val = *reinterpret_cast<const uint4*>(ring + wr.sb + v * 512);
          const uint32_t lim = uhi - eidx;   // elements of the vector inside the slice
          uint32_t kb = 0u;
          bool nanv = false;
#pragma unroll
          for (int e = 0; e < PV; ++e) {   // straight-line: no per-element loop
            const uint32_t b = vec_elem<DT>(val, e);
            const bool in = static_cast<uint32_t>(e) < lim;
            const bool isn = E::is_nan(b);
            const uint32_t kk = E::key(b);
            const bool pass = kk > tk || (kk == tk && eidx + e < ti);
            kb |= (in && !isn && pass) ? (1u << e) : 0u;
            nanv |= in && isn;
          }
          if (nanv) {
            if (!p.nan_flag) nan_trap();   // the pages' default policy: abort on NaN
            nan_thread = true;
          }
          const int bit = v * PV;          // a vector's bits never straddle the two words
          if (bit < 64) pend.w[0] |= static_cast<uint64_t>(kb) << bit;
          else pend.w[1] |= static_cast<uint64_t>(kb) << (bit - 64);
        }
        DSEL_TR(r, 6);
        // one reservation per warp for the round: a scan and one shared atomic
        const int mine = pend.count();
        const int incl = warp_incl_scan(mine, lane);
        const int wtot = __shfl_sync(0xffffffffu, incl, 31);
        if (wtot != 0) {   // warp-uniform
          int base = 0;
          if (lane == 0) base = atomicAdd(&ctl.add[radd], wtot);
          int pos = cnt + __shfl_sync(0xffffffffu, base, 0) + incl - mine;
#pragma unroll
          for (int wi = 0; wi < 2; ++wi) {
            uint64_t kb = pend.w[wi];
            while (kb && pos < cap) {   // slots past the buffer's end: the survivor waits
              const int bit = wi * 64 + __ffsll(static_cast<long long>(kb)) - 1;
              kb &= kb - 1ull;
              const int v = bit / PV, e = bit % PV;
              const uint32_t eidx = wr.eb + static_cast<uint32_t>(v * 32 * PV);
              const uint4 val = *reinterpret_cast<const uint4*>(ring + wr.sb + v * 512);
              const uint32_t bv = vec_elem_dyn<DT>(val, e);
              cb[pos] = static_cast<bits_t>(bv);
              ci[pos] = eidx + e;
              const uint64_t vv = (static_cast<uint64_t>(E::key(bv)) << p.idx_bits) | (idx_mask - (eidx + e));
              vmax = vv > vmax ? vv : vmax;   // largest radix word this thread wrote
              pend.clr(bit);
              ++pos;
            }
          }
        }
      }
      if (r == 0) DSEL_EV(2);
      DSEL_TR(r, 2);

      // ---- 4. the round's count (uniform after the barrier) ----
      const bool my_pend = (pend.w[0] | pend.w[1]) != 0ull;
      const bool warp_pend = __any_sync(0xffffffffu, my_pend);
      // ---- 5. refill this warp's stage (no other warp reads it), unless waiting
      //      survivors of the warp still have to be read from it ----
      auto refill = [&]() {
        __syncwarp();
        if (lane == 0) {
          fence_proxy_async();   // our reads of the stage come before the copy that overwrites it
          if (j0 + D < nb) issue(j0 + D);
        }
      };
      if (!warp_pend) refill();
      const bool any_pend = __syncthreads_or(my_pend) != 0;
      const int added = ctl.add[radd];
      if (r == 0) DSEL_EV(3);
      DSEL_TR(r, 3);
#ifdef DSEL_STATS
      if (tid == 0) ctl.st_appended += min(added, cap - cnt);
#endif
      if (!any_pend) {   // uniform
        cnt += added;
      } else {
        // rare: the buffer filled up; compact it, raise T, re-test the waiting
        // survivors and append them at offsets from per-warp counts
        cnt = cap;
        while (true) {   // uniform
          compact(p.b2 / 2);
          compacted = true;
          unsigned long long w2 = *reinterpret_cast<volatile unsigned long long*>(&ctl.t_w);
          w2 = w2 > t_own ? w2 : t_own;
          tk = static_cast<uint32_t>(w2 >> 32);
          ti = ~static_cast<uint32_t>(w2);
          int mine = 0;
#pragma unroll
          for (int wi = 0; wi < 2; ++wi) {
            uint64_t kb = pend.w[wi];
            while (kb) {
              const int bit = wi * 64 + __ffsll(static_cast<long long>(kb)) - 1;
              kb &= kb - 1ull;
              const int v = bit / PV, e = bit % PV;
              uint32_t voff, eidx;
              wr.locate(v, voff, eidx);
              const uint4 val = *reinterpret_cast<const uint4*>(ring + voff);
              const uint32_t kk = E::key(vec_elem_dyn<DT>(val, e));
              if (!(kk > tk || (kk == tk && eidx + e < ti))) pend.clr(bit);
              else ++mine;
            }
          }
          const int wcount = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(mine)));
          if (lane == 0) ctl.wc[par][warp] = wcount;
          __syncthreads();
          int total;
          const int woff = warp_prefix_of<NW>(ctl.wc[par], warp, lane, total);
          par ^= 1;
          const int space = cap - cnt;
          if (wcount != 0) {   // warp-uniform
            int rank = woff + warp_incl_scan(mine, lane) - mine;
#pragma unroll
            for (int wi = 0; wi < 2; ++wi) {
              uint64_t kb = pend.w[wi];
              while (kb) {
                const int bit = wi * 64 + __ffsll(static_cast<long long>(kb)) - 1;
                kb &= kb - 1ull;
                if (rank < space) {
                  const int v = bit / PV, e = bit % PV;
                  uint32_t voff, eidx;
                  wr.locate(v, voff, eidx);
                  const uint4 val = *reinterpret_cast<const uint4*>(ring + voff);
                  const uint32_t bv = vec_elem_dyn<DT>(val, e);
                  cb[cnt + rank] = static_cast<bits_t>(bv);
                  ci[cnt + rank] = eidx + e;
                  const uint64_t vv = (static_cast<uint64_t>(E::key(bv)) << p.idx_bits) | (idx_mask - (eidx + e));
                  vmax = vv > vmax ? vv : vmax;
                  pend.clr(bit);
                }
                ++rank;
              }
            }
          }
          if (total <= space) {
            cnt += total;
            break;
          }
          cnt = cap;
        }
        if (warp_pend) refill();
      }
      DSEL_TR(r, 4);
#ifdef DSEL_STATS
      ++st_rounds;
#endif
      // ---- 6. cut the buffer back when it holds k + B2 ----
      if (cnt >= p.k + p.b2) {   // uniform: cnt is the same register value everywhere
#ifdef DSEL_STATS
        const long long sc0 = clock64();
#endif
        compact(p.b2 / 2);
        compacted = true;
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
    // A sampled threshold holds only if at least k elements reached it; a
    // compaction proves that (it runs at k + B2 candidates).  Otherwise stream
    // the slice again with a proven seed (all values uniform in the CTA).
    if (!(spec && !compacted && cnt < p.k) || ctl.abort) break;
#ifdef DSEL_STATS
    if (tid == 0) ctl.st_refetch += 1;
#endif
    jb += nb;
    spec = false;
    compacted = false;
    cnt = 0;
    t_own = 0ull;
    vlo = 0ull;
    vmax = 0ull;
    }
    // A wait that gave up may leave a copy in flight: wait for it (bounded) before
    // this CTA's shared memory can go away.
    __syncthreads();
    if (ctl.abort && tid == 0) {
#pragma unroll 1
      for (int j = max(0, nb - D); j < nb; ++j) mbar_wait(smem_u32(&bars[(jb + j) % D]), ((jb + j) / D) & 1);
    }
#ifdef DSEL_STATS
    st_t1 = clock64();
#endif
    DSEL_EV(5);
    grid_launch_dependents();   // the next launch may start its prologue during the final phase

    const bool to_ws = p.groups > 1;
    const int sort_mode = to_ws ? (p.order == DSEL_ORDER_INDEX ? 1 : 0) : p.order;
    // index span of the candidates this CTA orders: its slice, or the cluster's
    // slices when rank 0 gathers them
    const bool cl_span = C > 1 && p.gather;
    const int64_t span_a = cl_span ? min(n, static_cast<int64_t>(g * C) * slice) : lo;
    const int64_t span_b = cl_span ? min(n, static_cast<int64_t>(g * C + C) * slice) : hi;
    finalize<DT, THREADS>(p, row, g, cb, ci, holes, ctl, cluster, cnt, nan_thread, vlo, vmax, to_ws, sort_mode,
                          ring, static_cast<uint32_t>(D * B * E::kBytes), static_cast<uint32_t>(span_a),
                          static_cast<uint32_t>(span_b - span_a));
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
    st[7] = static_cast<unsigned long long>(ctl.st_refetch);
#pragma unroll 1
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

#pragma unroll 1
  for (int i = tid; i < 3 * kBins; i += THREADS) (&ctl.hist[0][0])[i] = 0;
  if (tid == 0) {
    ctl.t_w = 0ull;
    ctl.nan_found = 0;
    ctl.abort = 0;
    ctl.hb = 0;
  }
  if (C > 1) cluster.sync();
  else __syncthreads();
  grid_dependency_wait();   // the streaming launch's workspace is complete and visible
  bool bad_end;
  const int64_t n = row_length(p, row, &bad_end);
  if (bad_end || n <= p.k) {
    if (crank == 0) {
      if (bad_end) write_sentinel_row<DT, THREADS>(p, row, DSEL_IDX_BAD_END);
      else finish_short_row<DT, THREADS>(p, row, n, cb, ci, ctl);
    }
  } else {
    // group prefix sums (groups <= kBins) in the histogram scratch
    int* pref = ctl.hsum;
    const int2* meta = p.ws_meta + row * p.groups;
    if (tid == 0) {
      int acc = 0, nan = 0;
#pragma unroll 1
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
#pragma unroll 1
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
                          p.order, nullptr, 0u, 0u, 0u);
  }
  if (C > 1) cluster.sync();
}

}  // namespace dsel
