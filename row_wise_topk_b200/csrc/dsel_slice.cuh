// Slice-resident TopK: the rows of a batch are cut into slices that fit in shared
// memory, one CTA per slice, and the slices of one row form a thread-block
// cluster whose rank-0 CTA leads.  Every CTA loads its whole slice with bulk
// copies (all in flight at once), so the row is read exactly once.  The method is
// the threshold filter of "DeepSeek releases DeepSelect, a TopK kernel for sparse
// attention and sampling" (method paragraph), laid out for the order in which the
// data lands:
//
//   A. threshold from a sample: the chunks are visited in a per-slice
//      pseudo-random order, and the first ns to arrive are a random sample of the
//      slice.  Either every CTA takes T_c, a lower edge of the k-th largest vector
//      maximum of its own sample (k vectors hold an element >= T_c: a valid
//      threshold for the whole row, found with no cluster barrier), or, when that
//      would let too many candidates through, the CTAs take the k'-th largest,
//      k' = ceil(k / C), and the cluster uses T = min_c T_c (C slices with k'
//      such vectors each: again at least k), one cluster barrier;
//   B. filter: every chunk, as it lands, is screened against T (one packed
//      compare per 16-byte vector); the survivors go straight into the leader's
//      candidate list through distributed shared memory;
//   C. exact finish, by the leader alone after one cluster barrier (the other
//      CTAs leave): histogram levels over the candidates' keys and a ranking of the
//      boundary bin's members by (key, index) give the composite boundary (K*, I*),
//      the k-th entry of the row in the order value descending, index ascending.
//      An entry is selected when (key, index) ranks at or before (K*, I*); index
//      order comes from a bitmap of the row.
//
// When the list overflows an exact fallback runs on the resident slices (every
// CTA): histogram levels down to a single key, then ranks in index order from
// bitmaps.  The code runs once per launch, so every instruction it executes is
// fetched cold: loops stay rolled, and bin searches run in one warp (the others
// wait at a barrier) instead of every warp reading the whole histogram.  No wait
// depends on another CTA except the hardware cluster barriers; the bulk-copy
// waits are bounded.
#pragma once

#include "dsel_resident.cuh"

namespace dsel {

constexpr int kSlBins = 1024;
constexpr int kSlMembers = 256;   // boundary members ranked directly
constexpr int kSlChunk = kSliceThreads * kVecBytes;   // bytes per chunk: one vector per thread

struct __align__(16) SliceCtl {
  uint32_t w_a[kWarpsMax];
  uint32_t w_b[kWarpsMax];
  int w_c[kWarpsMax];
  int bin, before, cnt;      // a bin search, broadcast to the CTA
  uint32_t t_key;            // this slice's threshold, broadcast to the CTA
  int m_n;                   // boundary members collected in m_w
  uint32_t kstar, istar;
  int flags;                 // bit 0: NaN seen, bit 1: list overflow, bit 2: a wait gave up
  // the leader's copy is updated by every CTA of the cluster (remote atomics)
  uint32_t t_max;            // largest slice threshold (each one valid alone)
  uint32_t t_min;            // smallest slice threshold (each valid for k / C)
  uint32_t top;              // largest sampled key
  uint32_t kmax;             // largest key of the row
  // read by the peers in the exact fallback
  int x_sel;
  int x_cnt;
  uint32_t x_istar;
  int segcnt[kSliceMaxCluster * (kSliceThreads / 32)];   // entries of each (slice, warp) list segment
  unsigned long long m_w[kSlMembers];   // boundary members (key << 32 | ~index)
};

// Phase timestamps of thread 0 (%globaltimer, ns) in counter builds only:
// g_stats[cta][i] for i = 0..15.
__device__ __forceinline__ void sl_mark(int i) {
#ifdef DSEL_STATS
  if (threadIdx.x == 0 && blockIdx.x < kStatsCtas) g_stats[blockIdx.x * kStatsFields + i] = global_ns();
#else
  (void)i;
#endif
}

template <bool CLUSTER>
__device__ __forceinline__ void sl_sync(cg::cluster_group& cluster) {
  if (CLUSTER) cluster.sync();
  else __syncthreads();
}

// Split cluster barrier: arrive (release) early, wait (acquire) only where the
// ordering is needed.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// 16-bit summary of a key kept per sampled vector: the key itself for bfloat16,
// its top 16 bits for float32 (so summary >= key16(t) is a superset test for
// key >= t).
template <int DT>
__device__ __forceinline__ uint32_t key16(uint32_t key) {
  return DT == DSEL_BF16 ? key : (key >> 16);
}

// Largest key of the first `valid` elements of a vector (all of them when valid
// >= PV); true on a NaN among them.
template <int DT>
__device__ __forceinline__ bool vec_max_valid(const uint4& x, int valid, uint32_t& key) {
  using E = Elem<DT>;
  if (valid >= E::kPerVec) return vec_max_key<DT>(x, key);
  uint32_t m = 0u;
  bool nan = false;
#pragma unroll 1
  for (int e = 0; e < valid; ++e) {
    const uint32_t b = vec_elem_dyn<DT>(x, e);
    nan |= E::is_nan(b);
    m = max(m, E::key(b));
  }
  key = m;
  return nan;
}

// Sum over the cluster of a 1024-bin histogram into `hs` (every CTA holds the
// same sum afterwards); the caller has made every peer's histogram complete with
// a cluster barrier.  Ends with a CTA barrier.
template <int THREADS>
__device__ __forceinline__ void cluster_hist_sum(const int* h, int* hs, int C, cg::cluster_group& cluster) {
#pragma unroll 1
  for (int b = threadIdx.x; b < kSlBins; b += THREADS) {
    int sum = 0;
#pragma unroll 4
    for (int r = 0; r < C; ++r) sum += cluster.map_shared_rank(h, r)[b];
    hs[b] = sum;
  }
  __syncthreads();
}

// Exclusive prefix over the cluster's slices of a per-slice count published in
// ctl.x_*: the caller has passed a cluster barrier after publishing it.
__device__ __forceinline__ int slices_before(const SliceCtl& ctl, const int SliceCtl::*field, int crank,
                                             cg::cluster_group& cluster, int lane) {
  const int v = lane < crank ? cluster.map_shared_rank(&ctl, lane)->*field : 0;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(v)));
}

// Bitmap rank over a slice: bm holds `words` 32-bit words (bit i = element i);
// after the caller has set its bits and passed a CTA barrier, pre[w] receives the
// number of set bits in words before w.  Returns the total.  Two CTA barriers.
template <int THREADS>
__device__ __noinline__ int bitmap_prefix(const uint32_t* bm, uint32_t* pre, int words, SliceCtl& ctl) {
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (words + THREADS - 1) / THREADS;
  const int a = min(words, tid * per), b = min(words, a + per);
  int s = 0;
#pragma unroll 1
  for (int w = a; w < b; ++w) s += __popc(bm[w]);
  const int incl = warp_incl_scan(s, lane);
  if (lane == 31) ctl.w_c[warp] = incl;
  __syncthreads();
  int total;
  int run = warp_prefix_of<NW>(ctl.w_c, warp, lane, total) + incl - s;
#pragma unroll 1
  for (int w = a; w < b; ++w) {
    pre[w] = static_cast<uint32_t>(run);
    run += __popc(bm[w]);
  }
  __syncthreads();
  return total;
}

__device__ __forceinline__ int bitmap_rank(const uint32_t* bm, const uint32_t* pre, uint32_t i) {
  return static_cast<int>(pre[i >> 5]) + __popc(bm[i >> 5] & ((1u << (i & 31u)) - 1u));
}

// Bitmap rank over a whole row with a coarse prefix: bp[b] = set bits in the
// blocks of 32 words before block b.  After the bits are set and a CTA barrier;
// two CTA barriers.  Returns the total.
template <int THREADS>
__device__ __noinline__ int row_bitmap_prefix(const uint32_t* bm, int* bp, int words, SliceCtl& ctl) {
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int blocks = (words + 31) / 32;
#pragma unroll 1
  for (int b = warp; b < blocks; b += NW) {   // one warp per block: its total
    const int w = b * 32 + lane;
    const int c = static_cast<int>(__reduce_add_sync(0xffffffffu, w < words ? __popc(bm[w]) : 0u));
    if (lane == 0) bp[b] = c;
  }
  __syncthreads();
  if (warp == 0) {   // exclusive scan of the block totals, 32 blocks at a time
    int run = 0;
#pragma unroll 1
    for (int b0 = 0; b0 < blocks; b0 += 32) {
      const int b = b0 + lane;
      const int c = b < blocks ? bp[b] : 0;
      const int incl = warp_incl_scan(c, lane);
      if (b < blocks) bp[b] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) ctl.w_c[0] = run;
  }
  __syncthreads();
  return ctl.w_c[0];
}

__device__ __forceinline__ int row_bitmap_rank(const uint32_t* bm, const int* bp, uint32_t i) {
  int r = bp[i >> 10];
#pragma unroll 1
  for (uint32_t w = (i >> 10) << 5; w < (i >> 5); ++w) r += __popc(bm[w]);
  return r + __popc(bm[i >> 5] & ((1u << (i & 31u)) - 1u));
}

// Everything a CTA of the slice kernel knows about its slice.
struct SliceGeom {
  int64_t row;
  uint32_t lo, n_sl;   // first row element of the slice, its length
  uint32_t n;          // the row's length
  int nch;             // chunks (the last one may be partial)
  int C, crank;
};

// Exact fallback on the resident slice: histogram levels over the keys >= lo_k
// down to a single key K*, then the ties at K* and the selected entries ranked in
// index order through bitmaps.  Runs on every CTA of the cluster together.
template <int DT, int THREADS, bool CLUSTER>
__device__ __noinline__ void slice_exact(const KParams& p, unsigned char* smem, const SliceGeom& g, uint32_t lo_k,
                                         uint32_t kmax_row, cg::cluster_group& cluster) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int PV = E::kPerVec;
  const int tid = threadIdx.x, lane = tid & 31;
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);
  SliceCtl& ctl = *reinterpret_cast<SliceCtl*>(smem + p.off_ctl);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + p.off_tab);   // bitmap, then its prefix
  const int words = static_cast<int>((g.n_sl + 31u) / 32u);
  uint32_t* pre = bm + words;
  const int k = p.k;
  auto load_vec = [&](int c) -> uint4 {
    return *reinterpret_cast<const uint4*>(smem + static_cast<size_t>(c) * kSlChunk + tid * kVecBytes);
  };
  auto valid_of = [&](int c) -> int { return static_cast<int>(g.n_sl) - (c * THREADS + tid) * PV; };

  // the peers may still read this CTA's histograms and list: meet first, then clear
  sl_sync<CLUSTER>(cluster);
#pragma unroll 1
  for (int i = tid; i < 3 * kSlBins / 4; i += THREADS) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  __syncthreads();

  // ---- levels: [lo_k, hi_k] holds the k-th largest key ----
  uint32_t hi_k = kmax_row;
  int need = k;
  int eq_total = 0;
#pragma unroll 1
  for (int level = 0;; ++level) {
    int* h = hist + (level & 1) * kSlBins;
    const int s = res_shift(hi_k - lo_k);
#pragma unroll 1
    for (int c = 0; c < g.nch; ++c) {
      const int valid = valid_of(c);
      if (valid <= 0) continue;
      const uint4 x = load_vec(c);
      uint32_t m = res_mask_ge<DT>(x, lo_k, valid);
#pragma unroll 1
      while (m != 0u) {
        const int e = __ffs(m) - 1;
        m &= m - 1u;
        const uint32_t kk = E::key(vec_elem_dyn<DT>(x, e));
        if (kk <= hi_k) atomicAdd(&h[(hi_k - kk) >> s], 1);
      }
    }
    sl_sync<CLUSTER>(cluster);
    {   // the other level buffer is read by nobody any more: clear it
      int4* z = reinterpret_cast<int4*>(hist + ((level + 1) & 1) * kSlBins);
#pragma unroll 1
      for (int i = tid; i < kSlBins / 4; i += THREADS) z[i] = make_int4(0, 0, 0, 0);
    }
    const int* H = h;
    if (CLUSTER) {
      cluster_hist_sum<THREADS>(h, hist + 2 * kSlBins, g.C, cluster);
      H = hist + 2 * kSlBins;
    }
    const BinHit bh = res_find_bin(H, need, lane);
    const uint32_t bhi = hi_k - (static_cast<uint32_t>(bh.bin) << s);
    const uint32_t blo = res_bin_lo(hi_k, lo_k, bh.bin, s);
    need -= bh.before;
    if (s == 0) {
      hi_k = bhi;
      eq_total = bh.cnt;
      break;
    }
    lo_k = blo;
    hi_k = bhi;
    if (CLUSTER) cluster.sync();   // every CTA has read the peers' level histogram
  }
  const uint32_t kstar = hi_k;
  const bool has_gt = kstar < kmax_row;
  auto masks = [&](const uint4& x, int valid, uint32_t& gt) -> uint32_t {   // returns eq
    const uint32_t ge = res_mask_ge<DT>(x, kstar, valid);
    gt = has_gt ? res_mask_ge<DT>(x, kstar + 1u, valid) : 0u;
    return ge & ~gt;
  };
  // ---- the need-th entry equal to K*, in index order ----
  uint32_t istar = 0xFFFFFFFFu;
  if (need < eq_total) {   // uniform over the cluster
#pragma unroll 1
    for (int i = tid; i < 2 * words; i += THREADS) bm[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int c = 0; c < g.nch; ++c) {
      const int valid = valid_of(c);
      if (valid <= 0) continue;
      uint32_t gt;
      const uint32_t eq = masks(load_vec(c), valid, gt);
      if (eq != 0u) {
        const uint32_t b0 = static_cast<uint32_t>(c * THREADS + tid) * PV;   // PV divides 32: one word
        atomicOr(&bm[b0 >> 5], eq << (b0 & 31u));
      }
    }
    __syncthreads();
    const int mine = bitmap_prefix<THREADS>(bm, pre, words, ctl);
    if (tid == 0) ctl.x_cnt = mine;
    int off = 0;
    if (CLUSTER) {
      cluster.sync();
      off = slices_before(ctl, &SliceCtl::x_cnt, g.crank, cluster, lane);
    }
    const int r = need - 1 - off;   // rank inside this slice of the boundary entry
    if (r >= 0 && r < mine) {
#pragma unroll 1
      for (int w = tid; w < words; w += THREADS) {
        const uint32_t bits = bm[w];
        if (static_cast<int>(pre[w]) <= r && r < static_cast<int>(pre[w]) + __popc(bits)) {
          uint32_t m = bits;
#pragma unroll 1
          for (int q = r - static_cast<int>(pre[w]); q > 0; --q) m &= m - 1u;
          ctl.x_istar = g.lo + static_cast<uint32_t>(w) * 32u + static_cast<uint32_t>(__ffs(m) - 1);
        }
      }
    }
    if (CLUSTER) {
      cluster.sync();
      int holder = 0;   // the slice holding the boundary entry
      {
        const int cnt = lane < g.C ? cluster.map_shared_rank(&ctl, lane)->x_cnt : 0;
        const int incl = warp_incl_scan(cnt, lane);
        holder = __ffs(__ballot_sync(0xffffffffu, lane < g.C && incl >= need)) - 1;
      }
      istar = cluster.map_shared_rank(&ctl, holder)->x_istar;
    } else {
      __syncthreads();
      istar = ctl.x_istar;
    }
  }
  // ---- selected entries, ranked in index order ----
#pragma unroll 1
  for (int i = tid; i < 2 * words; i += THREADS) bm[i] = 0u;
  __syncthreads();
#pragma unroll 1
  for (int c = 0; c < g.nch; ++c) {
    const int valid = valid_of(c);
    if (valid <= 0) continue;
    uint32_t gt;
    uint32_t eq = masks(load_vec(c), valid, gt);
    const uint32_t b0 = static_cast<uint32_t>(c * THREADS + tid) * PV;
    uint32_t keep = gt;
#pragma unroll 1
    while (eq != 0u) {
      const int e = __ffs(eq) - 1;
      eq &= eq - 1u;
      if (g.lo + b0 + static_cast<uint32_t>(e) <= istar) keep |= 1u << e;
    }
    if (keep != 0u) atomicOr(&bm[b0 >> 5], keep << (b0 & 31u));
  }
  __syncthreads();
  const int mine = bitmap_prefix<THREADS>(bm, pre, words, ctl);
  int off = 0;
  if (CLUSTER) {
    if (tid == 0) ctl.x_sel = mine;
    cluster.sync();
    off = slices_before(ctl, &SliceCtl::x_sel, g.crank, cluster, lane);
  }
  const int64_t obase = g.row * static_cast<int64_t>(k);
#pragma unroll 1
  for (int c = 0; c < g.nch; ++c) {
    const int valid = valid_of(c);
    if (valid <= 0) continue;
    const uint32_t b0 = static_cast<uint32_t>(c * THREADS + tid) * PV;
    uint32_t m = (bm[b0 >> 5] >> (b0 & 31u)) & ((1u << PV) - 1u);
    if (m == 0u) continue;
    const uint4 x = load_vec(c);
#pragma unroll 1
    while (m != 0u) {
      const int e = __ffs(m) - 1;
      m &= m - 1u;
      const int pos = off + bitmap_rank(bm, pre, b0 + static_cast<uint32_t>(e));
      if (pos < k) {
        const uint32_t gi = g.lo + b0 + static_cast<uint32_t>(e);
        if (p.index_i64) static_cast<int64_t*>(p.indices_out)[obase + pos] = static_cast<int64_t>(gi);
        else static_cast<int32_t*>(p.indices_out)[obase + pos] = static_cast<int32_t>(gi);
        if (p.return_value) static_cast<bits_t*>(p.values_out)[obase + pos] = static_cast<bits_t>(vec_elem_dyn<DT>(x, e));
      }
    }
  }
  if (CLUSTER) cluster.sync();   // the peers read this CTA's counts above: leave together
}

// The leader's candidate list: C * NW segments of `seg` entries, segment s
// (slice s / NW, warp s % NW) holding segcnt[s] entries.  Visits every entry,
// warp w taking segments w, w + NW, ... and its lanes the entries side by side;
// f(i, valid) runs in every lane, with the same trip count across the warp.
template <int THREADS, typename F>
__device__ __forceinline__ void for_list(const int* segcnt, int nseg, int seg, F&& f) {
  constexpr int NW = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll 1
  for (int s = warp; s < nseg; s += NW) {
    const int cnt = segcnt[s];
#pragma unroll 1
    for (int j0 = 0; j0 < cnt; j0 += 32) {
      const int j = j0 + lane;
      f(s * seg + j, j < cnt);
    }
  }
}

// The leader's exact finish when the boundary bin is too big to rank directly:
// histogram levels over the list entries with keys in [lo_k, hi_k] (the `need`-th
// largest of them is the boundary), one warp searching, until the boundary bin is
// one key or holds at most kSlMembers entries, which are ranked by (key, index);
// many entries of one key are ranked by index through the bitmap `bm` of the row,
// which is zero on entry and left for the caller to clear.  `h2` is two free
// histograms.  The result is the composite boundary (K*, I*).
template <int DT, int THREADS>
__device__ __noinline__ void list_boundary(const KParams& p, const SliceGeom& g, const typename Elem<DT>::bits_t* lbits,
                                           const uint32_t* lidx, const int* segcnt, int nseg, uint32_t lo_k,
                                           uint32_t hi_k, int need, int* h2, uint32_t* bm, SliceCtl& ctl,
                                           uint32_t& kstar, uint32_t& istar) {
  using E = Elem<DT>;
  constexpr int NW = THREADS / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int seg = p.seg;
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll 1
  for (int i = tid; i < 2 * kSlBins / 4; i += THREADS) reinterpret_cast<int4*>(h2)[i] = make_int4(0, 0, 0, 0);
  __syncthreads();
#pragma unroll 1
  for (int level = 0;; ++level) {
    int* h = h2 + (level & 1) * kSlBins;
    const int s = res_shift(hi_k - lo_k);
    for_list<THREADS>(segcnt, nseg, seg, [&](int i, bool valid) {
      if (valid) {
        const uint32_t kk = E::key(lbits[i]);
        if (kk >= lo_k && kk <= hi_k) atomicAdd(&h[(hi_k - kk) >> s], 1);
      }
    });
    __syncthreads();
    if (warp == 0) {
      const BinHit bh = res_find_bin(h, need, lane);
      if (lane == 0) {
        ctl.bin = bh.bin;
        ctl.before = bh.before;
        ctl.cnt = bh.cnt;
      }
    }
    {   // the other level buffer is read by nobody any more: clear it for the next level
      int4* z = reinterpret_cast<int4*>(h2 + ((level + 1) & 1) * kSlBins);
#pragma unroll 1
      for (int i = tid; i < kSlBins / 4; i += THREADS) z[i] = make_int4(0, 0, 0, 0);
    }
    __syncthreads();
    const int bin = ctl.bin, cnt = ctl.cnt;
    need -= ctl.before;
    const uint32_t bhi = hi_k - (static_cast<uint32_t>(bin) << s);
    const uint32_t blo = res_bin_lo(hi_k, lo_k, bin, s);
    if (s == 0 && cnt == need) {   // every entry of the boundary key is selected
      kstar = bhi;
      istar = 0xFFFFFFFFu;
      return;
    }
    auto member = [&](int i) -> bool {
      const uint32_t kk = E::key(lbits[i]);
      return kk >= blo && kk <= bhi;
    };
    if (cnt <= kSlMembers) {   // rank the members by (key, index); slots from per-warp counts
      int mine = 0;
      for_list<THREADS>(segcnt, nseg, seg, [&](int i, bool valid) { mine += valid && member(i) ? 1 : 0; });
      mine = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(mine)));
      if (lane == 0) ctl.w_c[warp] = mine;
      __syncthreads();
      int M;
      int pos = warp_prefix_of<NW>(ctl.w_c, warp, lane, M);
      if (mine != 0) {   // warp-uniform
        for_list<THREADS>(segcnt, nseg, seg, [&](int i, bool valid) {
          const bool m = valid && member(i);
          const unsigned bal = __ballot_sync(0xffffffffu, m);
          const int at = pos + __popc(bal & below);
          if (m && at < kSlMembers)
            ctl.m_w[at] = (static_cast<unsigned long long>(E::key(lbits[i])) << 32) | (~lidx[i]);
          pos += __popc(bal);
        });
      }
      __syncthreads();
      M = min(M, kSlMembers);
#pragma unroll 1
      for (int j = tid; j < M; j += THREADS) {
        const unsigned long long wj = ctl.m_w[j];
        int r = 0;
#pragma unroll 4
        for (int i = 0; i < M; ++i) r += ctl.m_w[i] > wj ? 1 : 0;
        if (r == need - 1) {
          ctl.kstar = static_cast<uint32_t>(wj >> 32);
          ctl.istar = ~static_cast<uint32_t>(wj);
        }
      }
      __syncthreads();
      kstar = ctl.kstar;
      istar = ctl.istar;
      return;
    }
    if (s == 0) {   // many entries of the boundary key: the need-th of them in index order
      kstar = bhi;
      const int words = static_cast<int>((g.n + 31u) / 32u);
      int* bp = reinterpret_cast<int*>(bm + words);
      for_list<THREADS>(segcnt, nseg, seg, [&](int i, bool valid) {
        if (valid && E::key(lbits[i]) == kstar) atomicOr(&bm[lidx[i] >> 5], 1u << (lidx[i] & 31u));
      });
      __syncthreads();
      row_bitmap_prefix<THREADS>(bm, bp, words, ctl);
      for_list<THREADS>(segcnt, nseg, seg, [&](int i, bool valid) {
        if (valid && E::key(lbits[i]) == kstar && row_bitmap_rank(bm, bp, lidx[i]) == need - 1) ctl.istar = lidx[i];
      });
      __syncthreads();
      istar = ctl.istar;
      return;
    }
    lo_k = blo;
    hi_k = bhi;
  }
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// One CTA per slice; clusters of C CTAs along x hold the C slices of one row.
// The slice lands in shared memory as chunks of one 16-byte vector per thread:
// thread t's vector of chunk c is slice vector c * THREADS + t, so (chunk, thread,
// element) is index order and every thread holds an even share of any index range.
template <int DT, int THREADS, bool CLUSTER>
__device__ __forceinline__ void slice_body(const KParams& p, unsigned char* smem, cg::cluster_group& cluster) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  constexpr int CE = THREADS * PV;   // elements per chunk
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);   // [3][kSlBins]: candidates, sample, spare
  uint16_t* vkm = reinterpret_cast<uint16_t*>(smem + p.off_tab) + threadIdx.x;   // [sample chunk][THREADS]
  bits_t* lbits = reinterpret_cast<bits_t*>(smem + p.off_cb);     // candidate list (leader): element bits
  uint32_t* lidx = reinterpret_cast<uint32_t*>(smem + p.off_ci);  //                          row index
  SliceCtl& ctl = *reinterpret_cast<SliceCtl*>(smem + p.off_ctl);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t below = (1u << lane) - 1u;
  SliceGeom g;
  g.C = CLUSTER ? static_cast<int>(cluster.num_blocks()) : 1;
  g.crank = CLUSTER ? static_cast<int>(cluster.block_rank()) : 0;
  g.row = CLUSTER ? static_cast<int64_t>(cluster_id_x()) : static_cast<int64_t>(blockIdx.x);
  const bool leader = g.crank == 0;
  const int k = p.k;
  const int seg = p.seg;
  sl_mark(0);

#pragma unroll 1
  for (int i = tid; i < 3 * kSlBins / 4; i += THREADS) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  if (tid == 0) {
    ctl.flags = 0;
    ctl.t_max = 0u;
    ctl.t_min = 0xFFFFFFFFu;
    ctl.top = 0u;
    ctl.kmax = 0u;
  }
  if (tid < p.vpt_cap) {
    mbar_init(smem_u32(&bars[tid]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the leader's counters and histogram are initialised: peers may update them
  // after the wait half of this barrier.  (Arriving here, before any copy is
  // issued: a cluster-scope release after a bulk copy waits for the copy to land.)
  // Every CTA of the row arrives, and waits below unless the row is short.
  if (CLUSTER) cluster_arrive();
  // the set-up above touched shared memory only: it may overlap the previous launch
  grid_dependency_wait();
  sl_mark(1);

  // ---- the slice, and its copies issued first ----
  uint32_t sl, pa;
  int nch_full;
  if (p.end == nullptr) {   // every row is row_stride long: the host computed the geometry
    g.n = static_cast<uint32_t>(p.row_stride);
    sl = p.sl_full;
    nch_full = p.nch_full;
    pa = p.pa_full;
  } else {
    bool bad_end;
    const int64_t n64 = row_length(p, g.row, &bad_end);
    if (bad_end || n64 <= k) {   // the same for every CTA of the row: all leave here
      if (leader) {
        if (bad_end) write_sentinel_row<DT, THREADS>(p, g.row, DSEL_IDX_BAD_END);
        else write_short_row<DT, THREADS>(p, g.row, n64);
      }
      return;
    }
    g.n = static_cast<uint32_t>(n64);
    sl = ((g.n + g.C - 1u) / static_cast<uint32_t>(g.C) + 15u) / 16u * 16u;
    nch_full = static_cast<int>((sl + CE - 1u) / CE);
    pa = 0u;   // set below, per slice
  }
  if (g.n <= static_cast<uint32_t>(k)) {   // rows of row_stride <= k elements
    if (leader) write_short_row<DT, THREADS>(p, g.row, g.n);
    return;
  }
  g.lo = min(g.n, static_cast<uint32_t>(g.crank) * sl);
  g.n_sl = min(g.n, g.lo + sl) - g.lo;
  g.nch = static_cast<int>((g.n_sl + CE - 1u) / CE);   // <= vpt_cap
  if (g.nch != nch_full || pa == 0u) pa = chunk_stride(static_cast<uint32_t>(g.nch));
  // chunk visiting order: j -> (pa * j + pc) mod nch
  const uint32_t pc = __umulhi(static_cast<uint32_t>((static_cast<uint64_t>(g.row) + 1u) * 0x9E3779B97F4A7C15ull >> 32) ^
                                   (static_cast<uint32_t>(g.crank) * 0x85EBCA6Bu),
                               static_cast<uint32_t>(g.nch));
  const char* rowp = static_cast<const char*>(p.x) + g.row * p.row_stride * E::kBytes;
  if (lane == 0 && warp < g.nch) {   // warp j issues the j-th chunk of the visiting order
    const int c = static_cast<int>((pa * static_cast<uint32_t>(warp) + pc) % static_cast<uint32_t>(g.nch));
    const uint32_t e0 = static_cast<uint32_t>(c) * CE;
    const uint32_t ne = min(static_cast<uint32_t>(CE), g.n_sl - e0);
    // the last chunk of the row may end inside a 16-byte unit: the copy rounds up,
    // which stays inside the row's padded stride (a multiple of 16 elements)
    const uint32_t bytes = (ne * E::kBytes + 15u) & ~15u;
    const uint32_t bar = smem_u32(&bars[c]);
    mbar_expect_tx(bar, bytes);
    bulk_g2s(smem_u32(smem + static_cast<size_t>(c) * kSlChunk), rowp + static_cast<size_t>(g.lo + e0) * E::kBytes,
             bytes, bar);
  }
#ifdef DSEL_STATS
  if (tid == 0 && blockIdx.x < 8) g_trace[blockIdx.x * 32 + 16] = static_cast<long long>(global_ns());
#endif
  grid_launch_dependents();
  sl_mark(2);

  auto load_vec = [&](int c) -> uint4 {
    return *reinterpret_cast<const uint4*>(smem + static_cast<size_t>(c) * kSlChunk + tid * kVecBytes);
  };
  auto valid_of = [&](int c) -> int { return static_cast<int>(g.n_sl) - (c * THREADS + tid) * PV; };
  bool late = false;
  auto wait_chunk = [&](int c) {
    if (!mbar_wait(smem_u32(&bars[c]), 0u)) late = true;
  };
  auto next_chunk = [&](int c) -> int {   // the chunk after c in the visiting order
    const uint32_t t = static_cast<uint32_t>(c) + pa;
    return static_cast<int>(t >= static_cast<uint32_t>(g.nch) ? t - static_cast<uint32_t>(g.nch) : t);
  };

  // ---- A. threshold from the first ns chunks of the visiting order ----
  // Candidates expected past a threshold taken from a fraction f of the row:
  // about 1.3 k / f.  Each slice's own k-th (each valid alone; the cluster keeps
  // the largest) while C slices' worth of candidates fit half the list with at most
  // half the slice as sample; otherwise per-slice k' = ceil(k / C) thresholds and
  // the cluster keeps the smallest (C slices with k' such vectors: at least k).
  const int lcap = p.capacity;
  auto chunks_for = [&](int64_t kk, int64_t slices) -> int {     // sample chunks for a list of lcap / 2
    const int64_t by_list = (13 * slices * kk * nch_full + 5 * lcap - 1) / (5 * lcap);
    const int64_t by_k = (2 * kk + THREADS - 1) / THREADS;
    const int64_t q = (nch_full + 3) / 4;
    return static_cast<int>(by_list > by_k ? (by_list > q ? by_list : q) : (by_k > q ? by_k : q));
  };
  const int ns_local = chunks_for(k, g.C);
  const bool local = !CLUSTER || 2 * ns_local <= nch_full;
  const int kq = local ? k : (k + g.C - 1) / g.C;
  const int ns = min(g.nch, local ? ns_local : chunks_for(k, 1));
  uint32_t tmax = 0u, tmin16 = 0xFFFFu;
  int tn = 0;
  bool tnan = false;
  {
    int c = static_cast<int>(pc);
#pragma unroll 1
    for (int j = 0; j < ns; ++j, c = next_chunk(c)) {
      wait_chunk(c);
#ifdef DSEL_STATS
      if (tid == 0 && blockIdx.x < 8) g_trace[blockIdx.x * 32 + j] = static_cast<long long>(global_ns());
#endif
      uint32_t s16 = 0u;
      const int valid = valid_of(c);
      if (valid > 0) {
        uint32_t key = 0u;
        if (vec_max_valid<DT>(load_vec(c), valid, key)) {
          tnan = true;
        } else {
          s16 = key16<DT>(key);
          tmax = max(tmax, key);
          tmin16 = min(tmin16, s16);
          ++tn;
        }
      }
      vkm[j * THREADS] = static_cast<uint16_t>(s16);
    }
  }
  sl_mark(3);
  tmax = __reduce_max_sync(0xffffffffu, tmax);
  tmin16 = __reduce_min_sync(0xffffffffu, tmin16);
  tn = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(tn)));
  if (lane == 0) {
    ctl.w_a[warp] = tmax;
    ctl.w_b[warp] = tmin16;
    ctl.w_c[warp] = tn;
  }
  __syncthreads();
  const uint32_t smax = __reduce_max_sync(0xffffffffu, lane < NW ? ctl.w_a[lane] : 0u);
  const uint32_t smin = __reduce_min_sync(0xffffffffu, lane < NW ? ctl.w_b[lane] : 0xFFFFu);
  const int sn = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(lane < NW ? ctl.w_c[lane] : 0)));
  uint32_t t_row = 0u;
  if (sn >= kq) {   // uniform in the CTA
    // bins 16 times narrower than the summaries' range needs, the last one open
    // below: the top sixteenth of the range, where the kq-th largest usually lies
    const uint32_t top16 = key16<DT>(smax);
    const int s = max(0, res_shift(top16 - smin) - 4);
    int* h = hist + kSlBins;
#pragma unroll 4
    for (int j = 0; j < ns; ++j) {
      const uint32_t m = vkm[j * THREADS];
      if (m != 0u) atomicAdd(&h[min((top16 - m) >> s, static_cast<uint32_t>(kSlBins - 1))], 1);
    }
    __syncthreads();
    if (warp == 0) {
      const BinHit bh = res_find_bin(h, kq, lane);
      if (lane == 0) {
        const uint32_t t16 = bh.bin == kSlBins - 1 ? smin : res_bin_lo(top16, smin, bh.bin, s);
        ctl.t_key = DT == DSEL_BF16 ? t16 : (t16 << 16);
      }
    }
    __syncthreads();
    t_row = ctl.t_key;
  }
  uint32_t top = smax;   // bins of the candidate histogram count down from here
  SliceCtl* lctl = CLUSTER ? cluster.map_shared_rank(&ctl, 0) : &ctl;
  if (CLUSTER) {   // the cluster's threshold and top, through the leader
    cluster_wait();   // the leader's counters are initialised
    if (tid == 0) {
      if (local) atomicMax(&lctl->t_max, t_row);
      else atomicMin(&lctl->t_min, t_row);
      atomicMax(&lctl->top, smax);
    }
#ifdef DSEL_STATS
    if (tid == 0 && blockIdx.x < 8) g_trace[blockIdx.x * 32 + 18] = static_cast<long long>(global_ns());
#endif
    cluster.sync();
#ifdef DSEL_STATS
    if (tid == 0 && blockIdx.x < 8) g_trace[blockIdx.x * 32 + 19] = static_cast<long long>(global_ns());
#endif
    if (lane == 0) {
      t_row = local ? lctl->t_max : lctl->t_min;
      top = lctl->top;
    }
    t_row = __shfl_sync(0xffffffffu, t_row, 0);
    top = __shfl_sync(0xffffffffu, top, 0);
  }
  top = max(top, t_row);
  const int sb = res_shift(top - t_row);   // one key per bin for bfloat16 when the range allows
  sl_mark(4);

  // ---- B. filter every chunk against T: this warp's segment of the leader's
  //      list, and this CTA's histogram of the candidates' keys ----
  const int sid = g.crank * NW + warp;
  bits_t* rbits = (CLUSTER ? cluster.map_shared_rank(lbits, 0) : lbits) + sid * seg;
  uint32_t* ridx = (CLUSTER ? cluster.map_shared_rank(lidx, 0) : lidx) + sid * seg;
  int* hc = hist;   // candidates, bins counting down from top (keys above top share bin 0)
  const uint32_t t16 = key16<DT>(t_row);
  uint32_t kmax_sl = tmax;   // largest key of the slice
  int wrun = 0;              // entries of this warp's segment (warp-uniform)
  {
    int c = static_cast<int>(pc);
#pragma unroll 1
    for (int j = 0; j < g.nch; ++j, c = next_chunk(c)) {
      const int valid = valid_of(c);
      bool cand = false;
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (j < ns) {
        const uint32_t sm = vkm[j * THREADS];
        cand = valid > 0 && sm >= t16 && sm != 0u;
        if (cand) x = load_vec(c);
      } else {
        wait_chunk(c);
#ifdef DSEL_STATS
        if (tid == 0 && blockIdx.x < 8) g_trace[blockIdx.x * 32 + j] = static_cast<long long>(global_ns());
#endif
        if (valid > 0) {
          x = load_vec(c);
          uint32_t key = 0u;
          if (vec_max_valid<DT>(x, valid, key)) {
            tnan = true;
          } else {
            kmax_sl = max(kmax_sl, key);
            cand = key >= t_row;
          }
        }
      }
      uint32_t m = cand ? res_mask_ge<DT>(x, t_row, valid) : 0u;
      const uint32_t g0 = g.lo + static_cast<uint32_t>(c * THREADS + tid) * PV;
#pragma unroll 1
      while (__any_sync(0xffffffffu, m != 0u)) {   // one candidate per lane per step
        const bool has = m != 0u;
        const unsigned bal = __ballot_sync(0xffffffffu, has);
        if (has) {
          const int e = __ffs(m) - 1;
          m &= m - 1u;
          const int pos = wrun + __popc(bal & below);
          const uint32_t b = vec_elem_dyn<DT>(x, e);
          const uint32_t kk = E::key(b);
          atomicAdd(&hc[kk >= top ? 0u : (top - kk) >> sb], 1);
          if (pos < seg) {
            rbits[pos] = static_cast<bits_t>(b);
            ridx[pos] = g0 + static_cast<uint32_t>(e);
          }
        }
        wrun += __popc(bal);
      }
#ifdef DSEL_STATS
      if (tid == 0 && blockIdx.x < 8 && j < 8) g_trace[blockIdx.x * 32 + 20 + j] = static_cast<long long>(global_ns());
#endif
    }
  }
  sl_mark(5);
  {
    const int f = (__any_sync(0xffffffffu, tnan) ? 1 : 0) | (wrun > seg ? 2 : 0) |
                  (__any_sync(0xffffffffu, late) ? 4 : 0);
    const uint32_t wk = __reduce_max_sync(0xffffffffu, kmax_sl);
    if (lane == 0) {
      lctl->segcnt[sid] = min(wrun, seg);
      // the flags go to every CTA's own copy: after the barrier below each reads
      // its own (the leader may be gone before a peer could read the leader's)
      if (f) {
        if (CLUSTER) {
#pragma unroll 1
          for (int r = 0; r < g.C; ++r) atomicOr(&cluster.map_shared_rank(&ctl, r)->flags, f);
        } else {
          atomicOr(&ctl.flags, f);
        }
      }
      atomicMax(&lctl->kmax, wk);
    }
  }
  if (CLUSTER && !leader) {   // this CTA's candidate histogram joins the leader's
    __syncthreads();
    int* lh = cluster.map_shared_rank(hc, 0);
#pragma unroll 1
    for (int b = tid; b < kSlBins; b += THREADS) {
      const int v = hc[b];
      if (v) atomicAdd(&lh[b], v);
    }
  }
  if (late && tid < g.nch) mbar_wait(smem_u32(&bars[tid]), 0u);   // a copy may still be landing
  sl_sync<CLUSTER>(cluster);   // the row's candidates are in the leader's list and histogram
  sl_mark(6);
  const int flags = ctl.flags;
  if ((flags & 1) && !p.nan_flag) nan_trap();   // the pages' default NaN policy
  if (flags & 1) {   // flag mode: the row's NaN sentinel
    if (leader) write_sentinel_row<DT, THREADS>(p, g.row, DSEL_IDX_NAN);
    return;
  }
  if (flags & 2) {   // a segment overflowed: every CTA selects exactly on its resident slice
    slice_exact<DT, THREADS, CLUSTER>(p, smem, g, t_row, lctl->kmax, cluster);
    return;
  }
  if (!leader) return;   // the leader finishes the row alone

  // ---- C. the boundary bin, from the summed histogram (one warp searches) ----
  const int nseg = g.C * NW;
#ifdef DSEL_STATS
  if (tid == 0 && blockIdx.x < kStatsCtas) {   // list length, sample chunks, mode, chunks
    int tot = 0;
    for (int s2 = 0; s2 < nseg; ++s2) tot += ctl.segcnt[s2];
    g_stats[blockIdx.x * kStatsFields + 12] = static_cast<unsigned long long>(tot);
    g_stats[blockIdx.x * kStatsFields + 13] = static_cast<unsigned long long>(ns);
    g_stats[blockIdx.x * kStatsFields + 14] = local ? 1ull : 0ull;
    g_stats[blockIdx.x * kStatsFields + 15] = static_cast<unsigned long long>(g.nch);
  }
#endif
  if (warp == 0) {
    const BinHit bh = res_find_bin(hc, k, lane);
    if (lane == 0) {
      ctl.bin = bh.bin;
      ctl.before = bh.before;
      ctl.cnt = bh.cnt;
    }
  }
  __syncthreads();
  const int bin = ctl.bin, bcnt = ctl.cnt;
  const int need = k - ctl.before;   // entries of the boundary bin to select (1..bcnt)
  const uint32_t bhi = bin == 0 ? 0xFFFFFFFFu : top - (static_cast<uint32_t>(bin) << sb);
  const uint32_t blo = res_bin_lo(top, t_row, bin, sb);
  // row bitmaps in the leader's dead slice: selected entries, then the block prefix
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem);
  const int words = static_cast<int>((g.n + 31u) / 32u);
  int* bp = reinterpret_cast<int*>(bm + words);
#pragma unroll 1
  for (int w = tid; w < words; w += THREADS) bm[w] = 0u;
  __syncthreads();
  const bool all_bin = bcnt == need;   // every member of the boundary bin is selected
  if (!all_bin && bcnt > kSlMembers) {   // heavy ties or a coarse bin: exact levels over the list
    uint32_t kstar = 0u, istar = 0u;
    list_boundary<DT, THREADS>(p, g, lbits, lidx, ctl.segcnt, nseg, blo, bhi == 0xFFFFFFFFu ? ctl.kmax : bhi,
                               need, hist + kSlBins, bm, ctl, kstar, istar);
#pragma unroll 1
    for (int w = tid; w < words; w += THREADS) bm[w] = 0u;
    __syncthreads();
    for_list<THREADS>(ctl.segcnt, nseg, seg, [&](int i, bool valid) {
      const uint32_t kk = E::key(lbits[i]);
      if (valid && (kk > kstar || (kk == kstar && lidx[i] <= istar))) atomicOr(&bm[lidx[i] >> 5], 1u << (lidx[i] & 31u));
    });
  } else {
    // entries above the boundary bin (and the whole bin when all of it is selected)
    // go into the bitmap; the bin's members are counted per warp
    const uint32_t sel_lo = all_bin ? blo : (bhi == 0xFFFFFFFFu ? 0xFFFFFFFFu : bhi + 1u);
    int mine = 0;
    for_list<THREADS>(ctl.segcnt, nseg, seg, [&](int i, bool valid) {
      if (valid) {
        const uint32_t kk = E::key(lbits[i]);
        if (kk >= sel_lo && (sel_lo != 0xFFFFFFFFu || all_bin)) atomicOr(&bm[lidx[i] >> 5], 1u << (lidx[i] & 31u));
        else if (!all_bin && kk >= blo) ++mine;
      }
    });
    if (!all_bin) {   // rank the members by (key, index): the first `need` are selected
      mine = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(mine)));
      if (lane == 0) ctl.w_c[warp] = mine;
      __syncthreads();
      int M;
      int pos = warp_prefix_of<NW>(ctl.w_c, warp, lane, M);
      if (mine != 0) {   // warp-uniform
        for_list<THREADS>(ctl.segcnt, nseg, seg, [&](int i, bool valid) {
          const uint32_t kk = valid ? E::key(lbits[i]) : 0u;
          const bool m = valid && kk >= blo && kk < sel_lo;
          const unsigned bal = __ballot_sync(0xffffffffu, m);
          if (m) ctl.m_w[pos + __popc(bal & below)] = (static_cast<unsigned long long>(kk) << 32) | (~lidx[i]);
          pos += __popc(bal);
        });
      }
      __syncthreads();
#pragma unroll 1
      for (int j = tid; j < M; j += THREADS) {
        const unsigned long long wj = ctl.m_w[j];
        int r = 0;
#pragma unroll 4
        for (int i = 0; i < M; ++i) r += ctl.m_w[i] > wj ? 1 : 0;
        if (r < need) {
          const uint32_t gi = ~static_cast<uint32_t>(wj);
          atomicOr(&bm[gi >> 5], 1u << (gi & 31u));
        }
      }
    }
  }
  __syncthreads();
  row_bitmap_prefix<THREADS>(bm, bp, words, ctl);
  sl_mark(7);

  // ---- output: every selected entry at its rank in index order ----
  const int64_t obase = g.row * static_cast<int64_t>(k);
  for_list<THREADS>(ctl.segcnt, nseg, seg, [&](int i, bool valid) {
    if (!valid) return;
    const uint32_t gi = lidx[i];
    if (!((bm[gi >> 5] >> (gi & 31u)) & 1u)) return;
    const int pos = row_bitmap_rank(bm, bp, gi);
    if (pos < k) {
      if (p.index_i64) static_cast<int64_t*>(p.indices_out)[obase + pos] = static_cast<int64_t>(gi);
      else static_cast<int32_t*>(p.indices_out)[obase + pos] = static_cast<int32_t>(gi);
      if (p.return_value) static_cast<bits_t*>(p.values_out)[obase + pos] = lbits[i];
    }
  });
  sl_mark(9);
}

template <int DT, int THREADS, bool CLUSTER>
__global__ void __launch_bounds__(THREADS, 1) topk_slice_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  slice_body<DT, THREADS, CLUSTER>(p, smem, cluster);
  sl_mark(11);
}

}  // namespace dsel
