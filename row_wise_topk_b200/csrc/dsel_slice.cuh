// Slice-resident TopK: the rows of a batch are cut into slices that fit in shared
// memory, one CTA per slice, and the slices of one row form a thread-block
// cluster.  Every CTA loads its whole slice with bulk copies (all in flight at
// once), so the row is read exactly once.  The method is the threshold filter of
// "DeepSeek releases DeepSelect, a TopK kernel for sparse attention and sampling"
// (method paragraph), laid out for the order in which the data lands:
//
//   A. threshold from the vector maxima: as each chunk lands, every 16-byte
//      vector's largest key goes, as a 16-bit summary, into a table and into a
//      histogram of fixed bins (16 summaries each, so every CTA of the cluster
//      has the same bins).  After one cluster barrier the CTAs sum the histograms
//      through distributed shared memory (coarse sums first, then the 16 fine
//      bins of one coarse bin) and take T, the lower edge of the bin that holds
//      the row's k-th largest vector maximum: at least k vectors hold an element
//      >= T, so T is a valid threshold, and it is the tightest one these bins give;
//   B. filter, dense in two steps: the vectors whose summary reaches T go into
//      this warp's vector list (one ballot per vector slot), then their elements
//      >= T, 32 vectors per warp step, into this warp's element list (which stays
//      in index order) and the CTA's histogram of candidate keys;
//   C. exact finish, shared by the cluster: after one cluster barrier the CTAs
//      sum their candidate histograms the same way and refine the bin that holds
//      the k-th entry (one cluster barrier per extra level) down to the boundary
//      key K*, or to a bin that is selected whole.  Each CTA then counts its
//      entries above K* and equal to it per block of 32 vectors; after one more
//      cluster barrier every CTA knows how many entries each slice contributes, so
//      it writes its own selection at its offset, ranked in index order from the
//      block counts.  The entries equal to K* are taken in index order across the
//      slices (the composite (value, index) order: value descending, lower index
//      first among equals).
//
// When a candidate list overflows an exact fallback runs on the resident slices
// (every CTA): histogram levels down to a single key, then ranks in index order
// from bitmaps.  No wait depends on another CTA except the hardware cluster
// barriers, which every CTA of a cluster passes equally often (each path is
// chosen from cluster-wide values); the bulk-copy waits are bounded.  A CTA that
// has read a peer's shared memory arrives at a last cluster barrier before it
// leaves.
#pragma once

#include "dsel_resident.cuh"

namespace dsel {

constexpr int kSlBins = 1024;
constexpr int kSlVBins = 4096;   // vector-maximum histogram: fixed bins of 16 key summaries
constexpr int kSlChunk = kSliceChunkBytes;                   // bytes per chunk
constexpr int kSlChunkVecs = kSliceChunkBytes / kVecBytes;   // 16-byte vectors per chunk

struct __align__(16) SliceCtl {
  uint32_t w_a[kWarpsMax];
  uint32_t w_b[kWarpsMax];
  int w_c[kWarpsMax];
  int bin, before, cnt;      // a bin search, broadcast to the CTA
  int bin2, before2, cnt2;   // the fine stage of a two-stage search
  // published to the cluster: the peers read these after a cluster barrier
  int flags;                 // bit 0: NaN seen, bit 1: list overflow, bit 2: a wait gave up
  uint32_t kmax;             // largest key of this slice
  int x_a;                   // entries selected above the boundary key
  int x_t;                   // entries equal to the boundary key
  int x_sel, x_cnt;          // exact fallback: selected / tied entries of this slice
  uint32_t x_istar;          // the last selected tie (row index)
  int n_list;                // entries in this CTA's candidate list
#ifdef DSEL_STATS
  unsigned long long marks[32];   // phase timestamps, written out when the CTA ends
#endif
};

// Phase timestamps of thread 0 in counter builds only: the SM's cycle counter
// (cheap to read), kept in shared memory (a global store before a cluster barrier
// would make the barrier's release wait for it) and written to g_stats[cta][i]
// when the CTA ends.  Cycles count from the CTA's own start: compare durations
// within a CTA.
__device__ __forceinline__ void sl_mark(SliceCtl& ctl, int i) {
#ifdef DSEL_STATS
  if (threadIdx.x == 0) ctl.marks[i] = static_cast<unsigned long long>(clock64());
#else
  (void)ctl;
  (void)i;
#endif
}

__device__ __forceinline__ void sl_marks_out(SliceCtl& ctl) {
#ifdef DSEL_STATS
  if (threadIdx.x == 0 && blockIdx.x < kStatsCtas) {
    ctl.marks[11] = static_cast<unsigned long long>(clock64());
#pragma unroll 1
    for (int i = 0; i < 16; ++i) g_stats[blockIdx.x * kStatsFields + i] = ctl.marks[i];
    if (blockIdx.x < kStatsCtas / 2) {   // per-chunk times in the upper half
#pragma unroll 1
      for (int i = 0; i < 16; ++i) g_stats[(kStatsCtas / 2 + blockIdx.x) * kStatsFields + i] = ctl.marks[16 + i];
    }
  }
#else
  (void)ctl;
#endif
}

template <bool CLUSTER>
__device__ __forceinline__ void sl_sync(cg::cluster_group& cluster) {
  if (CLUSTER) cluster.sync();
  else __syncthreads();
}

// Split cluster barrier: arrive (release) once this CTA is done reading its
// peers' shared memory, wait (acquire) just before it leaves.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// 16-bit summary of a key kept per sampled vector: the key itself for bfloat16,
// its top 16 bits for float32 (so summary >= key16(t) is a superset test for
// key >= t).
template <int DT>
__device__ __forceinline__ uint32_t key16(uint32_t key) {
  return DT == DSEL_BF16 ? key : (key >> 16);
}

// vec_max_key_fast and nacc_is_nan: dsel_resident.cuh.

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

// Coarse sums of a histogram kept beside it for the two-stage search:
// coarse[i] = fine[16 i] + ... + fine[16 i + 15], i < ncb.  The caller has made
// the fine histogram complete with a CTA barrier, and publishes both with a
// cluster barrier.
template <int THREADS>
__device__ __forceinline__ void coarse_sums(const int* fine, int* coarse, int ncb) {
#pragma unroll 1
  for (int i = threadIdx.x; i < ncb; i += THREADS) {
    const int4* f4 = reinterpret_cast<const int4*>(fine + 16 * i);
    int sum = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int4 v = f4[q];
      sum += v.x + v.y + v.z + v.w;
    }
    coarse[i] = sum;
  }
}

// Element i of an int array summed over the cluster's CTAs, four loads in flight.
template <bool CLUSTER>
__device__ __forceinline__ int cluster_sum_at(const int* a, int i, int C, cg::cluster_group& cluster) {
  if (!CLUSTER) return a[i];
  const int me = static_cast<int>(cluster.block_rank());
  int sum = 0;
#pragma unroll 1
  for (int r0 = 0; r0 < C; r0 += 4) {
    int v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + q;
      v[q] = r < C ? cluster.map_shared_rank(a, r + me < C ? r + me : r + me - C)[i] : 0;
    }
    sum += v[0] + v[1] + v[2] + v[3];
  }
  return sum;
}

// Bin of the need-th largest entry of a histogram of 16 * ncb bins (bin 0 the
// largest keys), summed over the cluster, in two stages: the coarse sums (ncb <=
// THREADS bins of 16) locate the coarse bin, whose 16 fine bins then locate the
// bin.  The caller has passed a cluster barrier after publishing both arrays.
// Two CTA barriers; bin = -1 when the histogram holds fewer than `need` entries.
// With `fx`, every warp also reads the cluster's flags (OR) and largest key (max)
// into fx[0], fx[1], those loads overlapping the search's own.
template <int THREADS, bool CLUSTER>
__device__ __forceinline__ BinHit cluster_find_bin(const int* fine, const int* coarse, int ncb, int need, int C,
                                                   SliceCtl& ctl, cg::cluster_group& cluster,
                                                   uint32_t* fx = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t f_or = 0u, k_max = 0u;
  if (fx != nullptr && lane < C) {
    const SliceCtl* pr = CLUSTER ? cluster.map_shared_rank(&ctl, lane) : &ctl;
    f_or = static_cast<uint32_t>(pr->flags);
    k_max = pr->kmax;
  }
  const int c = tid < ncb ? cluster_sum_at<CLUSTER>(coarse, tid, C, cluster) : 0;
  if (fx != nullptr) {
    fx[0] = __reduce_or_sync(0xffffffffu, f_or);
    fx[1] = __reduce_max_sync(0xffffffffu, k_max);
  }
  // the coarse bins, one per thread: a CTA-wide scan finds the one that holds the
  // need-th entry; the warp holding it then reads that bin's 16 fine bins before
  // the second barrier
  constexpr int NW = THREADS / 32;
  const int warp = tid >> 5;
  const int incl = warp_incl_scan(c, lane);
  if (lane == 31) ctl.w_c[warp] = incl;
  __syncthreads();
  int total;
  const int base = warp_prefix_of<NW>(ctl.w_c, warp, lane, total) + incl - c;
  if (total < need) {   // uniform in the CTA
    __syncthreads();
    BinHit r;
    r.bin = -1;
    r.before = 0;
    r.cnt = 0;
    return r;
  }
  const unsigned wb = __ballot_sync(0xffffffffu, base < need && need <= base + c);
  if (wb != 0u) {   // this warp holds the coarse bin (thread `src` of it)
    const int src = __ffs(wb) - 1;
    const int cb = __shfl_sync(0xffffffffu, tid, src);
    const int cbefore = __shfl_sync(0xffffffffu, base, src);
    const int need2 = need - cbefore;
    const int f = lane < 16 ? cluster_sum_at<CLUSTER>(fine, 16 * cb + lane, C, cluster) : 0;
    const int fincl = warp_incl_scan(f, lane);
    const int j = __ffs(__ballot_sync(0xffffffffu, lane < 16 && fincl >= need2)) - 1;
    if (lane == j) {
      ctl.bin2 = 16 * cb + j;
      ctl.before2 = cbefore + fincl - f;
      ctl.cnt2 = f;
    }
  }
  __syncthreads();
  BinHit r;
  r.bin = ctl.bin2;
  r.before = ctl.before2;
  r.cnt = ctl.cnt2;
  return r;
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
// index order through bitmaps.  Runs on every CTA of the cluster together and
// ends with a cluster barrier.  The slice lies in shared memory as one flat array
// of 16-byte vectors.
template <int DT, int THREADS, bool CLUSTER>
__device__ __noinline__ void slice_exact(const KParams& p, unsigned char* smem, int64_t row, uint32_t slice_lo,
                                         uint32_t n_sl, int C, int crank, uint32_t lo_k, uint32_t kmax_row,
                                         cg::cluster_group& cluster) {
  SliceGeom g;   // rebuilt from values: a reference argument would keep the caller's copy in local memory
  g.row = row;
  g.lo = slice_lo;
  g.n_sl = n_sl;
  g.C = C;
  g.crank = crank;
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int PV = E::kPerVec;
  const int tid = threadIdx.x, lane = tid & 31;
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);
  SliceCtl& ctl = *reinterpret_cast<SliceCtl*>(smem + p.off_ctl);
  uint32_t* bm = reinterpret_cast<uint32_t*>(smem + p.off_tab);   // bitmap, then its prefix
  const int words = static_cast<int>((g.n_sl + 31u) / 32u);
  uint32_t* pre = bm + words;
  const int nvec = static_cast<int>((g.n_sl + PV - 1u) / PV);
  const int k = p.k;
  auto load_vec = [&](int v) -> uint4 { return *reinterpret_cast<const uint4*>(smem + static_cast<size_t>(v) * kVecBytes); };
  auto valid_of = [&](int v) -> int { return static_cast<int>(g.n_sl) - v * PV; };

  // the peers may still read this CTA's control block: meet first, then clear
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
    for (int v = tid; v < nvec; v += THREADS) {
      const uint4 x = load_vec(v);
      uint32_t m = res_mask_ge<DT>(x, lo_k, valid_of(v));
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
    for (int v = tid; v < nvec; v += THREADS) {
      uint32_t gt;
      const uint32_t eq = masks(load_vec(v), valid_of(v), gt);
      if (eq != 0u) {
        const uint32_t b0 = static_cast<uint32_t>(v) * PV;   // PV divides 32: one word
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
  for (int v = tid; v < nvec; v += THREADS) {
    uint32_t gt;
    uint32_t eq = masks(load_vec(v), valid_of(v), gt);
    const uint32_t b0 = static_cast<uint32_t>(v) * PV;
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
  for (int v = tid; v < nvec; v += THREADS) {
    const uint32_t b0 = static_cast<uint32_t>(v) * PV;
    uint32_t m = (bm[b0 >> 5] >> (b0 & 31u)) & ((1u << PV) - 1u);
    if (m == 0u) continue;
    const uint4 x = load_vec(v);
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
  if (CLUSTER) cluster.sync();   // the peers have read this CTA's counts
}

__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}

// One of VT 16-byte vectors held in registers, picked by a run-time index.
template <int VT>
__device__ __forceinline__ uint4 pick(const uint4 (&xs)[VT], int i) {
  if constexpr (VT == 1) {
    return xs[0];
  } else if constexpr (VT == 2) {
    return i == 0 ? xs[0] : xs[1];
  } else {
    static_assert(VT == 4, "one, two or four vectors per thread and chunk");
    return i < 2 ? (i == 0 ? xs[0] : xs[1]) : (i == 2 ? xs[2] : xs[3]);
  }
}

// One CTA per slice; clusters of C CTAs along x hold the C slices of one row.
// The slice lands in shared memory as one flat array of 16-byte vectors, in
// chunks of kSlChunkVecs vectors; thread t screens vectors t, t + THREADS, ... of
// each chunk, so its loads are conflict-free and every thread holds an even share
// of any index range.
template <int DT, int THREADS, bool CLUSTER>
__device__ __forceinline__ void slice_body(const KParams& p, unsigned char* smem, cg::cluster_group& cluster) {
  using E = Elem<DT>;
  using bits_t = typename E::bits_t;
  constexpr int NW = THREADS / 32;
  constexpr int PV = E::kPerVec;
  constexpr int VT = kSlChunkVecs / THREADS;   // vectors per thread and chunk
  constexpr int CE = kSlChunkVecs * PV;        // elements per chunk
  static_assert(VT * THREADS == kSlChunkVecs && VT * PV <= 32, "one 32-bit candidate mask per chunk");
  static_assert(kSliceMaxChunks <= NW, "one warp issues each chunk");
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.off_bars);
  int* hist = reinterpret_cast<int*>(smem + p.off_hist);   // kSlVBins + kSlBins bins
  uint16_t* vkm = reinterpret_cast<uint16_t*>(smem + p.off_tab);   // every vector's key summary
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
  bits_t* wbits = reinterpret_cast<bits_t*>(smem + p.off_cb) + warp * seg;     // this warp's list segment
  uint32_t* widx = reinterpret_cast<uint32_t*>(smem + p.off_ci) + warp * seg;
#ifdef DSEL_STATS
  if (tid < 32) ctl.marks[tid] = 0ull;
#endif
  sl_mark(ctl, 0);

#pragma unroll 1
  for (int i = tid; i < (kSlVBins + kSlBins) / 4; i += THREADS) reinterpret_cast<int4*>(hist)[i] = make_int4(0, 0, 0, 0);
  if (tid == 0) {
    ctl.flags = 0;
    ctl.kmax = 0u;
    ctl.x_a = 0;
    ctl.x_t = 0;
    ctl.n_list = 0;
  }
  if (tid < p.vpt_cap) {
    mbar_init(smem_u32(&bars[tid]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  // the set-up above touched shared memory only: it may overlap the previous launch
  grid_dependency_wait();
  sl_mark(ctl, 1);

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
  grid_launch_dependents();
  sl_mark(ctl, 2);

  auto vec_of = [&](int c, int i) -> int { return c * kSlChunkVecs + i * THREADS + tid; };
  auto load_vec = [&](int v) -> uint4 { return *reinterpret_cast<const uint4*>(smem + static_cast<size_t>(v) * kVecBytes); };
  auto valid_of = [&](int v) -> int { return static_cast<int>(g.n_sl) - v * PV; };
  bool late = false;
#ifdef DSEL_STATS
  int st_tries = 0;   // try_wait calls of this thread (counter builds)
  auto wait_chunk = [&](int c) {
    const uint32_t bar = smem_u32(&bars[c]);
    ++st_tries;
    if (mbar_try_wait(bar, 0u)) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, 0u)) {
      ++st_tries;
      if (global_ns() - t0 > kWaitLimitNs) {
        atomicExch(&g_device_status, DSEL_ERR_DEVICE_TIMEOUT);
        late = true;
        return;
      }
    }
  };
#else
  auto wait_chunk = [&](int c) {
    if (!mbar_wait(smem_u32(&bars[c]), 0u)) late = true;
  };
#endif
  auto next_chunk = [&](int c) -> int {   // the chunk after c in the visiting order
    const uint32_t t = static_cast<uint32_t>(c) + pa;
    return static_cast<int>(t >= static_cast<uint32_t>(g.nch) ? t - static_cast<uint32_t>(g.nch) : t);
  };

  // ---- A. as each chunk lands: every vector's largest key, summarised in 16 bits,
  //      and a histogram of those summaries over fixed bins of 16 summaries
  //      (bin 0 = the largest), the same bins in every CTA of the cluster ----
  int* hv = hist;                  // [kSlVBins]: vector maxima
  int* hc = hist + kSlVBins;       // [kSlBins]: candidate keys
  bool tnan = false;
  uint32_t nacc = 0u;              // NaN-propagating maximum of every whole vector
  uint32_t kmax_c = 0u;            // largest key of the slice
  {
    int c = static_cast<int>(pc);
#pragma unroll 1
    for (int j = 0; j < g.nch; ++j, c = next_chunk(c)) {
      wait_chunk(c);
#ifdef DSEL_STATS
      if (tid == 0) ctl.marks[24 + j] = static_cast<unsigned long long>(clock64());
#endif
#pragma unroll
      for (int i = 0; i < VT; ++i) {
        const int v = vec_of(c, i);
        const int valid = valid_of(v);
        uint32_t s16 = 0u;
        if (valid >= PV) {
          const uint32_t key = vec_max_key_fast<DT>(load_vec(v), nacc);
          s16 = key16<DT>(key);
          kmax_c = max(kmax_c, key);
          atomicAdd(&hv[kSlVBins - 1 - static_cast<int>(s16 >> 4)], 1);
        } else if (valid > 0) {   // the slice's last vector, cut short
          uint32_t key = 0u;
          if (vec_max_valid<DT>(load_vec(v), valid, key)) {
            tnan = true;
          } else {
            s16 = key16<DT>(key);
            kmax_c = max(kmax_c, key);
            atomicAdd(&hv[kSlVBins - 1 - static_cast<int>(s16 >> 4)], 1);
          }
        }
        vkm[v] = static_cast<uint16_t>(s16);   // 0: no element (past the end, or a cut vector with a NaN)
      }
    }
  }
  tnan |= nacc_is_nan<DT>(nacc);
#ifdef DSEL_STATS
  if (lane == 0) atomicAdd(&ctl.marks[13], static_cast<unsigned long long>(st_tries));   // per warp (lane 0)
#endif
  {
    const int f = (__any_sync(0xffffffffu, tnan) ? 1 : 0) | (__any_sync(0xffffffffu, late) ? 4 : 0);
    const uint32_t wk = __reduce_max_sync(0xffffffffu, kmax_c);
    if (lane == 0) {
      if (f) atomicOr(&ctl.flags, f);
      atomicMax(&ctl.kmax, wk);
    }
  }
  int* hvc = hist + kSlVBins + kSlBins;   // coarse sums: vector maxima [256], candidates [64], levels [2][64]
  int* hcc = hvc + kSlVBins / 16;
  __syncthreads();
  coarse_sums<THREADS>(hv, hvc, kSlVBins / 16);
  sl_mark(ctl, 3);
  sl_sync<CLUSTER>(cluster);   // every CTA's vector-maximum histogram, flags and largest key are final
  sl_mark(ctl, 4);
  if ((ctl.flags & 4) && tid < g.nch) mbar_wait(smem_u32(&bars[tid]), 0u);   // a copy may still be landing
  // T: the lowest summary of the bin that holds the k-th largest vector maximum of
  // the row (at least k vectors hold an element >= T: a valid threshold), or 0
  // when the row has fewer than k vectors.  The same step reads the cluster's
  // flags and largest key.
  uint32_t t16 = 0u;
  int flags;
  uint32_t top;   // the row's largest key
  {
    uint32_t fx[2];
    const BinHit bh = cluster_find_bin<THREADS, CLUSTER>(hv, hvc, kSlVBins / 16, k, g.C, ctl, cluster, fx);
    if (bh.bin >= 0) t16 = static_cast<uint32_t>(kSlVBins - 1 - bh.bin) << 4;
    flags = static_cast<int>(fx[0]);
    top = fx[1];
  }
  if ((flags & 1) && !p.nan_flag) nan_trap();   // the pages' default NaN policy
  if (flags & 1) {   // flag mode: the row's NaN sentinel
    if (leader) write_sentinel_row<DT, THREADS>(p, g.row, DSEL_IDX_NAN);
    if (CLUSTER) cluster.sync();   // the peers have read this CTA's control block
    return;
  }
  const uint32_t t_row = DT == DSEL_BF16 ? t16 : (t16 << 16);
  const int sb = res_shift(top - t_row);   // one key per bin for bfloat16 when the range allows
  sl_mark(ctl, 5);

  // ---- B. filter, dense in two steps: the vectors whose summary reaches T into
  //      this warp's vector list (one ballot per vector slot), then their elements
  //      >= T into this warp's element list and the CTA's histogram of candidate
  //      keys (bins counting down from top), 32 vectors per warp step ----
  const uint32_t tb = E::bits_of_key(t_row);
  const uint32_t tv2 = DT == DSEL_BF16 ? (tb | (tb << 16)) : tb;   // T as packed element bits
  const int segv = seg / 2;
  uint32_t* wvec = reinterpret_cast<uint32_t*>(smem + p.off_cv) + warp * segv;
  int vrun = 0;   // vectors of this warp's vector list (warp-uniform)
#pragma unroll 1
  for (int c = 0; c < g.nch; ++c) {
    uint32_t sm[VT];
#pragma unroll
    for (int i = 0; i < VT; ++i) sm[i] = vkm[vec_of(c, i)];
#pragma unroll
    for (int i = 0; i < VT; ++i) {
      const bool cand = sm[i] >= t16 && sm[i] != 0u;
      const unsigned bal = __ballot_sync(0xffffffffu, cand);
      const int pos = vrun + __popc(bal & below);
      if (cand && pos < segv) wvec[pos] = static_cast<uint32_t>(vec_of(c, i));
      vrun += __popc(bal);
    }
  }
  const int vcnt = min(vrun, segv);
  int wrun = 0;   // entries of this warp's element list (warp-uniform)
#pragma unroll 1
  for (int j0 = 0; j0 < vcnt; j0 += 32) {
    const int j = j0 + lane;
    uint32_t m = 0u, v = 0u;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (j < vcnt) {
      v = wvec[j];
      x = load_vec(static_cast<int>(v));
      m = candidate_mask<DT>(x, tv2);
      const int valid = valid_of(static_cast<int>(v));
      if (valid < PV) m &= (1u << valid) - 1u;
    }
    const int cnt = __popc(m);
    const int incl = warp_incl_scan(cnt, lane);
    int pos = wrun + incl - cnt;
#pragma unroll 1
    while (m != 0u) {
      const int e = __ffs(m) - 1;
      m &= m - 1u;
      const uint32_t b = vec_elem_dyn<DT>(x, e);
      atomicAdd(&hc[(top - E::key(b)) >> sb], 1);
      if (pos < seg) {
        wbits[pos] = static_cast<bits_t>(b);
        widx[pos] = g.lo + v * PV + static_cast<uint32_t>(e);
      }
      ++pos;
    }
    wrun += __shfl_sync(0xffffffffu, incl, 31);
  }
  sl_mark(ctl, 6);
  const int wcnt = min(wrun, seg);   // this warp's entries
  if (lane == 0) {
    if (wrun > seg || vrun > segv) atomicOr(&ctl.flags, 2);
    atomicAdd(&ctl.n_list, wcnt);
  }
  __syncthreads();
  coarse_sums<THREADS>(hc, hcc, kSlBins / 16);
  sl_sync<CLUSTER>(cluster);   // every CTA's candidate histogram and list are final
  {   // the block counters of the ranking (in the dead summary table); the search's
      // barriers order this before the count pass (the fallback clears its own bitmaps)
    int* bz = reinterpret_cast<int*>(smem + p.off_tab);
#pragma unroll 1
    for (int i = tid; i < 2 * g.nch * (kSlChunkVecs / 32); i += THREADS) bz[i] = 0;
  }

  // ---- C. the boundary: histogram levels summed over the cluster ----
  auto for_mine = [&](auto&& f) {   // this warp's entries, side by side in its lanes
#pragma unroll 1
    for (int j = lane; j < wcnt; j += 32) f(E::key(wbits[j]), widx[j]);
  };
  uint32_t lo = t_row, hi = top;
  int s = sb, need = k;
  const int* h = hc;
  const int* hcs = hcc;
  bool all_bin;   // the boundary bin is selected whole: every key >= kb
  uint32_t kb;    // else the boundary key K*: every key > K*, and ties in index order
#pragma unroll 1
  for (int level = 0;; ++level) {
    uint32_t fx[2];
    const BinHit bh = cluster_find_bin<THREADS, CLUSTER>(h, hcs, kSlBins / 16, need, g.C, ctl, cluster,
                                                         level == 0 ? fx : nullptr);
    if (level == 0 && (fx[0] & 2u)) {   // a list overflowed (uniform): exact selection on the resident slices
      slice_exact<DT, THREADS, CLUSTER>(p, smem, g.row, g.lo, g.n_sl, g.C, g.crank, t_row, top, cluster);
      return;
    }
    if (bh.bin < 0) {   // cannot happen (the bins hold the row's entries >= lo): select from lo
      all_bin = true;
      kb = lo;
      break;
    }
    need -= bh.before;
    const uint32_t bhi = hi - (static_cast<uint32_t>(bh.bin) << s);
    const uint32_t blo = res_bin_lo(hi, lo, bh.bin, s);
    if (bh.cnt == need || blo == bhi) {
      all_bin = bh.cnt == need;
      kb = blo;
      break;
    }
    lo = blo;
    hi = bhi;
    s = res_shift(hi - lo);
    // levels 1, 2, ... alternate between two buffers in the vector-maximum
    // histogram's space: every CTA read their previous contents before the last
    // cluster barrier
    int* hn = hist + (level & 1) * kSlBins;
    int* hnc = hcc + kSlBins / 16 * (1 + (level & 1));
#pragma unroll 1
    for (int i = tid; i < kSlBins / 4; i += THREADS) reinterpret_cast<int4*>(hn)[i] = make_int4(0, 0, 0, 0);
    __syncthreads();
    for_mine([&](uint32_t kk, uint32_t) {
      if (kk >= lo && kk <= hi) atomicAdd(&hn[(hi - kk) >> s], 1);
    });
    __syncthreads();
    coarse_sums<THREADS>(hn, hnc, kSlBins / 16);
    sl_sync<CLUSTER>(cluster);   // the level's histograms are complete
    h = hn;
    hcs = hnc;
  }
  sl_mark(ctl, 7);
#ifdef DSEL_STATS
  if (tid == 0) {   // threshold summary, list entries
    ctl.marks[14] = static_cast<unsigned long long>(t16);
    ctl.marks[15] = static_cast<unsigned long long>(ctl.n_list);
  }
#endif

  // ---- this slice's share, and per-block counts for the index-order ranks ----
  // Block b (32 consecutive vectors of the slice) belongs to warp b % NW, and each
  // warp's list is in index order, so an entry's rank among this slice's entries
  // of a kind (above the boundary, or equal to it) is the count in earlier blocks
  // plus the warp's running count since the block's first entry.
  const int nblk = g.nch * (kSlChunkVecs / 32);
  int* ba = reinterpret_cast<int*>(smem + p.off_tab);   // [nblk] entries above the boundary, per block
  int* bt = ba + nblk;                                   // [nblk] entries equal to the boundary key
  int* sa = bt + nblk;                                   // [nblk] the owning warp's running counts at
  int* st = sa + nblk;                                   //        the block's first entry
  auto kinds = [&](uint32_t kk, bool& a, bool& t) {
    a = all_bin ? kk >= kb : kk > kb;
    t = !all_bin && kk == kb;
  };
  auto block_of = [&](uint32_t gi) -> int { return static_cast<int>((gi - g.lo) / static_cast<uint32_t>(PV * 32)); };
  {
    int ra = 0, rt = 0, last = -1;   // running counts and block (warp-uniform)
#pragma unroll 1
    for (int j0 = 0; j0 < wcnt; j0 += 32) {
      const int j = j0 + lane;
      const bool valid = j < wcnt;
      bool a = false, t = false;
      int b = -1;
      if (valid) {
        const uint32_t gi = widx[j];
        kinds(E::key(wbits[j]), a, t);
        b = block_of(gi);
      }
      const unsigned am = __ballot_sync(0xffffffffu, a), tm = __ballot_sync(0xffffffffu, t);
      const int prev = __shfl_up_sync(0xffffffffu, b, 1);
      if (valid && b != (lane == 0 ? last : prev)) {   // the block's first entry in this warp's list
        sa[b] = ra + __popc(am & below);
        st[b] = rt + __popc(tm & below);
      }
      if (a) atomicAdd(&ba[b], 1);
      if (t) atomicAdd(&bt[b], 1);
      ra += __popc(am);
      rt += __popc(tm);
      last = __shfl_sync(0xffffffffu, b, 31);
    }
    if (lane == 0) {
      if (ra) atomicAdd(&ctl.x_a, ra);
      if (rt) atomicAdd(&ctl.x_t, rt);
    }
  }
  sl_sync<CLUSTER>(cluster);   // every slice's counts are published
  int off, my_ties;
  {
    const SliceCtl* pr = CLUSTER ? cluster.map_shared_rank(&ctl, lane < g.C ? lane : 0) : &ctl;
    const int ar = lane < g.C ? pr->x_a : 0;
    const int tr = lane < g.C ? pr->x_t : 0;
    const int tin = warp_incl_scan(tr, lane);
    const int take = min(max(need - (tin - tr), 0), tr);   // ties slice `lane` contributes
    const int sel = ar + take;
    const int sin = warp_incl_scan(sel, lane);
    off = __shfl_sync(0xffffffffu, sin - sel, g.crank);
    my_ties = __shfl_sync(0xffffffffu, take, g.crank);
  }
  if (CLUSTER) cluster_arrive();   // done with the peers' shared memory
  sl_mark(ctl, 10);

  // exclusive prefix over the blocks of both counts (nblk <= 8 * 32 <= THREADS... or
  // several blocks per thread)
  {
    constexpr int NW2 = THREADS / 32;
    const int per = (nblk + THREADS - 1) / THREADS;
    const int b0 = min(nblk, tid * per), b1 = min(nblk, b0 + per);
    int xa = 0, xt = 0;
#pragma unroll 1
    for (int b = b0; b < b1; ++b) {
      xa += ba[b];
      xt += bt[b];
    }
    const int ia = warp_incl_scan(xa, lane), it = warp_incl_scan(xt, lane);
    if (lane == 31) {
      ctl.w_a[warp] = static_cast<uint32_t>(ia);
      ctl.w_b[warp] = static_cast<uint32_t>(it);
    }
    __syncthreads();
    int ta, tt;
    int ra = warp_prefix_of<NW2>(reinterpret_cast<const int*>(ctl.w_a), warp, lane, ta) + ia - xa;
    int rt = warp_prefix_of<NW2>(reinterpret_cast<const int*>(ctl.w_b), warp, lane, tt) + it - xt;
#pragma unroll 1
    for (int b = b0; b < b1; ++b) {
      const int ca = ba[b], ct = bt[b];
      ba[b] = ra;
      bt[b] = rt;
      ra += ca;
      rt += ct;
    }
    __syncthreads();
  }
  sl_mark(ctl, 8);

  // ---- output: every selected entry at its rank in index order ----
  {
    const int64_t obase = g.row * static_cast<int64_t>(k);
    int ra = 0, rt = 0;
#pragma unroll 1
    for (int j0 = 0; j0 < wcnt; j0 += 32) {
      const int j = j0 + lane;
      bool a = false, t = false;
      uint32_t gi = 0u, kk = 0u;
      if (j < wcnt) {
        gi = widx[j];
        kk = E::key(wbits[j]);
        kinds(kk, a, t);
      }
      const unsigned am = __ballot_sync(0xffffffffu, a), tm = __ballot_sync(0xffffffffu, t);
      if (a || t) {
        const int b = block_of(gi);
        const int rank_a = ba[b] + ra + __popc(am & below) - sa[b];   // above entries before this one
        const int rank_t = bt[b] + rt + __popc(tm & below) - st[b];   // boundary-key entries before it
        if (a || rank_t < my_ties) {
          const int pos = off + rank_a + min(rank_t, my_ties);
          if (pos < k) {
            if (p.index_i64) static_cast<int64_t*>(p.indices_out)[obase + pos] = static_cast<int64_t>(gi);
            else static_cast<int32_t*>(p.indices_out)[obase + pos] = static_cast<int32_t>(gi);
            if (p.return_value) static_cast<bits_t*>(p.values_out)[obase + pos] = wbits[j];
          }
        }
      }
      ra += __popc(am);
      rt += __popc(tm);
    }
  }
  sl_mark(ctl, 9);
  if (CLUSTER) cluster_wait();   // the peers are done with this CTA's shared memory
}

template <int DT, int THREADS, bool CLUSTER>
__global__ void __launch_bounds__(THREADS, 1) topk_slice_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  slice_body<DT, THREADS, CLUSTER>(p, smem, cluster);
  sl_marks_out(*reinterpret_cast<SliceCtl*>(smem + p.off_ctl));
}

}  // namespace dsel
